// Diagnostic entry point: the FMA-pipe exp2 that the attention softmax uses for part of its
// exponentials, applied elementwise, so tests can compare it with CUDA's exp2f.
#include "exp2_fma.cuh"
#include "gqe_common.cuh"

namespace {

__global__ void exp2_fma_kernel(const float* __restrict__ in, float* __restrict__ out, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = gqe::tc::exp2_fma2(make_float2(in[i], in[i + 1]));
    out[i] = r.x;
    out[i + 1] = r.y;
  } else if (i < n) {
    out[i] = gqe::tc::exp2_fma2(make_float2(in[i], in[i])).x;
  }
}

}  // namespace

extern "C" gqe_status gqe_exp2_fma(const float* in, float* out, int n, void* stream) {
  if (!in || !out || n < 0) return GQE_ERR_INVALID_ARG;
  if (n == 0) return GQE_OK;
  const int pairs = (n + 1) / 2;
  exp2_fma_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(in, out, n);
  return cudaGetLastError() == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Self-test of the failure-detection path: one warp waits, with the same bounded mbarrier
// wait the pipeline kernels use, on a barrier phase that nothing will complete. When the
// wait gives up it writes the timeout code to the handle's device status word, exactly as a
// pipeline kernel does, and the CTA returns. Nothing traps, spins without bound or leaves
// asynchronous copies in flight.
// ---------------------------------------------------------------------------------------
namespace {

__global__ void wait_timeout_kernel(int32_t* status, int64_t spin) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    gqe::tc::mbar_init(&bar, 1);  // expects one arrival; none is ever made
    gqe::tc::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = !__any_sync(0xffffffffu, !gqe::tc::mbar_wait(&bar, 0, spin));
  if (!ok && threadIdx.x == 0) atomicExch(status, gqe::kStatusTimeout);
}

}  // namespace

extern "C" gqe_status gqe_selftest_timeout(gqe_handle h, int64_t spin, void* stream) {
  if (!h || spin < 1) return GQE_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->ws.status, spin);
  return cudaGetLastError() == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}
