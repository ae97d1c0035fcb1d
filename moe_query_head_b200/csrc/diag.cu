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
