// gqe_route_static: the router's selection and load statistics from precomputed router
// logits, with all scratch memory in a fixed, file-scope device array instead of memory
// the caller or the library allocates.
//
// Who needs it: callers that cannot call cudaMalloc. Some run inside a host framework
// whose device memory belongs to another allocator (a caching allocator that must account
// for every byte, or a fixed memory budget carved out at start-up); some are plug-in or
// callback code that receives only its input and output buffers and has no allocation
// API; some are latency-critical paths where cudaMalloc's implicit device-wide
// synchronisation is not acceptable. gqe_create allocates a workspace, so those callers
// could not use the router otherwise. The paper has no counterpart of this entry point.
//
// The scratch holds the per-block partial token counts and probability sums, the bucket
// offsets, and the per-(token, group) selected probabilities and slot weights that the
// router kernel also writes. Its size is fixed below; every GPU that loads this library
// holds it until the process exits.
#include <mutex>

#include "gqe_common.cuh"

namespace {

using namespace gqe;

// Limits of the static scratch (see gqe.h): tokens, and token x selection entries.
constexpr int kStaticMaxTokens = 1 << 17;                        // 131072 tokens
constexpr int kStaticMaxEntries = 1 << 18;                       // M * G * k <= 262144
constexpr int kStaticMaxBlocks = kStaticMaxTokens / kRouteBlock;  // 1024 router blocks

constexpr size_t kOffPsel = 0;
constexpr size_t kOffW = kOffPsel + sizeof(float) * kStaticMaxEntries;
constexpr size_t kOffPartCounts = kOffW + sizeof(float) * kStaticMaxEntries;
constexpr size_t kOffPartProb = kOffPartCounts + sizeof(int32_t) * kStaticMaxBlocks * kMaxExperts;
constexpr size_t kOffOffsets = kOffPartProb + sizeof(float) * kStaticMaxBlocks * kMaxExperts;
// offsets: N + 1 <= kMaxExperts + 1 int32, rounded up to the array's 256-byte alignment
constexpr size_t kOffsetsBytes = (sizeof(int32_t) * (kMaxExperts + 1) + 255) / 256 * 256;
constexpr size_t kScratchBytes = kOffOffsets + kOffsetsBytes;
static_assert(kScratchBytes >= kOffOffsets + sizeof(int32_t) * (kMaxExperts + 1),
              "the scratch must hold offsets[0 .. kMaxExperts]");

// The scratch. In host code this name is only a host-side stand-in for the symbol, not a
// device address: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device.
gqe_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return GQE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return GQE_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GQE_OK;
}

}  // namespace

extern "C" gqe_status gqe_route_static(const float* logits, int M, int N, int G, int k,
                                       int32_t* sel, float* gates, int32_t* counts,
                                       float* mean_prob, float* aux_loss, void* stream) {
  if (!logits || !sel || !gates || !counts || !mean_prob) return GQE_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || G < 1 || k < 1 || N % G != 0 || k > N / G) return GQE_ERR_INVALID_ARG;
  if (N > kMaxExperts || k > kMaxTopK) return GQE_ERR_UNSUPPORTED;
  if (M > kStaticMaxTokens || (int64_t)M * G * k > kStaticMaxEntries) return GQE_ERR_WORKSPACE;
  void* base = nullptr;
  gqe_status s = scratch_address(&base);
  if (s != GQE_OK) return s;
  char* b = static_cast<char*>(base);
  float* psel = reinterpret_cast<float*>(b + kOffPsel);
  float* wslot = reinterpret_cast<float*>(b + kOffW);
  int32_t* part_counts = reinterpret_cast<int32_t*>(b + kOffPartCounts);
  float* part_prob = reinterpret_cast<float*>(b + kOffPartProb);
  int32_t* offsets = reinterpret_cast<int32_t*>(b + kOffOffsets);
  // Nothing in the scratch needs clearing: every element a call reads was written earlier
  // in the same call (each router block writes all N of its partials).
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  route_select_kernel<<<nblk, kRouteBlock, 0, st>>>(logits, M, N, G, k, sel, psel, gates, wslot,
                                                     part_counts, part_prob);
  if (cudaGetLastError() != cudaSuccess) return GQE_ERR_CUDA;
  route_scan_aux_kernel<<<1, 1024, 0, st>>>(part_counts, part_prob, nblk, M, N, G, k,
                                                    counts, mean_prob, offsets, aux_loss);
  if (cudaGetLastError() != cudaSuccess) return GQE_ERR_CUDA;
  return GQE_OK;
}
