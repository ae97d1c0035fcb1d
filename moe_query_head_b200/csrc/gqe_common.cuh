// Internal declarations shared by the GQE CUDA library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/gqe.h"

namespace gqe {

// Tokens per router block: the per-block partial statistics are indexed by this.
constexpr int kRouteBlock = 128;
// Maximum sizes this build supports.
constexpr int kMaxExperts = 64;
constexpr int kMaxTopK = 8;
// The dense projection's routing keeps its bucket cursors in two sets that alternate between
// calls; the set of the next call is a flag in device memory after them (see tc_gemm.cu).
constexpr int kRouteFlag = 2 * kMaxExperts;

// Device status word values (written by kernels whose bounded waits give up).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadInput = 2;  // a decode position outside its cache
constexpr int kStatusBadState = 3;  // routing cursors out of range (never expected)

// Partial-result slots of the decode attention: (sequence, group, key chunk) triples whose
// (m, l, O) are merged by a second kernel. Bounded independently of the cache length (the
// chunks grow with it), so the handle's workspace holds them.
constexpr int kDecodeSlots = 4096;

// ---------------------------------------------------------------------------------------
// Programmatic dependent launch. The forward's kernels are launched with it: a kernel may
// begin (its set-up: barriers, TMEM, tensor-map prefetch) while the previous kernel on the
// stream finishes, and waits for that kernel's completion and memory (pdl_wait) before it
// touches global memory. pdl_allow_next lets the next kernel begin launching.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// The dynamic shared-memory limit of a kernel is a per-device attribute: set it on the
// current device the first time that device launches the kernel (one flag per kernel and
// device, under a lock, so concurrent callers and handles on several devices are safe).
template <auto Kernel>
inline bool set_smem_limit_once(int smem) {
  static std::mutex mu;
  static uint64_t done = 0;  // bit d: set on device d (ordinals 0..63)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev < 0 || dev >= 64)
    return cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) ==
           cudaSuccess;
  std::lock_guard<std::mutex> lock(mu);
  if ((done >> dev) & 1u) return true;
  if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return false;
  done |= uint64_t(1) << dev;
  return true;
}

// ---------------------------------------------------------------------------------------
// Element access helpers: every kernel computes in fp32; storage is float or bf16.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Affine map from a GEMM output element (row m, column c) to memory: column c belongs to
// head c / head_w at offset c % head_w; address = base + head*head_stride + m*row_stride
// + (c % head_w)*col_stride (in elements of the output type).
struct OutMap {
  void* base;
  int64_t head_stride;
  int64_t row_stride;
  int64_t col_stride;
  int head_w;
  int f32;  // 1: store float; 0: store the handle's storage type
};

// ---------------------------------------------------------------------------------------
// The handle.
// ---------------------------------------------------------------------------------------
struct Workspace {
  void* K = nullptr;        // [G, M, d_h]
  void* V = nullptr;        // [G, M, d_h]
  void* Q = nullptr;        // [S, M, d_h]
  void* Z = nullptr;        // [M, D_o]
  float* lse = nullptr;     // [S, M] attention log2-sum-exp2 per (stream, token) (bf16 path)
  float* logits = nullptr;  // [M, N]
  int32_t* sel = nullptr;   // [M, G, k]
  float* psel = nullptr;    // [M, G, k]
  float* gates = nullptr;   // [M, G, k]
  float* w = nullptr;       // [M, G, k]
  int32_t* part_counts = nullptr;  // [nblk, N]; after the scan: bucket base of (blk, e)
  float* part_prob = nullptr;      // [nblk, N]
  int32_t* counts = nullptr;       // [N]
  float* mean_prob = nullptr;      // [N]
  int32_t* offsets = nullptr;      // [N + 1] bucket start of each expert (e M)
  int32_t* bucket = nullptr;       // [N * M] entries (token << 3) | rank; expert e's run of
                                   // counts[e] entries starts at e M
  int2* tile_list = nullptr;       // routed-projection tiles (expert | rows << 8, first slot)
  int32_t* tile_count = nullptr;   // number of routed-projection tiles
  int32_t* attn_counter = nullptr; // attention work-item counter
  // dense-projection routing: two sets (alternate calls) of bucket cursors and
  // fixed-point probability sums; a call's set is zero when it starts
  int32_t* rcur = nullptr;                // [2, kMaxExperts] cursors, then the set flag and an
                                          // exit counter (kRouteFlag, kRouteFlag + 1)
  unsigned long long* rpsum = nullptr;    // [2, kMaxExperts]
  int32_t* cursor = nullptr;       // [kMaxExperts] bucket cursors, then the routing ticket
                                   // (zero between calls)
  float* dec_part = nullptr;       // [kDecodeSlots, k + 1, d_h + 2] decode partial (m, l, O)
  int32_t* status = nullptr;       // device status word
  void* base = nullptr;            // the single allocation
  size_t bytes = 0;
};

// Backward-pass workspace (gqe_enable_backward), sized for max_tokens.
struct BwdBuffers {
  float* dZ = nullptr;                // [M, D_o] gradient of the concatenation
  __nv_bfloat16* dO = nullptr;        // [S, M, d_h] gradients of the stream outputs
  float* dsum = nullptr;              // [S, M] rowsum(dO * O)
  __nv_bfloat16* dl = nullptr;        // [M, N] gradient of the router logits
  __nv_bfloat16* dq_exp = nullptr;    // [M, N d_h] routed query gradients at their expert
  __nv_bfloat16* dq_sh = nullptr;     // [M, d_h] shared-head query gradient
  __nv_bfloat16* dk = nullptr;        // [M, G d_h] key gradients, token-major
  __nv_bfloat16* dv = nullptr;        // [M, G d_h] value gradients, token-major
  float* dgs = nullptr;               // [M, G k] per routed stream: dw (gqe), dp (weighted)
  float* slot_dot = nullptr;          // [M] <dslot, slot> of a whole-layer backward
  int* counter = nullptr;             // [4] work counters of the two attention kernels
  void* cublas_ws = nullptr;          // cuBLAS workspace
};

}  // namespace gqe

struct gqe_ctx {
  int dim, N, G, k, d_h, E;
  // the groups this handle computes, [g0, g1) (gqe_set_group_range; all G by default)
  int g0 = 0, g1 = 0;
  gqe_dtype dtype;
  int64_t max_tokens;
  int esz;  // bytes per stored element
  int device;
  int num_sms;
  int64_t spin_limit;
  gqe::Workspace ws;
  // measurement: events recorded around the stages (GQE_NUM_STAGES + 1, or none)
  cudaEvent_t stage_events[GQE_NUM_STAGES + 1] = {};
  int n_stage_events = 0;
  // state of the last forward
  int last_M = 0, last_S = 0, last_Do = 0, last_launches = 0;
  // what the last call was (1 gqe_forward, 2 gqe_decode) and its arguments, which a
  // gqe_backward must repeat
  int last_kind = 0, last_B = 0, last_T = 0, last_variant = -1, last_causal = -1,
      last_shared = -1, last_g0 = -1, last_g1 = -1;
  // backward pass (gqe_enable_backward)
  void* bwd_base = nullptr;
  size_t bwd_bytes = 0;
  void* cublas = nullptr;  // cublasHandle_t
  gqe::BwdBuffers bwd;
  int last_bwd_launches = 0;
  // the last gqe_backward_begin (checked by gqe_backward_finish): M, variant, and 1 once
  // it succeeded
  int bwd_begun = 0, bwd_M = 0, bwd_variant = -1;
};

namespace gqe {

// Router kernels (defined in route.cu), also launched by the static-scratch entry point.
__global__ void __launch_bounds__(kRouteBlock)
route_select_kernel(const float* __restrict__ logits, int M, int N, int G,
                                    int k, int32_t* __restrict__ sel, float* __restrict__ psel,
                                    float* __restrict__ gates, float* __restrict__ wslot,
                                    int32_t* __restrict__ part_counts,
                                    float* __restrict__ part_prob);
__global__ void __launch_bounds__(1024)
route_scan_aux_kernel(int32_t* __restrict__ part_counts,
                                      const float* __restrict__ part_prob, int nblk, int M,
                                      int N, int G, int k, int32_t* __restrict__ counts,
                                      float* __restrict__ mean_prob,
                                      int32_t* __restrict__ offsets, float* __restrict__ aux_out);

// Launchers implemented in the .cu files. Each returns the number of kernels launched
// (>= 0) or -1 if a launch failed.
int launch_simt_dense_proj(gqe_ctx* h, const void* x, int M, const void* W_r, const void* W_k,
                           const void* W_v, const void* W_shared, cudaStream_t st);
int launch_route_select(gqe_ctx* h, int M, cudaStream_t st);
int launch_route_fused(gqe_ctx* h, int M, float* aux_out, cudaStream_t st);
int launch_route_scan_aux(gqe_ctx* h, int M, float* aux_out, cudaStream_t st);
int launch_bucket(gqe_ctx* h, int M, cudaStream_t st);
int launch_simt_qproj(gqe_ctx* h, const void* x, int M, const void* W_q, cudaStream_t st);
int launch_simt_attention(gqe_ctx* h, int B, int T, int S, int has_shared, int variant,
                          int causal, int Do, cudaStream_t st);
int launch_combine(gqe_ctx* h, int M, int variant, int Do, cudaStream_t st);
int launch_simt_oproj(gqe_ctx* h, int M, int Do, const void* W_o, void* out, cudaStream_t st);
// tcgen05 paths (bf16)
int launch_tc_dense_proj(gqe_ctx* h, const void* x, int M, const void* W_r, const void* W_k,
                         const void* W_v, const void* W_shared, cudaStream_t st);
bool tc_dense_routes(const gqe_ctx* h);  // launch_tc_dense_proj also routes
int launch_tc_qproj(gqe_ctx* h, const void* x, int M, const void* W_q, bool from_cursors,
                    float* aux_out, cudaStream_t st);
int launch_tc_oproj(gqe_ctx* h, int M, int Do, const void* W_o, void* out, cudaStream_t st);
int launch_tc_attention(gqe_ctx* h, int B, int T, int S, int has_shared, int variant,
                        int causal, int Do, cudaStream_t st);
// Decode step: attention of one new token per sequence over its KV cache, and the append of
// the new token's K/V (decode.cu). bf16 handles.
int launch_tc_decode_attention(gqe_ctx* h, int B, int S, int has_shared, int variant, int Do,
                               void* k_cache, void* v_cache, int L_max, const int32_t* lengths,
                               cudaStream_t st);
int decode_chunks(const gqe_ctx* h, int B, int L_max);
// Backward pass (tc_attention_bwd.cu, backward.cu): bf16 handles with d_h <= 64.
bool tc_backward_supported(const gqe_ctx* h);
int launch_tc_attention_backward(gqe_ctx* h, const BwdBuffers& bb, int B, int T, int S,
                                 int has_shared, int causal, cudaStream_t st);
void backward_release(gqe_ctx* h);

}  // namespace gqe
