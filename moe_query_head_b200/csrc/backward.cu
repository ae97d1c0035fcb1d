// Backward pass of one GQE attention layer: gqe_enable_backward, gqe_backward and its two
// phases gqe_backward_begin / gqe_backward_finish.
//
// Training adds the load-balancing loss to the task loss and back-propagates through the
// layer ("GQE: Grouped Query Experts" README, Usage); the renormalised slot gives the router
// a differentiable path (gist.science summary, Output Construction). Given dy = dF/dy and the
// aux coefficient dA, the gradients of F = <dy, y> + dA L are formed in this order:
//   phase 1 (begin)
//   1. dZ = dy W_o                                              (plain GEMM, cuBLAS)
//   2. combine_bwd_kernel, one warp per token: the stream gradients dO from dZ by variant
//      (routed blocks, the slot's share w dslot, the shared block), D = rowsum(dO * O), and
//      per routed stream dw = <dslot, O> (gqe) or dp = <dZ, O> (weighted_concat); for gqe
//      also <dslot, slot> = sum over the streams of w dw
//   3. the attention backward (tc_attention_bwd.cu): dQ into dQ_exp [M, N d_h] (each routed
//      row at the column block of its expert, zero elsewhere) and dQ_sh, dK and dV [M, G d_h]
//   phase 2 (finish)
//   4. router_bwd_kernel, one warp per token: the selected probabilities' gradients (for gqe
//      the slot weights w = p_sel / P_t differentiated with their denominator:
//      dp_sel = (dw - <dslot, slot>) / P_t), the aux term dA (E/G) f / M on every p, and the
//      per-group softmax Jacobian: the router logits' gradient dl [M, N]
//   5. dW_o = dy^T Z, the weight gradients dW = (gradient)^T x and dx = sum of (gradient) W
//      over the router, the query heads (dQ_exp: the unselected heads' blocks are zero, so one
//      dense GEMM serves every expert), the K, V and shared projections (plain GEMMs, cuBLAS)
// The top-k selection is held constant (its sets are the forward's).
//
// A handle restricted to groups [g0, g1) (gqe_set_group_range) computes its share: every
// step above is local to its groups except <dslot, slot>, which sums over all of the
// layer's streams; phase 1 writes this handle's share of it, the caller sums the shares over
// the ranges, and phase 2 takes the sum. The router gradient of the other groups is zero
// here, so the layer's gradients are the sums of the ranges' shares.
#include <cublas_v2.h>
#include <string.h>

#include "gqe_common.cuh"

namespace gqe {

namespace {

struct CombBwd {
  const float* dZ;          // [M, Do] this handle's Z columns
  const __nv_bfloat16* Z;   // [M, Do]
  const float* psel;        // [M, gk] the layer's routing (every group)
  const float* w;           // [M, gk]
  const int32_t* sel;       // [M, gk]
  const float* logits;      // [M, N]
  const int32_t* counts;    // [N]
  __nv_bfloat16* dO;        // [S, M, d_h] this handle's streams
  float* dsum;              // [S, M]
  float* dgs;               // [M, Sr] per routed stream of this handle: dw (gqe), dp (weighted)
  float* slot_dot;          // [M] phase 1: this handle's share of <dslot, slot>
  const float* slot_dot_in; // [M] phase 2: the sum over the layer's ranges
  __nv_bfloat16* dl;        // [M, N]
  int M, N, G, E, k, d_h, Do, variant, has_shared, shared_col;
  int gk;                   // G k: row stride of the routing arrays
  int g0, g1;               // this handle's groups
  int Sr;                   // its routed streams, (g1 - g0) k, numbered from group g0
  float dA;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

constexpr int kCombWarps = 8;

// Phase 1, one warp per token; lane l holds head dims l, l + 32, l + 64 and l + 96
// (d_h <= 128).
constexpr int kDimsPerLane = 4;
__global__ void __launch_bounds__(kCombWarps * 32) combine_bwd_kernel(const CombBwd P) {
  pdl_wait();
  pdl_allow_next();
  const int wi = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t = (int64_t)blockIdx.x * kCombWarps + wi;
  if (t >= P.M) return;
  const int DH = P.d_h;
  bool v[kDimsPerLane];
#pragma unroll
  for (int h = 0; h < kDimsPerLane; ++h) v[h] = lane + 32 * h < DH;
  const float* dz = P.dZ + t * P.Do;
  const __nv_bfloat16* z = P.Z + t * P.Do;
  const bool gqe = P.variant == GQE_VARIANT_GQE;
  const bool wcat = P.variant == GQE_VARIANT_WEIGHTED_CONCAT;
  const int64_t rt = t * P.gk + (int64_t)P.g0 * P.k;  // this handle's first stream's routing
  float ds[kDimsPerLane];  // the slot's gradient
#pragma unroll
  for (int h = 0; h < kDimsPerLane; ++h)
    ds[h] = (gqe && v[h]) ? dz[P.Sr * DH + lane + 32 * h] : 0.f;
  float dot = 0.f;  // <dslot, slot> over this handle's streams: sum of w dw
  // routed streams
  for (int s = 0; s < P.Sr; ++s) {
    const int c = s * DH;
    float o[kDimsPerLane], d[kDimsPerLane];
    float gs = 0.f, dd = 0.f;
    const float p = wcat ? P.psel[rt + s] : 1.f;
    const float ww = gqe ? P.w[rt + s] : 0.f;
#pragma unroll
    for (int h = 0; h < kDimsPerLane; ++h) {
      o[h] = v[h] ? __bfloat162float(z[c + lane + 32 * h]) : 0.f;
      const float b = v[h] ? dz[c + lane + 32 * h] : 0.f;
      if (wcat) {
        // Z holds p O: O = Z / p; dO = p dZ; dp = <dZ, O>
        o[h] /= p;
        d[h] = p * b;
        gs += b * o[h];
      } else if (gqe) {
        // dO = dZ + w dslot; dw = <dslot, O>
        d[h] = fmaf(ww, ds[h], b);
        gs += ds[h] * o[h];
      } else {
        d[h] = b;
      }
      // D from the bf16 dO the attention backward reads
      d[h] = bf16_round(d[h]);
      dd += d[h] * o[h];
    }
    gs = (wcat || gqe) ? warp_sum(gs) : 0.f;
    dot = fmaf(gs, ww, dot);
    const float D = warp_sum(dd);
    __nv_bfloat16* dst = P.dO + ((int64_t)s * P.M + t) * DH;
#pragma unroll
    for (int h = 0; h < kDimsPerLane; ++h)
      if (v[h]) dst[lane + 32 * h] = __float2bfloat16_rn(d[h]);
    if (lane == 0) {
      P.dsum[(int64_t)s * P.M + t] = D;
      P.dgs[t * P.Sr + s] = gs;
    }
  }
  if (lane == 0) P.slot_dot[t] = dot;
  if (P.has_shared) {
    const int c = P.shared_col;
    float d[kDimsPerLane], dd = 0.f;
#pragma unroll
    for (int h = 0; h < kDimsPerLane; ++h) {
      const float o = v[h] ? __bfloat162float(z[c + lane + 32 * h]) : 0.f;
      d[h] = v[h] ? bf16_round(dz[c + lane + 32 * h]) : 0.f;
      dd += d[h] * o;
    }
    const float D = warp_sum(dd);
    __nv_bfloat16* dst = P.dO + ((int64_t)P.Sr * P.M + t) * DH;
#pragma unroll
    for (int h = 0; h < kDimsPerLane; ++h)
      if (v[h]) dst[lane + 32 * h] = __float2bfloat16_rn(d[h]);
    if (lane == 0) P.dsum[(int64_t)P.Sr * P.M + t] = D;
  }
}

// Phase 2, one warp per token: the router logits' gradient of this handle's groups (zero
// for the others).
__global__ void __launch_bounds__(kCombWarps * 32) router_bwd_kernel(const CombBwd P) {
  __shared__ float s_g[kCombWarps][kMaxExperts];  // per routed stream: dp_sel
  pdl_wait();
  pdl_allow_next();
  const int wi = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t t = (int64_t)blockIdx.x * kCombWarps + wi;
  if (t >= P.M) return;
  const bool gqe = P.variant == GQE_VARIANT_GQE;
  const bool wcat = P.variant == GQE_VARIANT_WEIGHTED_CONCAT;
  float* g = s_g[wi];
  if (gqe) {
    // w = p_sel / P_t over the layer's G k selections: dp_sel = (dw - sum(dw w)) / P_t,
    // sum(dw w) = <dslot, slot>
    float pt = 0.f;
    for (int s = lane; s < P.gk; s += 32) pt += P.psel[t * P.gk + s];
    pt = warp_sum(pt);
    const float dot = P.slot_dot_in[t];
    for (int s = lane; s < P.Sr; s += 32) g[s] = (P.dgs[t * P.Sr + s] - dot) / pt;
  } else {
    for (int s = lane; s < P.Sr; s += 32) g[s] = wcat ? P.dgs[t * P.Sr + s] : 0.f;
  }
  __syncwarp();
  // router logits: dp on every p of the group (selected terms and the aux term), then the
  // per-group softmax Jacobian dl = p (dp - sum p dp)
  const float aux_c = P.dA * (float)P.E / (float)P.G / ((float)P.M * (float)P.k * (float)P.M);
  for (int gg = 0; gg < P.G; ++gg) {
    const int e0 = gg * P.E;
    if (gg < P.g0 || gg >= P.g1) {
      // another range's group
      for (int j = lane; j < P.E; j += 32) P.dl[t * P.N + e0 + j] = __float2bfloat16_rn(0.f);
      continue;
    }
    const int32_t* sl = P.sel + t * P.gk + gg * P.k;  // the group's selections
    const float* gsel = g + (gg - P.g0) * P.k;          // and their dp_sel
    for (int jb = 0; jb < P.E; jb += 32) {
      const int j = jb + lane;
      const bool in = j < P.E;
      const float l = in ? P.logits[t * P.N + e0 + j] : -INFINITY;
      // the group's softmax over all E experts (E may exceed 32: reduce over the chunks)
      float mx = -INFINITY;
      for (int jj = lane; jj < P.E; jj += 32) mx = fmaxf(mx, P.logits[t * P.N + e0 + jj]);
      mx = warp_max(mx);
      float den = 0.f;
      for (int jj = lane; jj < P.E; jj += 32) den += expf(P.logits[t * P.N + e0 + jj] - mx);
      den = warp_sum(den);
      const float p = in ? expf(l - mx) / den : 0.f;
      float dp = in ? aux_c * (float)P.counts[e0 + j] : 0.f;
      for (int r = 0; r < P.k; ++r)
        if (in && sl[r] == j) dp += gsel[r];
      // sum over the group of p dp
      float spd = 0.f;
      for (int jj = lane; jj < P.E; jj += 32) {
        const float lj = P.logits[t * P.N + e0 + jj];
        const float pj = expf(lj - mx) / den;
        float dpj = aux_c * (float)P.counts[e0 + jj];
        for (int r = 0; r < P.k; ++r)
          if (sl[r] == jj) dpj += gsel[r];
        spd += pj * dpj;
      }
      spd = warp_sum(spd);
      if (in) P.dl[t * P.N + e0 + j] = __float2bfloat16_rn(p * (dp - spd));
    }
  }
}

// Row-major C[m x n] (fp32) = op(A)[m x k] op(B)[k x n] + beta C, bf16 operands: the
// column-major call computes C^T = op(B)^T op(A)^T with the same transpose letters.
bool gemm_rm(cublasHandle_t hb, bool ta, bool tb, int m, int n, int k, const void* A, int lda,
             const void* B, int ldb, float* C, int ldc, float beta) {
  const float alpha = 1.f;
  return cublasGemmEx(hb, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, n, m,
                      k, &alpha, B, CUDA_R_16BF, ldb, A, CUDA_R_16BF, lda, &beta, C,
                      CUDA_R_32F, ldc, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) ==
         CUBLAS_STATUS_SUCCESS;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
constexpr size_t kCublasWorkspace = size_t(32) << 20;

// Backward workspace layout; with base == nullptr only the size.
size_t bwd_layout(BwdBuffers& b, char* base, const gqe_ctx* h) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const int64_t M = h->max_tokens;
  const int64_t S = (int64_t)h->G * h->k + 1;
  const int64_t Do = ((int64_t)h->G * h->k + 2) * h->d_h;
  b.dZ = (float*)take((size_t)M * Do * 4);
  b.dO = (__nv_bfloat16*)take((size_t)S * M * h->d_h * 2);
  b.dsum = (float*)take((size_t)S * M * 4);
  b.dl = (__nv_bfloat16*)take((size_t)M * h->N * 2);
  b.dq_exp = (__nv_bfloat16*)take((size_t)M * h->N * h->d_h * 2);
  b.dq_sh = (__nv_bfloat16*)take((size_t)M * h->d_h * 2);
  b.dk = (__nv_bfloat16*)take((size_t)M * h->G * h->d_h * 2);
  b.dv = (__nv_bfloat16*)take((size_t)M * h->G * h->d_h * 2);
  b.dgs = (float*)take((size_t)M * h->G * h->k * 4);
  b.slot_dot = (float*)take((size_t)M * 4);
  b.counter = (int*)take(16 * sizeof(int));
  b.cublas_ws = take(kCublasWorkspace);
  return off;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sizes of one backward call on this handle's groups.
struct BwdCall {
  int M, S, Do, Sr, Gl, Nl, has_shared;
};

// The arguments both phases take: checked against the handle and its last forward (which
// must be a gqe_forward with the same x, weights, B, T, variant, causal, presence of W_shared
// and group range).
gqe_status check_call(const gqe_ctx* h, const void* x, int B, int T, const void* W_r,
                      const void* W_q, const void* W_k, const void* W_v, const void* W_shared,
                      const void* W_o, int N, int G, int k, int d_h, int variant, int causal,
                      const void* dy, BwdCall& c) {
  if (!h->bwd_base) return GQE_ERR_INVALID_ARG;  // gqe_enable_backward first
  if (N != h->N || G != h->G || k != h->k || d_h != h->d_h) return GQE_ERR_INVALID_ARG;
  if (B < 1 || T < 1) return GQE_ERR_INVALID_ARG;
  if (variant < GQE_VARIANT_GQE || variant > GQE_VARIANT_HARD_CONCAT) return GQE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return GQE_ERR_INVALID_ARG;
  if (!x || !W_r || !W_q || !W_k || !W_v || !W_o || !dy) return GQE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_r, W_q, W_k, W_v, W_o, dy};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GQE_ERR_INVALID_ARG;
  if (W_shared && !aligned16(W_shared)) return GQE_ERR_INVALID_ARG;
  const int64_t M64 = (int64_t)B * T;
  if (M64 > h->max_tokens) return GQE_ERR_WORKSPACE;
  c.M = (int)M64;
  c.has_shared = W_shared != nullptr;
  // the saved state must be this layer's last forward, on the same groups
  if (h->last_kind != 1 || h->last_M != c.M || h->last_B != B || h->last_T != T ||
      h->last_variant != variant || h->last_causal != causal ||
      h->last_shared != c.has_shared || h->last_g0 != h->g0 || h->last_g1 != h->g1)
    return GQE_ERR_INVALID_ARG;
  c.Gl = h->g1 - h->g0;
  c.Sr = c.Gl * k;
  c.Nl = c.Gl * h->E;
  c.S = c.Sr + c.has_shared;
  c.Do = (c.Sr + (variant == GQE_VARIANT_GQE ? 1 : 0) + c.has_shared) * d_h;
  return GQE_OK;
}

CombBwd comb_args(const gqe_ctx* h, const BwdCall& c, int variant, float aux_grad) {
  const BwdBuffers& b = h->bwd;
  CombBwd a;
  memset(&a, 0, sizeof(a));
  a.dZ = b.dZ;
  a.Z = static_cast<const __nv_bfloat16*>(h->ws.Z);
  a.psel = h->ws.psel;
  a.w = h->ws.w;
  a.sel = h->ws.sel;
  a.logits = h->ws.logits;
  a.counts = h->ws.counts;
  a.dO = b.dO;
  a.dsum = b.dsum;
  a.dgs = b.dgs;
  a.dl = b.dl;
  a.M = c.M;
  a.N = h->N;
  a.G = h->G;
  a.E = h->E;
  a.k = h->k;
  a.d_h = h->d_h;
  a.Do = c.Do;
  a.variant = variant;
  a.has_shared = c.has_shared;
  a.shared_col = (c.Sr + (variant == GQE_VARIANT_GQE ? 1 : 0)) * h->d_h;
  a.gk = h->G * h->k;
  a.g0 = h->g0;
  a.g1 = h->g1;
  a.Sr = c.Sr;
  a.dA = aux_grad;
  return a;
}

// Phase 1: dZ, the stream gradients and this handle's share of <dslot, slot> (slot_dot
// [M], device), the attention backward.
gqe_status phase1(gqe_ctx* h, const BwdCall& c, int B, int T, const void* W_o, int variant,
                  int causal, const void* dy, float* slot_dot, cudaStream_t st) {
  cublasHandle_t hb = static_cast<cublasHandle_t>(h->cublas);
  if (cublasSetStream(hb, st) != CUBLAS_STATUS_SUCCESS) return GQE_ERR_CUDA;
  const BwdBuffers& b = h->bwd;
  const int dim = h->dim, d_h = h->d_h;
  int launches = 0;
  bool ok = gemm_rm(hb, false, false, c.M, c.Do, dim, dy, dim, W_o, c.Do, b.dZ, c.Do, 0.f);
  // dQ_exp is zero outside the selected heads' blocks
  ok = ok && cudaMemsetAsync(b.dq_exp, 0, (size_t)c.M * c.Nl * d_h * 2, st) == cudaSuccess;
  if (ok) {
    CombBwd a = comb_args(h, c, variant, 0.f);
    a.slot_dot = slot_dot;
    combine_bwd_kernel<<<(c.M + kCombWarps - 1) / kCombWarps, kCombWarps * 32, 0, st>>>(a);
    ok = cudaGetLastError() == cudaSuccess;
    ++launches;
  }
  if (ok) {
    const int n = launch_tc_attention_backward(h, b, B, T, c.S, c.has_shared, causal, st);
    ok = n >= 0;
    launches += n > 0 ? n : 0;
  }
  h->last_bwd_launches = launches;
  h->bwd_begun = ok ? 1 : 0;
  h->bwd_M = c.M;
  h->bwd_variant = variant;
  return ok ? GQE_OK : GQE_ERR_CUDA;
}

// Phase 2: the router backward with <dslot, slot> summed over the layer (slot_dot_in [M],
// device), dW_o, the weight gradients and dx.
gqe_status phase2(gqe_ctx* h, const BwdCall& c, const void* x, const void* W_r,
                  const void* W_q, const void* W_k, const void* W_v, const void* W_shared,
                  int variant, const void* dy, float aux_grad, const float* slot_dot_in,
                  float* dx, float* dW_r, float* dW_q, float* dW_k, float* dW_v,
                  float* dW_shared, float* dW_o, cudaStream_t st) {
  if (!h->bwd_begun || h->bwd_M != c.M || h->bwd_variant != variant) return GQE_ERR_INVALID_ARG;
  h->bwd_begun = 0;
  cublasHandle_t hb = static_cast<cublasHandle_t>(h->cublas);
  if (cublasSetStream(hb, st) != CUBLAS_STATUS_SUCCESS) return GQE_ERR_CUDA;
  const BwdBuffers& b = h->bwd;
  const int dim = h->dim, d_h = h->d_h, N = h->N, M = c.M;
  bool ok = true;
  {
    CombBwd a = comb_args(h, c, variant, aux_grad);
    a.slot_dot_in = slot_dot_in;
    router_bwd_kernel<<<(M + kCombWarps - 1) / kCombWarps, kCombWarps * 32, 0, st>>>(a);
    ok = cudaGetLastError() == cudaSuccess;
    ++h->last_bwd_launches;
  }
  const int Nd = c.Nl * d_h, Gd = c.Gl * d_h;
  ok = ok && gemm_rm(hb, true, false, dim, c.Do, M, dy, dim, h->ws.Z, c.Do, dW_o, c.Do, 0.f);
  ok = ok && gemm_rm(hb, true, false, Nd, dim, M, b.dq_exp, Nd, x, dim, dW_q, dim, 0.f);
  ok = ok && gemm_rm(hb, true, false, Gd, dim, M, b.dk, Gd, x, dim, dW_k, dim, 0.f);
  ok = ok && gemm_rm(hb, true, false, Gd, dim, M, b.dv, Gd, x, dim, dW_v, dim, 0.f);
  ok = ok && gemm_rm(hb, true, false, N, dim, M, b.dl, N, x, dim, dW_r, dim, 0.f);
  if (c.has_shared)
    ok = ok && gemm_rm(hb, true, false, d_h, dim, M, b.dq_sh, d_h, x, dim, dW_shared, dim, 0.f);
  ok = ok && gemm_rm(hb, false, false, M, dim, Nd, b.dq_exp, Nd, W_q, dim, dx, dim, 0.f);
  ok = ok && gemm_rm(hb, false, false, M, dim, Gd, b.dk, Gd, W_k, dim, dx, dim, 1.f);
  ok = ok && gemm_rm(hb, false, false, M, dim, Gd, b.dv, Gd, W_v, dim, dx, dim, 1.f);
  ok = ok && gemm_rm(hb, false, false, M, dim, N, b.dl, N, W_r, dim, dx, dim, 1.f);
  if (c.has_shared)
    ok = ok && gemm_rm(hb, false, false, M, dim, d_h, b.dq_sh, d_h, W_shared, dim, dx, dim, 1.f);
  return ok ? GQE_OK : GQE_ERR_CUDA;
}

bool outputs_ok(const void* W_shared, const float* dx, const float* dW_r, const float* dW_q,
                const float* dW_k, const float* dW_v, const float* dW_shared,
                const float* dW_o) {
  if (!dx || !dW_r || !dW_q || !dW_k || !dW_v || !dW_o) return false;
  if ((W_shared == nullptr) != (dW_shared == nullptr)) return false;
  const void* outs[] = {dx, dW_r, dW_q, dW_k, dW_v, dW_o};
  for (const void* p : outs)
    if (!aligned16(p)) return false;
  return !dW_shared || aligned16(dW_shared);
}

}  // namespace

void backward_release(gqe_ctx* h) {
  if (h->cublas) cublasDestroy(static_cast<cublasHandle_t>(h->cublas));
  if (h->bwd_base) cudaFree(h->bwd_base);
  h->cublas = nullptr;
  h->bwd_base = nullptr;
}

}  // namespace gqe

using namespace gqe;

extern "C" {

gqe_status gqe_enable_backward(gqe_handle h) {
  if (!h) return GQE_ERR_INVALID_ARG;
  if (!tc_backward_supported(h)) return GQE_ERR_UNSUPPORTED;
  if (h->bwd_base) return GQE_OK;
  const size_t bytes = bwd_layout(h->bwd, nullptr, h);
  void* base = nullptr;
  if (cudaMalloc(&base, bytes) != cudaSuccess) {
    cudaGetLastError();
    return GQE_ERR_CUDA;
  }
  if (cudaMemset(base, 0, bytes) != cudaSuccess) {
    cudaFree(base);
    return GQE_ERR_CUDA;
  }
  cublasHandle_t hb = nullptr;
  if (cublasCreate(&hb) != CUBLAS_STATUS_SUCCESS) {
    cudaFree(base);
    return GQE_ERR_CUDA;
  }
  bwd_layout(h->bwd, static_cast<char*>(base), h);
  if (cublasSetWorkspace(hb, h->bwd.cublas_ws, kCublasWorkspace) != CUBLAS_STATUS_SUCCESS) {
    cublasDestroy(hb);
    cudaFree(base);
    return GQE_ERR_CUDA;
  }
  h->bwd_base = base;
  h->bwd_bytes = bytes;
  h->cublas = hb;
  return GQE_OK;
}

gqe_status gqe_backward(gqe_handle h, const void* x, int B, int T, const void* W_r,
                        const void* W_q, const void* W_k, const void* W_v, const void* W_shared,
                        const void* W_o, int N, int G, int k, int d_h, int variant, int causal,
                        const void* dy, float aux_grad, float* dx, float* dW_r, float* dW_q,
                        float* dW_k, float* dW_v, float* dW_shared, float* dW_o, void* stream) {
  if (!h) return GQE_ERR_INVALID_ARG;
  // a part of the layer needs the sum of <dslot, slot> over the parts: the two phases
  if (h->g0 != 0 || h->g1 != h->G) return GQE_ERR_UNSUPPORTED;
  BwdCall c;
  gqe_status r = check_call(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h,
                            variant, causal, dy, c);
  if (r != GQE_OK) return r;
  if (!outputs_ok(W_shared, dx, dW_r, dW_q, dW_k, dW_v, dW_shared, dW_o))
    return GQE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  r = phase1(h, c, B, T, W_o, variant, causal, dy, h->bwd.slot_dot, st);
  if (r != GQE_OK) return r;
  return phase2(h, c, x, W_r, W_q, W_k, W_v, W_shared, variant, dy, aux_grad, h->bwd.slot_dot,
                dx, dW_r, dW_q, dW_k, dW_v, dW_shared, dW_o, st);
}

gqe_status gqe_backward_begin(gqe_handle h, const void* x, int B, int T, const void* W_r,
                              const void* W_q, const void* W_k, const void* W_v,
                              const void* W_shared, const void* W_o, int N, int G, int k,
                              int d_h, int variant, int causal, const void* dy, float* slot_dot,
                              void* stream) {
  if (!h) return GQE_ERR_INVALID_ARG;
  h->bwd_begun = 0;
  BwdCall c;
  const gqe_status r = check_call(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h,
                                  variant, causal, dy, c);
  if (r != GQE_OK) return r;
  if (!slot_dot || (reinterpret_cast<uintptr_t>(slot_dot) & 3u)) return GQE_ERR_INVALID_ARG;
  return phase1(h, c, B, T, W_o, variant, causal, dy, slot_dot, static_cast<cudaStream_t>(stream));
}

gqe_status gqe_backward_finish(gqe_handle h, const void* x, int B, int T, const void* W_r,
                               const void* W_q, const void* W_k, const void* W_v,
                               const void* W_shared, const void* W_o, int N, int G, int k,
                               int d_h, int variant, int causal, const void* dy, float aux_grad,
                               const float* slot_dot, float* dx, float* dW_r, float* dW_q,
                               float* dW_k, float* dW_v, float* dW_shared, float* dW_o,
                               void* stream) {
  if (!h) return GQE_ERR_INVALID_ARG;
  BwdCall c;
  const gqe_status r = check_call(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h,
                                  variant, causal, dy, c);
  if (r != GQE_OK) return r;
  if (!slot_dot || (reinterpret_cast<uintptr_t>(slot_dot) & 3u)) return GQE_ERR_INVALID_ARG;
  if (!outputs_ok(W_shared, dx, dW_r, dW_q, dW_k, dW_v, dW_shared, dW_o))
    return GQE_ERR_INVALID_ARG;
  return phase2(h, c, x, W_r, W_q, W_k, W_v, W_shared, variant, dy, aux_grad, slot_dot, dx,
                dW_r, dW_q, dW_k, dW_v, dW_shared, dW_o, static_cast<cudaStream_t>(stream));
}

int gqe_backward_launches(gqe_handle h) { return h ? h->last_bwd_launches : -1; }

}  // extern "C"
