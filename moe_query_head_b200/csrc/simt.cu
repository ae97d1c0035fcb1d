// CUDA-core (FFMA) kernels: the fp32 path of every stage, and the reference-shaped
// general kernels used for shapes the tensor-core kernels do not take.
//
//   - projections (router logits, K, V, shared Q), the expert-bucketed routed Q
//     projection and W_o as tiled fp32 GEMMs;
//   - causal / non-causal softmax attention, one KV tile at a time with a running max;
//   - the output construction of the three variants ("GQE: Grouped Query Experts"
//     README, Ablations; gist.science summary, Output Construction).
#include "gqe_common.cuh"

namespace gqe {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__device__ __forceinline__ void store_out(const OutMap& o, int64_t m, int c, float v) {
  const int head = c / o.head_w, col = c % o.head_w;
  const int64_t idx = head * o.head_stride + m * o.row_stride + col * o.col_stride;
  if (o.f32)
    static_cast<float*>(o.base)[idx] = v;
  else
    static_cast<T*>(o.base)[idx] = from_f32<T>(v);
}

// C[m, n] = sum_k A[row(m), k] * B[n, k] for one BM x BN tile; 256 threads, 4x4 each.
// row(m) = m, or gather[m] >> 3 (the token of a bucket entry) when gather is non-null.
template <typename T>
__device__ __forceinline__ void gemm_tile(const T* __restrict__ A, int64_t lda,
                                          const int32_t* __restrict__ gather, int Mrows,
                                          const T* __restrict__ Bm, int64_t ldb, int N, int K,
                                          int m0, int n0, float acc[4][4]) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  // each thread loads 4 elements of A and 4 of B per K tile
  const int lr = tid / 4;        // 0..63 row within tile
  const int lk = (tid % 4) * 4;  // 0,4,8,12
  int64_t arow = -1;
  if (m0 + lr < Mrows) arow = gather ? (int64_t)(gather[m0 + lr] >> 3) : (int64_t)(m0 + lr);
  const bool brow_ok = n0 + lr < N;
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int kk = k0 + lk + u;
      As[lk + u][lr] = (arow >= 0 && kk < K) ? to_f32(A[arow * lda + kk]) : 0.f;
      Bs[lk + u][lr] = (brow_ok && kk < K) ? to_f32(Bm[(int64_t)(n0 + lr) * ldb + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

struct DenseProblem {
  const void* B;
  int N;
  OutMap out;
};
struct DenseArgs {
  DenseProblem p[4];
  int count;
};

// x [M, K] times up to four weight matrices (router, K, V, shared query): grid.z picks one.
template <typename T>
__global__ void __launch_bounds__(256) dense_proj_kernel(const T* __restrict__ x, int M, int K,
                                                         DenseArgs args) {
  const DenseProblem& P = args.p[blockIdx.z];
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  if (n0 >= P.N) return;
  float acc[4][4];
  gemm_tile<T>(x, K, nullptr, M, static_cast<const T*>(P.B), K, P.N, K, m0, n0, acc);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < M && n < P.N) store_out<T>(P.out, m, n, acc[i][j]);
    }
}

// Routed Q projection: grid (row tiles, column tiles, expert). Expert e's rows are its
// bucket entries; row i projects token t = entry >> 3 with W_q[e] and lands in query
// stream g*k + (entry & 7) at token position t.
template <typename T>
__global__ void __launch_bounds__(256)
qproj_kernel(const T* __restrict__ x, int M, int K, const T* __restrict__ Wq, int d_h, int E,
             int k, const int32_t* __restrict__ offsets, const int32_t* __restrict__ counts,
             const int32_t* __restrict__ bucket,
             T* __restrict__ Q) {
  const int e = blockIdx.z;
  const int beg = offsets[e], cnt = counts[e];
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  if (m0 >= cnt) return;
  float acc[4][4];
  gemm_tile<T>(x, K, bucket + beg, cnt, Wq + (int64_t)e * d_h * K, K, d_h, K, m0, n0, acc);
  const int g = e / E;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= cnt) continue;
    const int ent = bucket[beg + m];
    const int64_t t = min(ent >> 3, M - 1);
    const int s = g * k + min(ent & 7, k - 1);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < d_h) Q[((int64_t)s * M + t) * d_h + n] = from_f32<T>(acc[i][j]);
    }
  }
}

// y = Z W_o^T: Z [M, Do], W_o [dim, Do], y [M, dim].
template <typename T>
__global__ void __launch_bounds__(256) oproj_kernel(const T* __restrict__ Z, int M, int Do,
                                                    const T* __restrict__ Wo, int dim,
                                                    T* __restrict__ y) {
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
  float acc[4][4];
  gemm_tile<T>(Z, Do, nullptr, M, Wo, Do, dim, Do, m0, n0, acc);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < M && n < dim) y[(int64_t)m * dim + n] = from_f32<T>(acc[i][j]);
    }
}

// Softmax attention, CUDA cores. Block = 32 query rows x 4 threads (each thread owns DH/4
// of the head dimensions); grid (row tiles, stream, batch). Stream s < G*k reads KV head
// s / k; the shared stream reads KV head 0. The normalised output row goes straight into
// its column block of Z; for weighted_concat the routed blocks are scaled by the router
// probability p of their expert here.
constexpr int ATT_ROWS = 32, ATT_KEYS = 32;

template <typename T, int DH>
__global__ void __launch_bounds__(128)
attention_kernel(const T* __restrict__ Q, const T* __restrict__ Kc, const T* __restrict__ Vc,
                 T* __restrict__ Z, const float* __restrict__ psel, int M, int Tlen, int G,
                 int k, int Do, int shared_col, int weighted, int causal, float scale_log2) {
  constexpr int PD = DH / 4;
  __shared__ float Ks[ATT_KEYS][DH + 1];
  __shared__ float Vs[ATT_KEYS][DH + 1];
  const int s = blockIdx.y, b = blockIdx.z;
  const int Sr = G * k;
  const int kvh = s < Sr ? s / k : 0;
  const int row = threadIdx.x / 4, sub = threadIdx.x % 4;
  const int t = blockIdx.x * ATT_ROWS + row;  // position within the sequence
  const bool valid = t < Tlen;
  const int64_t tok = (int64_t)b * Tlen + (valid ? t : Tlen - 1);
  float q[PD], o[PD];
#pragma unroll
  for (int c = 0; c < PD; ++c) {
    q[c] = to_f32(Q[((int64_t)s * M + tok) * DH + sub * PD + c]) * scale_log2;
    o[c] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;
  const int row0 = blockIdx.x * ATT_ROWS;
  const int kv_end = causal ? min(Tlen, row0 + ATT_ROWS) : Tlen;
  const T* Kh = Kc + (int64_t)kvh * M * DH + (int64_t)b * Tlen * DH;
  const T* Vh = Vc + (int64_t)kvh * M * DH + (int64_t)b * Tlen * DH;
  for (int u0 = 0; u0 < kv_end; u0 += ATT_KEYS) {
    __syncthreads();
    for (int i = threadIdx.x; i < ATT_KEYS * DH; i += 128) {
      const int kr = i / DH, kc = i % DH;
      Ks[kr][kc] = (u0 + kr < Tlen) ? to_f32(Kh[(int64_t)(u0 + kr) * DH + kc]) : 0.f;
      Vs[kr][kc] = (u0 + kr < Tlen) ? to_f32(Vh[(int64_t)(u0 + kr) * DH + kc]) : 0.f;
    }
    __syncthreads();
    float sc[ATT_KEYS];
    float mt = m_run;
#pragma unroll
    for (int j = 0; j < ATT_KEYS; ++j) {
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < PD; ++c) part = fmaf(q[c], Ks[j][sub * PD + c], part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      const int u = u0 + j;
      const bool ok = u < Tlen && (!causal || u <= t);
      sc[j] = ok ? part : -INFINITY;
      mt = fmaxf(mt, sc[j]);
    }
    const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - mt);
    l_run *= alpha;
#pragma unroll
    for (int c = 0; c < PD; ++c) o[c] *= alpha;
#pragma unroll
    for (int j = 0; j < ATT_KEYS; ++j) {
      const float p = (sc[j] == -INFINITY) ? 0.f : exp2f(sc[j] - mt);
      l_run += p;
#pragma unroll
      for (int c = 0; c < PD; ++c) o[c] = fmaf(p, Vs[j][sub * PD + c], o[c]);
    }
    m_run = mt;
  }
  if (!valid) return;
  float scale = 1.f / l_run;
  int col;
  if (s < Sr) {
    col = s * DH;
    if (weighted) scale *= psel[tok * Sr + s];
  } else {
    col = shared_col;
  }
#pragma unroll
  for (int c = 0; c < PD; ++c) Z[tok * Do + col + sub * PD + c] = from_f32<T>(o[c] * scale);
}

// Variant gqe: the renormalised slot rho_t = sum_s w[t, s] * O[t, s] over the routed
// streams, read back from Z's routed blocks and written to Z's slot block. The slot weights
// are the whole layer's [M, w_stride]; a handle restricted to a group range reads its
// streams' columns from w_off on, so the ranges' slots sum to the layer's.
// One thread per 16 bytes of the slot (8 bf16 or 4 fp32 values): 16-byte loads of every
// routed block, fp32 accumulation, one 16-byte store.
template <typename T>
__global__ void slot_kernel(T* __restrict__ Z, const float* __restrict__ w, int M, int Sr,
                            int d_h, int Do, int w_stride, int w_off) {
  constexpr int VEC = 16 / sizeof(T);
  pdl_wait();  // Z and the slot weights are complete from here on
  pdl_allow_next();
  const int per_tok = d_h / VEC;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)M * per_tok) return;
  const int64_t t = i / per_tok;
  const int c0 = (int)(i % per_tok) * VEC;
  float acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
  const T* zt = Z + t * Do + c0;
  // eight streams per batch: all their loads are issued before the first use
  for (int s0 = 0; s0 < Sr; s0 += 8) {
    uint4 raw[8];
    float ws[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool in = s0 + u < Sr;
      ws[u] = in ? w[t * w_stride + w_off + s0 + u] : 0.f;
      raw[u] = in ? *reinterpret_cast<const uint4*>(zt + (int64_t)(s0 + u) * d_h)
                  : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const T* val = reinterpret_cast<const T*>(&raw[u]);
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = fmaf(ws[u], to_f32(val[v]), acc[v]);
    }
  }
  uint4 out;
  T* o = reinterpret_cast<T*>(&out);
#pragma unroll
  for (int v = 0; v < VEC; ++v) o[v] = from_f32<T>(acc[v]);
  *reinterpret_cast<uint4*>(Z + t * Do + (int64_t)Sr * d_h + c0) = out;
}

template <typename T>
int dense_proj_t(gqe_ctx* h, const void* x, int M, const void* W_r, const void* W_k,
                 const void* W_v, const void* W_shared, cudaStream_t st) {
  const int d_h = h->d_h, G = h->G;
  const int S = G * h->k + (W_shared ? 1 : 0);
  DenseArgs a{};
  int n = 0;
  a.p[n++] = DenseProblem{W_r, h->N, OutMap{h->ws.logits, 0, h->N, 1, 1 << 30, 1}};
  a.p[n++] = DenseProblem{W_k, G * d_h, OutMap{h->ws.K, (int64_t)M * d_h, d_h, 1, d_h, 0}};
  a.p[n++] = DenseProblem{W_v, G * d_h, OutMap{h->ws.V, (int64_t)M * d_h, d_h, 1, d_h, 0}};
  if (W_shared) {
    void* qs = static_cast<char*>(h->ws.Q) + (int64_t)(S - 1) * M * d_h * h->esz;
    a.p[n++] = DenseProblem{W_shared, d_h, OutMap{qs, 0, d_h, 1, d_h, 0}};
  }
  a.count = n;
  int maxN = 0;
  for (int i = 0; i < n; ++i) maxN = a.p[i].N > maxN ? a.p[i].N : maxN;
  dim3 grid((M + BM - 1) / BM, (maxN + BN - 1) / BN, n);
  dense_proj_kernel<T><<<grid, 256, 0, st>>>(static_cast<const T*>(x), M, h->dim, a);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

template <typename T, int DH>
void attention_launch(gqe_ctx* h, int B, int T_, int S, int shared_col, int weighted,
                      int causal, int Do, cudaStream_t st) {
  const int M = B * T_;
  dim3 grid((T_ + ATT_ROWS - 1) / ATT_ROWS, S, B);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  attention_kernel<T, DH><<<grid, 128, 0, st>>>(
      static_cast<const T*>(h->ws.Q), static_cast<const T*>(h->ws.K),
      static_cast<const T*>(h->ws.V), static_cast<T*>(h->ws.Z), h->ws.psel, M, T_, h->G,
      h->k, Do, shared_col, weighted, causal, scale_log2);
}

template <typename T>
int attention_t(gqe_ctx* h, int B, int T_, int S, int has_shared, int variant, int causal,
                int Do, cudaStream_t st) {
  const int Sr = h->G * h->k;
  const int shared_col = (Sr + (variant == GQE_VARIANT_GQE ? 1 : 0)) * h->d_h;
  const int weighted = variant == GQE_VARIANT_WEIGHTED_CONCAT;
  (void)has_shared;
  switch (h->d_h) {
    case 16: attention_launch<T, 16>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 32: attention_launch<T, 32>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 48: attention_launch<T, 48>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 64: attention_launch<T, 64>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 80: attention_launch<T, 80>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 96: attention_launch<T, 96>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 112: attention_launch<T, 112>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    case 128: attention_launch<T, 128>(h, B, T_, S, shared_col, weighted, causal, Do, st); break;
    default: return -1;
  }
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int launch_simt_dense_proj(gqe_ctx* h, const void* x, int M, const void* W_r, const void* W_k,
                           const void* W_v, const void* W_shared, cudaStream_t st) {
  if (h->dtype == GQE_F32) return dense_proj_t<float>(h, x, M, W_r, W_k, W_v, W_shared, st);
  return dense_proj_t<__nv_bfloat16>(h, x, M, W_r, W_k, W_v, W_shared, st);
}

int launch_simt_qproj(gqe_ctx* h, const void* x, int M, const void* W_q, cudaStream_t st) {
  dim3 grid((M + BM - 1) / BM, (h->d_h + BN - 1) / BN, h->N);
  if (h->dtype == GQE_F32)
    qproj_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float*>(x), M, h->dim, static_cast<const float*>(W_q), h->d_h, h->E,
        h->k, h->ws.offsets, h->ws.counts, h->ws.bucket, static_cast<float*>(h->ws.Q));
  else
    qproj_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), M, h->dim,
        static_cast<const __nv_bfloat16*>(W_q), h->d_h, h->E, h->k, h->ws.offsets,
        h->ws.counts, h->ws.bucket, static_cast<__nv_bfloat16*>(h->ws.Q));
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_simt_attention(gqe_ctx* h, int B, int T, int S, int has_shared, int variant,
                          int causal, int Do, cudaStream_t st) {
  if (h->dtype == GQE_F32) return attention_t<float>(h, B, T, S, has_shared, variant, causal, Do, st);
  return attention_t<__nv_bfloat16>(h, B, T, S, has_shared, variant, causal, Do, st);
}

int launch_combine(gqe_ctx* h, int M, int variant, int Do, cudaStream_t st) {
  if (variant != GQE_VARIANT_GQE) return 0;  // weighted_concat is applied in attention
  // the handle's routed streams; the slot weights are the whole layer's [M, G k]
  const int Sr = (h->g1 - h->g0) * h->k;
  const int w_stride = h->G * h->k, w_off = h->g0 * h->k;
  const int64_t n = (int64_t)M * h->d_h / (16 / h->esz);
  const int blocks = (int)((n + 255) / 256);
  if (h->dtype == GQE_F32)
    slot_kernel<float><<<blocks, 256, 0, st>>>(static_cast<float*>(h->ws.Z), h->ws.w, M, Sr,
                                               h->d_h, Do, w_stride, w_off);
  else
    return launch_pdl(slot_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                      static_cast<__nv_bfloat16*>(h->ws.Z), static_cast<const float*>(h->ws.w),
                      M, Sr, h->d_h, Do, w_stride, w_off) == cudaSuccess
               ? 1
               : -1;
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_simt_oproj(gqe_ctx* h, int M, int Do, const void* W_o, void* out, cudaStream_t st) {
  dim3 grid((M + BM - 1) / BM, (h->dim + BN - 1) / BN);
  if (h->dtype == GQE_F32)
    oproj_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(h->ws.Z), M, Do,
                                              static_cast<const float*>(W_o), h->dim,
                                              static_cast<float*>(out));
  else
    oproj_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(h->ws.Z), M, Do,
        static_cast<const __nv_bfloat16*>(W_o), h->dim, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace gqe
