// Decode step with a KV cache: attention of one new token per sequence over its cached
// keys and values, and the append of the new token's K/V to the cache.
//
// GQE keeps the KV heads dense and unchanged ("GQE: Grouped Query Experts" README,
// Algorithm Overview), so generation caches K and V as GQA does, and the routing and the
// sparse query heads apply to each new token: for group g the new token has k routed query
// streams (s = g*k + r) and, in group 0, the always-on shared stream (it reads KV head 0;
// gist.science summary, Output Construction). A step for B sequences runs the forward's
// projection, routing, combine and W_o kernels on the B new tokens; this file holds the part
// that differs: the attention of stream s of sequence b over positions 0..L_b of its KV head,
// where positions < L_b come from the cache and position L_b is the new token.
//
// The work is HBM-bound (every cached K/V row is read once, shared by all query streams of
// its group), so it runs on CUDA cores. CTA (chunk c, group g, sequence b) streams its key
// range in tiles of 64 rows through a cp.async ring in shared memory (rows padded by 16
// bytes so the per-key 16-byte reads are conflict-free); warp w owns queries w, w+4, w+8 of
// the group: scores with one key per lane (two per tile), the online softmax with warp
// shuffles, P V with each lane owning pairs of head dimensions. With one chunk per sequence
// and group the CTA writes Z directly; otherwise it writes (m, l, O) to a partial slot and
// decode_merge_kernel combines the chunks.
#include <string.h>

#include "gqe_common.cuh"
#include "tc_ptx.cuh"

namespace gqe {
namespace {

using tc::smem_u32;

constexpr int THREADS = 128;
constexpr int WARPS = THREADS / 32;
constexpr int TKD = 64;      // keys per tile
constexpr int STAGES = 3;    // tiles in flight
constexpr int MAXQ = kMaxTopK + 1;

struct DecParams {
  const __nv_bfloat16* Knew;  // [G, B, d_h] the new tokens' keys (workspace)
  const __nv_bfloat16* Vnew;
  const __nv_bfloat16* Q;     // [S, B, d_h]
  __nv_bfloat16* kc;          // [G, B, L_max, d_h] caches
  __nv_bfloat16* vc;
  const int32_t* lengths;     // [B]
  __nv_bfloat16* Z;           // [B, Do]
  const float* psel;          // [B, G*k]
  float* part;                // [B, G, nc, k+1, d_h + 2] partial (m, l, O) per chunk
  int32_t* status;
  int B, G, k, S, Sr, has_shared, Do, shared_col, weighted, L_max, nc, chunk;
  float scale_log2;
};

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int DH>
struct DecCfg {
  static constexpr int ROWB = DH * 2 + 16;        // padded row bytes
  static constexpr int TILE = TKD * ROWB;         // one K or V tile
  static constexpr int CHUNKS = DH / 8;           // 16-byte pieces per row
  static constexpr int NP = (DH / 2 + 31) / 32;   // dim pairs per lane
  static constexpr int SMEM = STAGES * 2 * TILE + MAXQ * DH * 4;
};

// stream index of query i of group g (routed streams first, then the shared one)
__device__ __forceinline__ int stream_of(const DecParams& P, int g, int i) {
  return i < P.k ? g * P.k + i : P.Sr;
}

// QPW: queries per warp (1 for up to four queries per group, i.e. k <= 3 with the shared
// head; up to 3 for k = 8), a compile-time count so the per-query state stays in registers.
template <int DH, int QPW>
__global__ void __launch_bounds__(THREADS) decode_attn_kernel(const DecParams P) {
  using C = DecCfg<DH>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = smem + STAGES * C::TILE;
  float* sQ = reinterpret_cast<float*>(smem + 2 * STAGES * C::TILE);  // [MAXQ][DH]
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  pdl_wait();  // the new tokens' K, V and Q are complete from here on
  pdl_allow_next();
  const int L = P.lengths[b];
  if (L < 0 || L >= P.L_max) {
    // the new position lies outside the cache: nothing is read or written for this sequence
    if (tid == 0 && c == 0 && g == 0) atomicExch(P.status, kStatusBadInput);
    return;
  }
  const int nq = P.k + ((g == 0 && P.has_shared) ? 1 : 0);
  const int n_keys = L + 1;
  const int k0 = c * P.chunk;
  const int k1 = min(n_keys, k0 + P.chunk);
  const size_t head_off = ((size_t)g * P.B + b) * P.L_max * DH;  // cache rows of (g, b)
  const size_t new_off = ((size_t)g * P.B + b) * DH;
  // the chunk holding the new position appends the new K/V to the caches
  if (k0 <= L && L < k0 + P.chunk) {
    for (int i = tid; i < C::CHUNKS; i += THREADS) {
      reinterpret_cast<uint4*>(P.kc + head_off + (size_t)L * DH)[i] =
          reinterpret_cast<const uint4*>(P.Knew + new_off)[i];
      reinterpret_cast<uint4*>(P.vc + head_off + (size_t)L * DH)[i] =
          reinterpret_cast<const uint4*>(P.Vnew + new_off)[i];
    }
  }
  // queries of this group, prescaled to log2 units
  for (int e = tid; e < nq * DH; e += THREADS) {
    const int i = e / DH, d = e % DH;
    const int s = stream_of(P, g, i);
    sQ[e] = __bfloat162float(P.Q[((size_t)s * P.B + b) * DH + d]) * P.scale_log2;
  }
  const int ntiles = k1 > k0 ? (k1 - k0 + TKD - 1) / TKD : 0;
  // K / V tile t: rows k0 + t*TKD ...; position L is the new token (from the workspace),
  // rows past the range are zero-filled and masked
  auto load_tile = [&](int t, int st) {
    const int base = k0 + t * TKD;
    for (int e = tid; e < TKD * C::CHUNKS; e += THREADS) {
      const int r = e / C::CHUNKS, ch = e % C::CHUNKS;
      const int u = base + r;
      const uint32_t dk = smem_u32(sK + st * C::TILE + r * C::ROWB + ch * 16);
      const uint32_t dv = smem_u32(sV + st * C::TILE + r * C::ROWB + ch * 16);
      const __nv_bfloat16* ks;
      const __nv_bfloat16* vs;
      uint32_t bytes = 16;
      if (u < L) {
        ks = P.kc + head_off + (size_t)u * DH + ch * 8;
        vs = P.vc + head_off + (size_t)u * DH + ch * 8;
      } else {
        ks = P.Knew + new_off + ch * 8;  // u == L, or a masked row (zero-filled)
        vs = P.Vnew + new_off + ch * 8;
        if (u != L || u >= k1) bytes = 0;
      }
      cp16(dk, ks, bytes);
      cp16(dv, vs, bytes);
    }
  };
  for (int t = 0; t < STAGES - 1; ++t) {
    if (t < ntiles) load_tile(t, t);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  float m[QPW], l[QPW];
  float2 o[QPW][C::NP];
#pragma unroll
  for (int a = 0; a < QPW; ++a) {
    m[a] = -INFINITY;
    l[a] = 0.f;
#pragma unroll
    for (int p = 0; p < C::NP; ++p) o[a][p] = make_float2(0.f, 0.f);
  }
  __syncthreads();  // sQ written
  for (int t = 0; t < ntiles; ++t) {
    if (t + STAGES - 1 < ntiles) load_tile(t + STAGES - 1, (t + STAGES - 1) % STAGES);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group %0;" ::"n"(STAGES - 1) : "memory");
    __syncthreads();  // tile t is in shared memory for every thread
    const int st = t % STAGES;
    const uint8_t* kt = sK + st * C::TILE;
    const uint8_t* vt = sV + st * C::TILE;
    const int base = k0 + t * TKD;
#pragma unroll
    for (int a = 0; a < QPW; ++a) {
      const int i = warp + a * WARPS;
      if (i >= nq) break;  // warp-uniform
      const float* q = sQ + i * DH;
      // scores of keys lane and lane + 32
      float sc[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = lane + 32 * h;
        const uint8_t* row = kt + r * C::ROWB;
        float acc = 0.f;
#pragma unroll
        for (int ch = 0; ch < C::CHUNKS; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(row + ch * 16);
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            acc = fmaf(q[ch * 8 + 2 * e], f.x, acc);
            acc = fmaf(q[ch * 8 + 2 * e + 1], f.y, acc);
          }
        }
        sc[h] = base + r < k1 ? acc : -INFINITY;
      }
      float mt = fmaxf(sc[0], sc[1]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m[a], mt);  // finite: every tile holds at least one key
      const float alpha = ex2(m[a] - m_new);  // 0 when m was -inf
      const float p0 = ex2(sc[0] - m_new), p1 = ex2(sc[1] - m_new);
      float ps = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[a] = l[a] * alpha + ps;
      m[a] = m_new;
#pragma unroll
      for (int p = 0; p < C::NP; ++p) {
        o[a][p].x *= alpha;
        o[a][p].y *= alpha;
      }
      // O += P V: lane owns dimension pairs lane, lane + 32, ...
#pragma unroll 4
      for (int j = 0; j < TKD; ++j) {
        const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
        const uint8_t* row = vt + j * C::ROWB;
#pragma unroll
        for (int p = 0; p < C::NP; ++p) {
          const int d2 = lane + 32 * p;
          if (2 * d2 < DH) {
            const float2 f =
                __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row + 4 * d2));
            o[a][p].x = fmaf(pj, f.x, o[a][p].x);
            o[a][p].y = fmaf(pj, f.y, o[a][p].y);
          }
        }
      }
    }
    __syncthreads();  // every warp is done with stage st before it is refilled
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // results
#pragma unroll
  for (int a = 0; a < QPW; ++a) {
    const int i = warp + a * WARPS;
    if (i >= nq) break;
    const int s = stream_of(P, g, i);
    if (P.nc == 1) {
      float scale = 1.f / l[a];
      int col;
      if (s < P.Sr) {
        col = s * DH;
        if (P.weighted) scale *= P.psel[(size_t)b * P.Sr + s];
      } else {
        col = P.shared_col;
      }
      __nv_bfloat16* dst = P.Z + (size_t)b * P.Do + col;
#pragma unroll
      for (int p = 0; p < C::NP; ++p) {
        const int d2 = lane + 32 * p;
        if (2 * d2 < DH)
          *reinterpret_cast<__nv_bfloat162*>(dst + 2 * d2) =
              __floats2bfloat162_rn(o[a][p].x * scale, o[a][p].y * scale);
      }
    } else {
      float* slot = P.part + ((((size_t)b * P.G + g) * P.nc + c) * (P.k + 1) + i) * (DH + 2);
      if (lane == 0) {
        slot[0] = ntiles ? m[a] : -INFINITY;
        slot[1] = l[a];
      }
#pragma unroll
      for (int p = 0; p < C::NP; ++p) {
        const int d2 = lane + 32 * p;
        if (2 * d2 < DH) {
          slot[2 + 2 * d2] = o[a][p].x;
          slot[2 + 2 * d2 + 1] = o[a][p].y;
        }
      }
    }
  }
}

// Combines the chunks' (m, l, O) of every (sequence, group, query) and writes Z.
__global__ void __launch_bounds__(THREADS) decode_merge_kernel(const DecParams P, int DH) {
  const int g = blockIdx.x, b = blockIdx.y;
  pdl_wait();
  pdl_allow_next();
  const int L = P.lengths[b];
  if (L < 0 || L >= P.L_max) return;  // flagged by the attention kernel
  const int nq = P.k + ((g == 0 && P.has_shared) ? 1 : 0);
  for (int e = threadIdx.x; e < nq * DH; e += THREADS) {
    const int i = e / DH, d = e % DH;
    const float* base = P.part + (((size_t)b * P.G + g) * P.nc * (P.k + 1) + i) * (DH + 2);
    const size_t cstride = (size_t)(P.k + 1) * (DH + 2);
    float mx = -INFINITY;
    for (int c = 0; c < P.nc; ++c) mx = fmaxf(mx, base[c * cstride]);
    float l = 0.f, o = 0.f;
    for (int c = 0; c < P.nc; ++c) {
      const float* sl = base + c * cstride;
      if (sl[0] == -INFINITY) continue;  // a chunk past the sequence's last position
      const float w = ex2(sl[0] - mx);
      l += w * sl[1];
      o += w * sl[2 + d];
    }
    const int s = stream_of(P, g, i);
    float scale = 1.f / l;
    int col;
    if (s < P.Sr) {
      col = s * DH;
      if (P.weighted) scale *= P.psel[(size_t)b * P.Sr + s];
    } else {
      col = P.shared_col;
    }
    P.Z[(size_t)b * P.Do + col + d] = __float2bfloat16_rn(o * scale);
  }
}

template <int DH, int QPW>
int launch_attn(const DecParams& P, cudaStream_t st) {
  using C = DecCfg<DH>;
  if (!set_smem_limit_once<decode_attn_kernel<DH, QPW>>(C::SMEM)) return -1;
  return launch_pdl(decode_attn_kernel<DH, QPW>, dim3(P.nc, P.G, P.B), dim3(THREADS), C::SMEM,
                    st, P) == cudaSuccess
             ? 1
             : -1;
}

template <int DH>
int launch_dh(const DecParams& P, cudaStream_t st) {
  const int nq_max = P.k + (P.has_shared ? 1 : 0);
  const int qpw = (nq_max + WARPS - 1) / WARPS;
  const int r = qpw <= 1 ? launch_attn<DH, 1>(P, st)
                : qpw == 2 ? launch_attn<DH, 2>(P, st)
                           : launch_attn<DH, 3>(P, st);
  if (r < 0) return -1;
  if (P.nc == 1) return 1;
  return launch_pdl(decode_merge_kernel, dim3(P.G, P.B), dim3(THREADS), 0, st, P, DH) ==
                 cudaSuccess
             ? 2
             : -1;
}

}  // namespace

// Chunks per (sequence, group): enough CTAs for four per SM (measured: 7 % faster than two
// per SM at 64 sequences of 8192 cached tokens, where it splits each sequence in two), at
// least one tile each, and partial slots within the workspace's kDecodeSlots.
int decode_chunks(const gqe_ctx* h, int B, int L_max) {
  const int64_t bg = (int64_t)B * h->G;
  int64_t nc = (4 * (int64_t)h->num_sms + bg - 1) / bg;
  const int64_t max_by_len = ((int64_t)L_max + TKD - 1) / TKD;
  if (nc > max_by_len) nc = max_by_len;
  while (nc > 1 && bg * nc > kDecodeSlots) --nc;
  return nc < 1 ? 1 : (int)nc;
}

int launch_tc_decode_attention(gqe_ctx* h, int B, int S, int has_shared, int variant, int Do,
                               void* k_cache, void* v_cache, int L_max, const int32_t* lengths,
                               cudaStream_t st) {
  DecParams P;
  memset(&P, 0, sizeof(P));
  const int d_h = h->d_h;
  P.Knew = static_cast<const __nv_bfloat16*>(h->ws.K);
  P.Vnew = static_cast<const __nv_bfloat16*>(h->ws.V);
  P.Q = static_cast<const __nv_bfloat16*>(h->ws.Q);
  P.kc = static_cast<__nv_bfloat16*>(k_cache);
  P.vc = static_cast<__nv_bfloat16*>(v_cache);
  P.lengths = lengths;
  P.Z = static_cast<__nv_bfloat16*>(h->ws.Z);
  P.psel = h->ws.psel;
  P.part = h->ws.dec_part;
  P.status = h->ws.status;
  P.B = B;
  P.G = h->G;
  P.k = h->k;
  P.S = S;
  P.Sr = h->G * h->k;
  P.has_shared = has_shared;
  P.Do = Do;
  P.shared_col = (P.Sr + (variant == GQE_VARIANT_GQE ? 1 : 0)) * d_h;
  P.weighted = variant == GQE_VARIANT_WEIGHTED_CONCAT;
  P.L_max = L_max;
  P.nc = decode_chunks(h, B, L_max);
  // keys per chunk: a multiple of the tile, covering positions 0 .. L_max - 1
  const int64_t per = ((int64_t)L_max + P.nc - 1) / P.nc;
  P.chunk = (int)((per + TKD - 1) / TKD * TKD);
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)d_h);
  switch (d_h) {
    case 16: return launch_dh<16>(P, st);
    case 32: return launch_dh<32>(P, st);
    case 48: return launch_dh<48>(P, st);
    case 64: return launch_dh<64>(P, st);
    case 80: return launch_dh<80>(P, st);
    case 96: return launch_dh<96>(P, st);
    case 112: return launch_dh<112>(P, st);
    case 128: return launch_dh<128>(P, st);
    default: return -1;
  }
}

}  // namespace gqe
