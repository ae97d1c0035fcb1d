// Decode step with a KV cache: attention of one new token per sequence over its cached
// keys and values, and the append of the new token's K/V to the cache.
//
// GQE keeps the KV heads dense and unchanged ("GQE: Grouped Query Experts" README,
// Algorithm Overview), so generation caches K and V as GQA does, and the routing and the
// sparse query heads apply to each new token: for group g the new token has k routed query
// streams (s = g*k + r) and, in group 0, the always-on shared stream (it reads KV head 0;
// gist.science summary, Output Construction). A step for B sequences runs the forward's
// projection, routing and W_o kernels on the B new tokens; this file holds the parts that
// differ: the attention of stream s of sequence b over positions 0..L_b of its KV head,
// where positions < L_b come from the cache and position L_b is the new token, and the
// combine of the key chunks and the gqe slot.
//
// The work is HBM-bound (every cached K/V row is read once, shared by all query streams of
// its group), so it runs on CUDA cores. CTA (chunk c, group g, sequence b) streams its key
// range in tiles of 64 rows through a two-stage cp.async ring in shared memory (dense rows
// for d_h an odd multiple of 16, else rows padded by 16 bytes: see DecCfg). Each of the four
// warps takes 16 keys of every tile for all of the group's queries,
// so the work is spread evenly however few queries a group has (two at k = 1 in group 0,
// one elsewhere): a score per (key, half of the head dims) lane pair, the online softmax
// over the warp's keys with shuffles, P V with each lane owning pairs of head dimensions.
// After the last tile the four warps' (m, l, O) are merged in shared memory. With one chunk
// per sequence and group the CTA writes Z directly; otherwise it writes (m, l, O) to a
// partial slot. decode_finish_kernel, one CTA per sequence, then combines the chunks of
// every (group, query) and, for the gqe variant, forms the sequence's renormalised slot from
// the Z blocks it has just written (gist.science summary, Output Construction), in the order
// and precision of the forward's slot kernel.
#include <string.h>

#include "gqe_common.cuh"
#include "tc_ptx.cuh"

namespace gqe {
namespace {

using tc::smem_u32;

constexpr int THREADS = 128;
constexpr int WARPS = THREADS / 32;
constexpr int TKD = 64;      // keys per tile
constexpr int STAGES = 2;    // tiles in flight (two: the smaller footprint fits more CTAs per SM)
constexpr int MAXQ = kMaxTopK + 1;
constexpr int KPW = TKD / WARPS;  // keys of a tile per warp

struct DecParams {
  const __nv_bfloat16* Knew;  // [G, B, d_h] the new tokens' keys (workspace)
  const __nv_bfloat16* Vnew;
  const __nv_bfloat16* Q;     // [S, B, d_h]
  __nv_bfloat16* kc;          // [G, B, L_max, d_h] caches
  __nv_bfloat16* vc;
  const int32_t* lengths;     // [B]
  __nv_bfloat16* Z;           // [B, Do]
  const float* psel;          // [B, psel_stride]: stream s's p at column psel_off + s
  float* part;                // [B, G, nc, k+1, d_h + 2] partial (m, l, O) per chunk
  const float* wslot;         // [B, w_stride] slot weights: stream s's at column w_off + s
  int32_t* status;
  // G, S, Sr: this handle's KV heads, streams and routed streams (a group range counts
  // from its first group; the caches hold its heads only)
  int B, G, k, S, Sr, has_shared, Do, shared_col, weighted, L_max, nc, chunk;
  int psel_stride, psel_off;
  int slot, w_stride, w_off;  // slot: form the gqe slot at column Sr d_h
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
  // Dense rows where two lanes per key (key = lane / 2, half = lane % 2) read them without
  // bank conflicts (d_h an odd multiple of 16: the 16-byte reads of eight lanes fall on
  // distinct banks); else rows padded by 16 bytes with a lane per key and half.
  static constexpr bool DENSE = DH % 32 == 16;
  static constexpr int ROWB = DENSE ? DH * 2 : DH * 2 + 16;  // row bytes in the ring
  static constexpr int TILE = TKD * ROWB;         // one K or V tile
  static constexpr int CHUNKS = DH / 8;           // 16-byte pieces per row
  static constexpr int NP = (DH / 2 + 31) / 32;   // dim pairs per lane
  static constexpr int SMEM = STAGES * 2 * TILE + MAXQ * DH * 4;
  static_assert(STAGES * 2 * TILE >= WARPS * MAXQ * (DH + 2) * 4,
                "the ring holds the warps' states for the merge");
};

// stream index of query i of group g (routed streams first, then the shared one)
__device__ __forceinline__ int stream_of(const DecParams& P, int g, int i) {
  return i < P.k ? g * P.k + i : P.Sr;
}

// QMAX: the most queries a group can have at this launch (k, plus the shared head in group
// 0): 2, 4 or 9, a compile-time count so the per-query state stays in registers.
// With at most two queries per group and d_h <= 48 the state fits 64 registers, so eight
// CTAs share an SM (the work is bound by the bytes in flight: more CTAs, more of them).
template <int DH, int QMAX>
__global__ void __launch_bounds__(THREADS, (DH <= 48 && QMAX <= 2) ? 8 : 1)
decode_attn_kernel(const DecParams P) {
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
  // Every warp takes a quarter of each tile (keys 16 w .. 16 w + 15) for every query, with
  // its own online-softmax state; the four states are merged after the last tile. Score:
  // one key and one half of the head dims per lane (key = lane / 2, half = lane % 2 on dense
  // rows; key = lane % 16, half = lane / 16 on padded ones), halves summed by a shuffle.
  // P V: lanes own dimension pairs and loop over the warp's 16 keys.
  const int kq = C::DENSE ? lane >> 1 : lane & 15, half = C::DENSE ? lane & 1 : lane >> 4;
  constexpr int kHalfXor = C::DENSE ? 1 : 16;  // the lane holding the key's other half
  constexpr int kKeyLane = C::DENSE ? 2 : 1;   // lane stride between keys
  const int krow = warp * KPW + kq;
  float m[QMAX], l[QMAX];
  float2 o[QMAX][C::NP];
#pragma unroll
  for (int a = 0; a < QMAX; ++a) {
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
    const bool key_ok = k0 + t * TKD + krow < k1;
    // this lane's half of its key's row, as floats
    float kf[DH / 2];
    {
      const uint8_t* row = kt + krow * C::ROWB + half * DH;
#pragma unroll
      for (int ch = 0; ch < DH / 16; ++ch) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + ch * 16);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(p2[e]);
          kf[ch * 8 + 2 * e] = f.x;
          kf[ch * 8 + 2 * e + 1] = f.y;
        }
      }
    }
#pragma unroll
    for (int a = 0; a < QMAX; ++a) {
      if (a >= nq) break;  // uniform over the CTA
      const float* q = sQ + a * DH + half * (DH / 2);
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < DH / 2; ++d) acc = fmaf(q[d], kf[d], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, kHalfXor);
      const float sc = key_ok ? acc : -INFINITY;
      float mt = sc;
#pragma unroll
      for (int off = 8 * kKeyLane; off >= kKeyLane; off >>= 1)
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m[a], mt);
      // a warp whose keys are all masked so far keeps m = -inf, l = 0, O = 0
      const float m_ref = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2(m[a] - m_ref);  // 0 while m is -inf
      const float pk = ex2(sc - m_ref);       // 0 for a masked key
      float ps = pk;
#pragma unroll
      for (int off = 8 * kKeyLane; off >= kKeyLane; off >>= 1)
        ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[a] = l[a] * alpha + ps;
      m[a] = m_new;
#pragma unroll
      for (int p = 0; p < C::NP; ++p) {
        o[a][p].x *= alpha;
        o[a][p].y *= alpha;
      }
#pragma unroll
      for (int j = 0; j < KPW; ++j) {
        const float pj = __shfl_sync(0xffffffffu, pk, j * kKeyLane);
        const uint8_t* row = vt + (warp * KPW + j) * C::ROWB;
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
  __syncthreads();  // the ring is free: it holds the warps' states for the merge
  // merge the four warps' (m, l, O) of every query: state of (warp, query) at
  // sM[(warp * MAXQ + query) * (DH + 2)]: m, l, then O
  float* sM = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int a = 0; a < QMAX; ++a) {
    if (a >= nq) break;
    float* st = sM + (warp * MAXQ + a) * (DH + 2);
    if (lane == 0) {
      st[0] = m[a];
      st[1] = l[a];
    }
#pragma unroll
    for (int p = 0; p < C::NP; ++p) {
      const int d2 = lane + 32 * p;
      if (2 * d2 < DH) {
        st[2 + 2 * d2] = o[a][p].x;
        st[2 + 2 * d2 + 1] = o[a][p].y;
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < nq * DH; e += THREADS) {
    const int i = e / DH, d = e % DH;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) mx = fmaxf(mx, sM[(w * MAXQ + i) * (DH + 2)]);
    const float mref = mx == -INFINITY ? 0.f : mx;
    float lt = 0.f, ot = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float* st = sM + (w * MAXQ + i) * (DH + 2);
      const float f = ex2(st[0] - mref);  // 0 for a warp that saw no key
      lt += f * st[1];
      ot += f * st[2 + d];
    }
    const int s = stream_of(P, g, i);
    if (P.nc == 1) {
      float scale = 1.f / lt;
      int col;
      if (s < P.Sr) {
        col = s * DH;
        if (P.weighted) scale *= P.psel[(size_t)b * P.psel_stride + P.psel_off + s];
      } else {
        col = P.shared_col;
      }
      P.Z[(size_t)b * P.Do + col + d] = __float2bfloat16_rn(ot * scale);
    } else {
      float* slot = P.part + ((((size_t)b * P.G + g) * P.nc + c) * (P.k + 1) + i) * (DH + 2);
      if (d == 0) {
        slot[0] = ntiles ? mx : -INFINITY;
        slot[1] = lt;
      }
      slot[2 + d] = ot;
    }
  }
}

// One CTA per sequence: combines the key chunks' (m, l, O) of every (group, query) of the
// sequence and writes Z (when keys are split), then forms the gqe slot from Z's routed
// blocks (a fixed order: stream 0 first, fp32 fused multiply-adds of the bf16 values).
constexpr int FINISH_THREADS = 512;
__global__ void __launch_bounds__(FINISH_THREADS) decode_finish_kernel(const DecParams P,
                                                                       int DH) {
  const int b = blockIdx.x;
  pdl_wait();
  pdl_allow_next();
  const int L = P.lengths[b];
  if (L < 0 || L >= P.L_max) return;  // flagged by the attention kernel
  if (P.nc > 1) {
    // queries: k per group, then the shared one (group 0, query index k)
    const int nqs = P.G * P.k + P.has_shared;
    const size_t cstride = (size_t)(P.k + 1) * (DH + 2);
    for (int e = threadIdx.x; e < nqs * DH; e += FINISH_THREADS) {
      const int q = e / DH, d = e % DH;
      const int g = q < P.G * P.k ? q / P.k : 0;
      const int i = q < P.G * P.k ? q % P.k : P.k;
      const float* base = P.part + (((size_t)b * P.G + g) * P.nc * (P.k + 1) + i) * (DH + 2);
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
        if (P.weighted) scale *= P.psel[(size_t)b * P.psel_stride + P.psel_off + s];
      } else {
        col = P.shared_col;
      }
      P.Z[(size_t)b * P.Do + col + d] = __float2bfloat16_rn(o * scale);
    }
    __syncthreads();  // the sequence's routed blocks of Z are written
  }
  if (P.slot) {
    const float* w = P.wslot + (size_t)b * P.w_stride + P.w_off;
    __nv_bfloat16* z = P.Z + (size_t)b * P.Do;
    for (int d = threadIdx.x; d < DH; d += FINISH_THREADS) {
      float acc = 0.f;
      for (int s = 0; s < P.Sr; ++s) acc = fmaf(w[s], __bfloat162float(z[s * DH + d]), acc);
      z[(size_t)P.Sr * DH + d] = __float2bfloat16_rn(acc);
    }
  }
}

template <int DH, int QMAX>
int launch_attn(const DecParams& P, cudaStream_t st) {
  using C = DecCfg<DH>;
  if (!set_smem_limit_once<decode_attn_kernel<DH, QMAX>>(C::SMEM)) return -1;
  return launch_pdl(decode_attn_kernel<DH, QMAX>, dim3(P.nc, P.G, P.B), dim3(THREADS), C::SMEM,
                    st, P) == cudaSuccess
             ? 1
             : -1;
}

template <int DH>
int launch_dh(const DecParams& P, cudaStream_t st) {
  const int nq_max = P.k + (P.has_shared ? 1 : 0);
  const int r = nq_max <= 2 ? launch_attn<DH, 2>(P, st)
                : nq_max <= 4 ? launch_attn<DH, 4>(P, st)
                              : launch_attn<DH, MAXQ>(P, st);
  if (r < 0) return -1;
  if (P.nc == 1 && !P.slot) return 1;
  return launch_pdl(decode_finish_kernel, dim3(P.B), dim3(FINISH_THREADS), 0, st, P, DH) ==
                 cudaSuccess
             ? 2
             : -1;
}

}  // namespace

// Chunks per (sequence, group): enough CTAs for sixteen per SM, about three waves of the
// five resident at d_h = 48 (measured at 64 sequences of 8192 cached tokens: 232 us with one
// chunk per (sequence, group), 195 us with two, 182 us with three, 169 us with five, 167 us
// with seven), at least one tile each, and partial slots within the workspace's
// kDecodeSlots.
int decode_chunks(const gqe_ctx* h, int B, int L_max) {
  const int64_t bg = (int64_t)B * (h->g1 - h->g0);  // (sequence, KV head) pairs
  int64_t nc = (16 * (int64_t)h->num_sms + bg - 1) / bg;
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
  P.wslot = h->ws.w;
  P.status = h->ws.status;
  P.B = B;
  P.G = h->g1 - h->g0;
  P.k = h->k;
  P.S = S;
  P.Sr = P.G * h->k;
  P.psel_stride = h->G * h->k;
  P.psel_off = h->g0 * h->k;
  P.has_shared = has_shared;
  P.Do = Do;
  P.shared_col = (P.Sr + (variant == GQE_VARIANT_GQE ? 1 : 0)) * d_h;
  P.weighted = variant == GQE_VARIANT_WEIGHTED_CONCAT;
  P.slot = variant == GQE_VARIANT_GQE;
  P.w_stride = h->G * h->k;  // the slot weights are the whole layer's
  P.w_off = h->g0 * h->k;
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
