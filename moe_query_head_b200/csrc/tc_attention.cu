// Tensor-core (tcgen05) causal / non-causal softmax attention of the GQE query streams.
//
// Stream s < G*k holds the routed queries of group s / k and reads that group's dense KV
// head; the last stream is the always-on shared head and reads KV head 0 ("GQE: Grouped
// Query Experts" README, Algorithm Overview; gist.science summary, Output Construction).
// Every stream has one query per token, so the work is a grouped-query attention with
// S = G*k + 1 query heads over G KV heads; the savings of GQE come from S < N + 1.
//
// Work item = (sequence b, stream s, 128-query tile); a persistent CTA per SM takes items
// heaviest first (causal tiles near the end of the sequence have the most keys).
//   warp 0     TMA: the Q tile once per item, then K and V tiles into a ring of stages;
//   warp 1     TMEM owner; one lane issues S = Q K^T (A and B from shared memory) into
//              one of two TMEM S buffers, then O += P V with P read from TMEM (the TS form)
//              and V as an MN-major shared-memory operand;
//   warps 2-5  softmax: one query row per thread, 128 scores per KV tile in registers,
//              exp2 with the running row maximum, P written back over S as bf16 pairs.
//              O is rescaled in TMEM only when a row maximum grows by more than 2^8
//              (rare after the first tiles), so the common path never waits on P V. At
//              the end of an item the same warps normalise O by the row sum, apply the
//              weighted_concat scale if any, and store the row into its block of Z.
#include <cudaTypedefs.h>

#include "gqe_common.cuh"
#include "tc_ptx.cuh"

namespace gqe {

bool tmap_bf16_2d_ext(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                      uint64_t ld, uint32_t box_cols, uint32_t box_rows,
                      CUtensorMapSwizzle sw);

namespace {

using namespace tc;

constexpr int THREADS = 192;
constexpr int TQ = 128;   // queries per tile (MMA M, TMEM lanes)
constexpr int TK = 128;   // keys per tile (S MMA N)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int DH>
struct Cfg {
  static constexpr int CW = (DH % 64 == 0) ? 64 : (DH % 32 == 0) ? 32 : 16;  // chunk width
  static constexpr int NC = DH / CW;                                         // chunks
  static constexpr uint32_t LAYOUT =
      CW == 64 ? kSwizzle128B : (CW == 32 ? kSwizzle64B : kSwizzle32B);
  static constexpr int ROW_BYTES = CW * 2;          // bytes per row inside a chunk
  static constexpr int CHUNK_BYTES = 128 * ROW_BYTES;
  static constexpr int TILE_BYTES = 128 * DH * 2;   // one Q, K or V tile
  static constexpr int STAGES = DH <= 64 ? 4 : (DH <= 96 ? 3 : 2);
  static constexpr int SMEM = TILE_BYTES + STAGES * 2 * TILE_BYTES + 1024 + 256;
};

struct Params {
  CUtensorMap tm_q, tm_k, tm_v;
  __nv_bfloat16* Z;
  const float* psel;
  int M, T, B, S, Sr, k, Do, shared_col, weighted, causal;
  int nq, items;
  float scale_log2;
  int32_t* status;
  int64_t spin;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Item {
  int b, s, qt;
};
__device__ __forceinline__ Item decode(const Params& P, int i) {
  Item it;
  const int bs = P.B * P.S;
  it.qt = P.causal ? P.nq - 1 - i / bs : i / bs;
  const int r = i % bs;
  it.s = r % P.S;
  it.b = r / P.S;
  return it;
}
__device__ __forceinline__ int kv_tiles(const Params& P, const Item& it) {
  return P.causal ? it.qt + 1 : P.nq;
}

// Waits (lane 0 polls, the warp follows); on giving up flags the timeout.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const Params& P,
                                          volatile int* abort_flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, P.spin);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (!ok && (threadIdx.x & 31) == 0) {
    *abort_flag = 1;
    atomicExch(P.status, kStatusTimeout);
  }
  return ok;
}

template <int DH>
__global__ void __launch_bounds__(THREADS, 1) attn_kernel(const __grid_constant__ Params P) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::TILE_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sKV + C::STAGES * 2 * C::TILE_BYTES);
  uint64_t* q_full = bar;
  uint64_t* q_empty = bar + 1;
  uint64_t* kv_full = bar + 2;
  uint64_t* kv_empty = kv_full + C::STAGES;
  uint64_t* s_full = kv_empty + C::STAGES;
  uint64_t* p_ready = s_full + 2;
  uint64_t* pv_done = p_ready + 2;
  uint64_t* o_full = pv_done + 2;
  uint64_t* o_free = o_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(o_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_ready[b], 4);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.tm_q);
    prefetch_tmap(&P.tm_k);
    prefetch_tmap(&P.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_o = tmem + 256;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA loads
    if (lane == 0) {
      int stage = 0;
      uint32_t kv_phase = 0, q_phase = 0;
      for (int i = blockIdx.x; i < P.items && !*abort_flag; i += gridDim.x) {
        const Item it = decode(P, i);
        const int q0 = it.qt * TQ;
        const int nkv = kv_tiles(P, it);
        if (!mbar_wait(q_empty, q_phase ^ 1, P.spin)) {
          *abort_flag = 1;
          atomicExch(P.status, kStatusTimeout);
          break;
        }
        q_phase ^= 1;
        mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
        const int qrow = it.s * P.M + it.b * P.T + q0;
#pragma unroll
        for (int c = 0; c < C::NC; ++c)
          tma_load_2d(sQ + c * C::CHUNK_BYTES, &P.tm_q, c * C::CW, qrow, q_full);
        const int kvh = it.s < P.Sr ? it.s / P.k : 0;
        for (int j = 0; j < nkv; ++j) {
          if (!mbar_wait(&kv_empty[stage], kv_phase ^ 1, P.spin)) {
            *abort_flag = 1;
            atomicExch(P.status, kStatusTimeout);
            break;
          }
          mbar_arrive_expect_tx(&kv_full[stage], 2 * C::TILE_BYTES);
          const int krow = kvh * P.M + it.b * P.T + j * TK;
          uint8_t* sK = sKV + stage * 2 * C::TILE_BYTES;
#pragma unroll
          for (int c = 0; c < C::NC; ++c) {
            tma_load_2d(sK + c * C::CHUNK_BYTES, &P.tm_k, c * C::CW, krow, &kv_full[stage]);
            tma_load_2d(sK + C::TILE_BYTES + c * C::CHUNK_BYTES, &P.tm_v, c * C::CW, krow,
                        &kv_full[stage]);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            kv_phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    const uint32_t idesc_s = idesc_bf16_f32(TQ, TK);
    const uint32_t idesc_pv = idesc_bf16_f32(TQ, DH) | (1u << 16);  // B (V) MN-major
    const uint32_t q_addr = smem_u32(sQ);
    int stage = 0;
    uint32_t kv_phase = 0, q_phase = 0;
    uint32_t jt = 0;
    int item_no = 0;
    bool ok = true;
    // O += P V for the KV tile held in `st`, whose S/P buffer is jt_ & 1.
    auto issue_pv = [&](int st, uint32_t jt_, bool first) -> bool {
      const int buf = jt_ & 1;
      if (!warp_wait(&p_ready[buf], (jt_ >> 1) & 1, P, abort_flag)) return false;
      if (first && item_no > 0 &&
          !warp_wait(o_free, (item_no - 1) & 1, P, abort_flag))
        return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t v_addr = smem_u32(sKV + st * 2 * C::TILE_BYTES + C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          // V as the MN-major B operand (N = head dim, K = keys): 16 keys are two 8-row
          // groups (SBO apart) of every chunk; the chunks are the MN atoms (LBO apart).
          const uint64_t vd = smem_desc_mn(v_addr + kk * 16 * C::ROW_BYTES, C::CHUNK_BYTES,
                                           8 * C::ROW_BYTES, C::LAYOUT);
          mma_ts(tmem_o, tmem + buf * 128 + kk * 8, vd, idesc_pv,
                 (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&kv_empty[st]);
        mma_commit(&pv_done[buf]);
      }
      __syncwarp();
      return true;
    };
    for (int i = blockIdx.x; i < P.items && ok && !*abort_flag; i += gridDim.x) {
      const Item it = decode(P, i);
      const int nkv = kv_tiles(P, it);
      if (!warp_wait(q_full, q_phase, P, abort_flag)) break;
      q_phase ^= 1;
      tc_fence_after();
      int pst = 0;
      uint32_t pjt = 0;
      for (int j = 0; j < nkv; ++j) {
        const int buf = jt & 1;
        if (!warp_wait(&kv_full[stage], kv_phase, P, abort_flag)) { ok = false; break; }
        if (jt >= 2 && !warp_wait(&pv_done[buf], ((jt - 2) >> 1) & 1, P, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t k_addr = smem_u32(sKV + stage * 2 * C::TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const int ch = (kk * 16) / C::CW, off = ((kk * 16) % C::CW) * 2;
            const uint64_t qd = smem_desc(q_addr + ch * C::CHUNK_BYTES + off, 8 * C::ROW_BYTES, C::LAYOUT);
            const uint64_t kd = smem_desc(k_addr + ch * C::CHUNK_BYTES + off, 8 * C::ROW_BYTES, C::LAYOUT);
            mma_ss(tmem + buf * 128, qd, kd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[buf]);
          if (j == nkv - 1) mma_commit(q_empty);
        }
        __syncwarp();
        if (j >= 1 && !issue_pv(pst, pjt, j == 1)) { ok = false; break; }
        pst = stage;
        pjt = jt;
        ++jt;
        if (++stage == C::STAGES) {
          stage = 0;
          kv_phase ^= 1;
        }
      }
      if (!ok) break;
      if (!issue_pv(pst, pjt, nkv == 1)) break;
      if (lane == 0) mma_commit(o_full);
      __syncwarp();
      ++item_no;
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    uint32_t jt = 0;
    int item_no = 0;
    const float cs = P.scale_log2;
    for (int i = blockIdx.x; i < P.items && !*abort_flag; i += gridDim.x) {
      const Item it = decode(P, i);
      const int q0 = it.qt * TQ;
      const int q = q0 + row;  // query position within the sequence
      const int nkv = kv_tiles(P, it);
      float m_used = 0.f, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv; ++j, ++jt) {
        const int buf = jt & 1;
        if (!warp_wait(&s_full[buf], (jt >> 1) & 1, P, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float s[TK];
        {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(tmem + lane_off + buf * 128 + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) s[c * 32 + x] = __uint_as_float(r[x]);
          }
        }
        const int kv0 = j * TK;
        const bool edge = (P.causal && kv0 + TK - 1 > q0) || (kv0 + TK > P.T);
        if (edge) {
#pragma unroll
          for (int c = 0; c < TK; ++c) {
            const int key = kv0 + c;
            if (key >= P.T || (P.causal && key > q)) s[c] = -INFINITY;
          }
        }
        float mx = s[0];
#pragma unroll
        for (int c = 1; c < TK; ++c) mx = fmaxf(mx, s[c]);
        float m_new = mx * cs;
        if (m_new == -INFINITY) m_new = 0.f;  // a row with every key masked
        bool need = false;
        float alpha = 1.f;
        if (j == 0) {
          m_used = m_new;
        } else if (m_new > m_used + kRescaleThreshold) {
          need = true;
          alpha = fast_exp2(m_used - m_new);
          m_used = m_new;
        }
        if (__any_sync(0xffffffffu, need)) {
          // O holds the sum through KV tile j-1: wait for that P V, then rescale in TMEM.
          if (!warp_wait(&pv_done[buf ^ 1], ((jt - 1) >> 1) & 1, P, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < DH; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem_o + lane_off + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 16; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
            tmem_st16(tmem_o + lane_off + c0, r);
          }
          tmem_wait_st();
          l *= alpha;
        }
        const float neg_m = -m_used;
#pragma unroll
        for (int c0 = 0; c0 < TK; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float p0 = fast_exp2(fmaf(s[c0 + 2 * x], cs, neg_m));
            const float p1 = fast_exp2(fmaf(s[c0 + 2 * x + 1], cs, neg_m));
            l += p0 + p1;
            pk[x] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tmem + lane_off + buf * 128 + c0 / 2, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready[buf]);
      }
      if (!ok) break;
      // ---- epilogue: O / l into Z
      if (!warp_wait(o_full, item_no & 1, P, abort_flag)) break;
      tc_fence_after();
      const bool valid = q < P.T;
      const int64_t tok = (int64_t)it.b * P.T + q;
      float scale = 1.f / l;
      int col;
      if (it.s < P.Sr) {
        col = it.s * DH;
        if (P.weighted && valid) scale *= P.psel[tok * P.Sr + it.s];
      } else {
        col = P.shared_col;
      }
      __nv_bfloat16* dst = P.Z + tok * P.Do + col;
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_o + lane_off + c0, r);
        tmem_wait_ld();
        if (valid) {
          uint4 v0, v1;
          v0.x = pack_bf16x2(__uint_as_float(r[0]) * scale, __uint_as_float(r[1]) * scale);
          v0.y = pack_bf16x2(__uint_as_float(r[2]) * scale, __uint_as_float(r[3]) * scale);
          v0.z = pack_bf16x2(__uint_as_float(r[4]) * scale, __uint_as_float(r[5]) * scale);
          v0.w = pack_bf16x2(__uint_as_float(r[6]) * scale, __uint_as_float(r[7]) * scale);
          v1.x = pack_bf16x2(__uint_as_float(r[8]) * scale, __uint_as_float(r[9]) * scale);
          v1.y = pack_bf16x2(__uint_as_float(r[10]) * scale, __uint_as_float(r[11]) * scale);
          v1.z = pack_bf16x2(__uint_as_float(r[12]) * scale, __uint_as_float(r[13]) * scale);
          v1.w = pack_bf16x2(__uint_as_float(r[14]) * scale, __uint_as_float(r[15]) * scale);
          *reinterpret_cast<uint4*>(dst + c0) = v0;
          *reinterpret_cast<uint4*>(dst + c0 + 8) = v1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      ++item_no;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH>
int launch_dh(gqe_ctx* h, int B, int T, int S, int shared_col, int weighted, int causal,
              int Do, cudaStream_t st) {
  using C = Cfg<DH>;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(attn_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM) != cudaSuccess)
      return -1;
    configured = true;
  }
  const int M = B * T;
  Params P;
  memset(&P, 0, sizeof(P));
  const CUtensorMapSwizzle sw = C::CW == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : C::CW == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!tmap_bf16_2d_ext(&P.tm_q, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW, TQ, sw) ||
      !tmap_bf16_2d_ext(&P.tm_k, h->ws.K, DH, (uint64_t)h->G * M, DH, C::CW, TK, sw) ||
      !tmap_bf16_2d_ext(&P.tm_v, h->ws.V, DH, (uint64_t)h->G * M, DH, C::CW, TK, sw))
    return -1;
  P.Z = static_cast<__nv_bfloat16*>(h->ws.Z);
  P.psel = h->ws.psel;
  P.M = M;
  P.T = T;
  P.B = B;
  P.S = S;
  P.Sr = h->G * h->k;
  P.k = h->k;
  P.Do = Do;
  P.shared_col = shared_col;
  P.weighted = weighted;
  P.causal = causal;
  P.nq = (T + TQ - 1) / TQ;
  P.items = B * S * P.nq;
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  P.status = h->ws.status;
  P.spin = h->spin_limit > 0 ? h->spin_limit : (int64_t)1 << 22;
  const int grid = P.items < h->num_sms ? P.items : h->num_sms;
  attn_kernel<DH><<<grid, THREADS, C::SMEM, st>>>(P);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace

int launch_tc_attention(gqe_ctx* h, int B, int T, int S, int has_shared, int variant,
                        int causal, int Do, cudaStream_t st) {
  (void)has_shared;
  const int Sr = h->G * h->k;
  const int shared_col = (Sr + (variant == GQE_VARIANT_GQE ? 1 : 0)) * h->d_h;
  const int weighted = variant == GQE_VARIANT_WEIGHTED_CONCAT;
  switch (h->d_h) {
    case 16: return launch_dh<16>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 32: return launch_dh<32>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 48: return launch_dh<48>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 64: return launch_dh<64>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 80: return launch_dh<80>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 96: return launch_dh<96>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 112: return launch_dh<112>(h, B, T, S, shared_col, weighted, causal, Do, st);
    case 128: return launch_dh<128>(h, B, T, S, shared_col, weighted, causal, Do, st);
    default: return -1;
  }
}

}  // namespace gqe
