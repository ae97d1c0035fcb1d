// Tensor-core (tcgen05) causal / non-causal softmax attention of the GQE query streams.
//
// Stream s < G*k holds the routed queries of group s / k and reads that group's dense KV
// head; the last stream is the always-on shared head and reads KV head 0 ("GQE: Grouped
// Query Experts" README, Algorithm Overview; gist.science summary, Output Construction).
// Every stream has one query per token, so the work is a grouped-query attention with
// S = G*k + 1 query heads over G KV heads; the savings of GQE come from S < N + 1.
//
// Work item = (sequence b, stream s, 128-query tile); persistent CTAs, two per SM, take
// items heaviest first (causal tiles near the end of a sequence have the most keys). The
// two CTAs of an SM interleave: while one computes exponentials the other's products run,
// and each hides the other's waits. Per CTA:
//   warp 0     TMA: the Q tile once per item, then K tiles into their own ring;
//   warp 1     owns the TMEM columns; one elected lane issues S = Q K^T (A and B from
//              shared memory) into TMEM and O += P V with P read from TMEM (the TS form)
//              and V as an MN-major shared-memory operand;
//   warp 2     TMA: V tiles into a second ring (a K tile is released as soon as its S is
//              done, so K runs ahead of the V tiles that the later P V products still hold);
//   warp 3     idle. With two CTAs per SM the launch gives every thread 128 registers;
//              warps 0-3 drop to 48 (setmaxnreg) so that the softmax warpgroup can take 208;
//   warps 4-7  softmax: one query row per thread, 128 scores per KV tile in registers,
//              exp2 against the running row maximum, P kept in registers as bf16 pairs until
//              the tile is done, then written to TMEM. O is rescaled in TMEM only when a row
//              maximum grows by more than 2^8 (rare after the first tiles). At the end of an
//              item the same warps normalise O by the row sum, apply the weighted_concat
//              scale if any, and store the row into its block of Z.
// P has TMEM columns of its own. S runs a tile ahead of the softmax warps: once P(j) is in
// TMEM the MMA warp issues P(j) V at once (the softmax warps wait for it before they write
// P(j+1)), then S(j+2) as soon as they hold S(j+1) in registers. For head dims up to 48 the row sums come from the tensor core (a chunk of
// ones after every V tile). Head dims above 64 run one CTA per SM with 512 TMEM columns.
#include <cudaTypedefs.h>

#include "gqe_common.cuh"
#include "exp2_fma.cuh"
#include "tc_ptx.cuh"

namespace gqe {

bool tmap_bf16_2d_ext(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                      uint64_t ld, uint32_t box_cols, uint32_t box_rows,
                      CUtensorMapSwizzle sw);
bool tmap_bf16_chunked(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                       uint64_t ld, uint32_t chunk_cols, uint32_t box_rows,
                       CUtensorMapSwizzle sw);

namespace {

using namespace tc;

// Warps: 0 Q/K loads, 1 MMA, 2 V loads, 3 idle (it only hands its registers to the softmax
// warpgroup), 4-7 softmax + epilogue.
constexpr int THREADS = 256;
constexpr int kSmallRegs = 48;   // warpgroup 0 after setmaxnreg.dec (two CTAs per SM)
constexpr int kLargeRegs = 208;  // softmax warpgroup after setmaxnreg.inc
constexpr int TQ = 128;                    // queries per tile (MMA M, TMEM lanes)
constexpr int TK = 128;                    // keys per tile (S MMA N)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int DH>
struct Cfg {
  // Chunk width (columns per swizzle atom). Head dims with tensor-core row sums (<= 48)
  // use 16-column chunks, so the 16 columns of ones after a V tile are exactly one chunk and
  // the P V operand of N = d_h + 16 columns is a whole number of chunks.
  static constexpr int CW = (DH % 64 == 0) ? 64 : (DH % 32 == 0 && DH > 48) ? 32 : 16;
  static constexpr int NC = DH / CW;                                         // chunks
  static constexpr uint32_t LAYOUT =
      CW == 64 ? kSwizzle128B : (CW == 32 ? kSwizzle64B : kSwizzle32B);
  static constexpr int ROW_BYTES = CW * 2;          // bytes per row inside a chunk
  static constexpr int CHUNK_BYTES = 128 * ROW_BYTES;
  static constexpr int TILE_BYTES = 128 * DH * 2;   // one Q, K or V tile
  // Small head dims let the tensor core form the softmax row sums: every V tile is
  // followed by a constant chunk of ones, so O += P [V | 1] leaves sum_j P in the columns
  // after the head dim (from the same bf16 P the product uses). Larger head dims keep the
  // sums in registers (their products are already the larger cost).
  static constexpr bool SUM_MMA = DH <= 48;
  static constexpr int ONES_BYTES = SUM_MMA ? CHUNK_BYTES : 0;
  static constexpr int N_PV = DH + (SUM_MMA ? 16 : 0);  // PV MMA width
  static constexpr int V_BYTES = TILE_BYTES + ONES_BYTES;  // one V stage
  // Two CTAs per SM while both fit (TMEM 256 columns each, shared memory), else one.
  static constexpr int CTAS = DH <= 64 ? 2 : 1;
  static constexpr int TMEM_COLS = CTAS == 2 ? 256 : 512;
  // Separate K and V rings: a K tile is released as soon as its S product is done, so K
  // runs several tiles ahead of the V tiles that the later P V products hold.
  static constexpr int K_STAGES = DH <= 48 ? 4 : 3;
  static constexpr int V_STAGES = DH == 64 ? 2 : 3;
  static constexpr int SMEM = TILE_BYTES * (1 + K_STAGES) + V_STAGES * V_BYTES + 1024 + 256;
  // TMEM columns: S at 0, P (bf16 pairs) at 128, O at 192.
  static constexpr int P_COL = 128;
  static constexpr int O_COL = 192;
  static_assert(O_COL + N_PV <= TMEM_COLS, "TMEM budget");
  static_assert(!SUM_MMA || CW == 16, "the ones chunk must be one 16-column chunk");
  static_assert(N_PV % CW == 0, "P V reads whole chunks");
  static_assert(CTAS * (SMEM + 1024) <= 228 * 1024, "shared memory budget");
};
// Exponentials: of every 8 pairs of scores, this many go to the FMA-pipe polynomial and
// the rest to the MUFU unit (16 results per SM per clock on B200).
#ifndef GQE_ATTN_FMA_PAIRS_OF_8
#define GQE_ATTN_FMA_PAIRS_OF_8 3
#endif
constexpr int kFmaPairsOf8 = GQE_ATTN_FMA_PAIRS_OF_8;

struct Params {
  CUtensorMap tm_q, tm_k, tm_v;
  __nv_bfloat16* Z;
  float* lse;  // [S, M] per-row log2-sum-exp2 of the scaled scores (for the backward pass)
  const float* psel;  // [M, psel_stride]: stream s's p at column psel_off + s
  int M, T, B, S, Sr, k, Do, shared_col, weighted, causal;
  int psel_stride, psel_off;
  int nq, items;
  int chunked;  // 1: tm_q / tm_k / tm_v are 3D chunked maps, one copy per tile
  float scale_log2;
  int* next_item;  // [2] item counter and exit counter (zero at launch; the last CTA to
                   // leave sets both back to zero)
  int32_t* status;
  int64_t spin;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Item {
  int b, s, qt, nkv;
};
__device__ __forceinline__ Item decode(const Params& P, int i) {
  Item it;
  const int bs = P.B * P.S;
  it.qt = P.causal ? P.nq - 1 - i / bs : i / bs;
  const int r = i % bs;
  it.s = r % P.S;
  it.b = r / P.S;
  it.nkv = P.causal ? it.qt + 1 : P.nq;
  return it;
}

// Waits with every lane polling (no divergence); the outcome is made warp-uniform. On
// giving up, flags the timeout.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const Params& P,
                                          volatile int* abort_flag) {
  const bool ok = !__any_sync(0xffffffffu, !mbar_wait(bar, parity, P.spin));
  if (!ok && (threadIdx.x & 31) == 0) {
    *abort_flag = 1;
    atomicExch(P.status, kStatusTimeout);
  }
  return ok;
}

template <int DH>
__global__ void __launch_bounds__(THREADS, Cfg<DH>::CTAS)
attn_kernel(const __grid_constant__ Params P) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::TILE_BYTES;                 // K ring
  uint8_t* sV = sK + C::K_STAGES * C::TILE_BYTES;     // V ring: V tile[, ones chunk]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sV + C::V_STAGES * C::V_BYTES);
  uint64_t* q_full = bar;
  uint64_t* q_empty = bar + 1;
  uint64_t* k_full = bar + 2;
  uint64_t* k_empty = k_full + C::K_STAGES;
  uint64_t* v_full = k_empty + C::K_STAGES;
  uint64_t* v_empty = v_full + C::V_STAGES;
  uint64_t* s_full = v_empty + C::V_STAGES;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_ready = s_free + 1;
  uint64_t* pv_done = p_ready + 1;
  uint64_t* o_full = pv_done + 1;
  uint64_t* o_free = o_full + 1;
  uint64_t* item_full = o_free + 1;   // [2] item ring, filled by the K/Q load warp
  uint64_t* item_empty = item_full + 2;  // [2] read by the V load, MMA and softmax warps
  volatile int* item_ring = reinterpret_cast<volatile int*>(item_empty + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(item_empty + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if constexpr (C::SUM_MMA) {
    // the constant ones chunk after every stage's V tile (bf16 1.0 in every element, so
    // the swizzle does not matter); TMA never writes it
    for (int st = 0; st < C::V_STAGES; ++st) {
      uint4* o = reinterpret_cast<uint4*>(sV + st * C::V_BYTES + C::TILE_BYTES);
      for (int i = threadIdx.x; i < C::ONES_BYTES / 16; i += THREADS)
        o[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    }
    fence_async_shared();
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::K_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < C::V_STAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_ready, 4);
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    for (int r = 0; r < 2; ++r) {
      mbar_init(&item_full[r], 1);
      mbar_init(&item_empty[r], 6);  // the V load warp, the MMA warp, four softmax warps
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
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
  pdl_wait();  // Q, K, V and (weighted_concat) p_sel are complete from here on
  pdl_allow_next();

  // MMA and softmax warps: the next item index from the ring (warp-collective); the slot
  // is released as soon as it has been read. -1 means no work is left.
  auto next_item = [&](int& i, int& islot, uint32_t& iphase) -> bool {
    if (!warp_wait(&item_full[islot], iphase, P, abort_flag)) return false;
    i = item_ring[islot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[islot]);
    if (++islot == 2) {
      islot = 0;
      iphase ^= 1;
    }
    return true;
  };

  // Two CTAs per SM launch with 128 registers per thread; warpgroup 0 (TMA, MMA and two
  // idle warps) gives most of its share to the softmax warpgroup. The two counts add up
  // to the launch allocation exactly: 48 * 128 + 208 * 128 = 256 * 128.
  static_assert(kSmallRegs * 128 + kLargeRegs * 128 == THREADS * (65536 / (2 * THREADS)),
                "register split must equal the launch allocation");
  if (warp < 4) {
  if constexpr (C::CTAS == 2) setmaxnreg_dec<kSmallRegs>();
  if (warp == 0) {
    // ---------------------------------------------------------------- Q and K loads
    if (lane == 0) {
      int kst = 0;
      uint32_t k_phase = 0, q_phase = 0;
      int islot = 0;
      uint32_t iphase = 0;
      while (!*abort_flag) {
        // claim the next item (heaviest first) and publish it to the other warps
        if (!mbar_wait(&item_empty[islot], iphase ^ 1, P.spin)) {
          *abort_flag = 1;
          atomicExch(P.status, kStatusTimeout);
          break;
        }
        int i = atomicAdd(P.next_item, 1);
        if (i >= P.items) i = -1;
        item_ring[islot] = i;
        mbar_arrive(&item_full[islot]);
        if (++islot == 2) {
          islot = 0;
          iphase ^= 1;
        }
        if (i < 0) break;
        const Item it = decode(P, i);
        if (!mbar_wait(q_empty, q_phase ^ 1, P.spin)) {
          *abort_flag = 1;
          atomicExch(P.status, kStatusTimeout);
          break;
        }
        q_phase ^= 1;
        mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
        const int qrow = it.s * P.M + it.b * P.T + it.qt * TQ;
        if (C::NC > 1 && P.chunked) {
          tma_load_3d(sQ, &P.tm_q, 0, qrow, 0, q_full);
        } else {
#pragma unroll
          for (int c = 0; c < C::NC; ++c)
            tma_load_2d(sQ + c * C::CHUNK_BYTES, &P.tm_q, c * C::CW, qrow, q_full);
        }
        const int kvh = it.s < P.Sr ? it.s / P.k : 0;
        const int krow0 = kvh * P.M + it.b * P.T;
        for (int j = 0; j < it.nkv; ++j) {
          if (!mbar_wait(&k_empty[kst], k_phase ^ 1, P.spin)) {
            *abort_flag = 1;
            atomicExch(P.status, kStatusTimeout);
            break;
          }
          mbar_arrive_expect_tx(&k_full[kst], C::TILE_BYTES);
          if (C::NC > 1 && P.chunked) {
            tma_load_3d(sK + kst * C::TILE_BYTES, &P.tm_k, 0, krow0 + j * TK, 0, &k_full[kst]);
          } else {
#pragma unroll
            for (int c = 0; c < C::NC; ++c)
              tma_load_2d(sK + kst * C::TILE_BYTES + c * C::CHUNK_BYTES, &P.tm_k, c * C::CW,
                          krow0 + j * TK, &k_full[kst]);
          }
          if (++kst == C::K_STAGES) {
            kst = 0;
            k_phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- V loads
    if (lane == 0) {
      int vst = 0;
      uint32_t v_phase = 0;
      int islot = 0;
      uint32_t iphase = 0;
      while (!*abort_flag) {
        if (!mbar_wait(&item_full[islot], iphase, P.spin)) {
          *abort_flag = 1;
          atomicExch(P.status, kStatusTimeout);
          break;
        }
        const int i = item_ring[islot];
        mbar_arrive(&item_empty[islot]);
        if (++islot == 2) {
          islot = 0;
          iphase ^= 1;
        }
        if (i < 0) break;
        const Item it = decode(P, i);
        const int kvh = it.s < P.Sr ? it.s / P.k : 0;
        const int krow0 = kvh * P.M + it.b * P.T;
        for (int j = 0; j < it.nkv; ++j) {
          if (!mbar_wait(&v_empty[vst], v_phase ^ 1, P.spin)) {
            *abort_flag = 1;
            atomicExch(P.status, kStatusTimeout);
            break;
          }
          mbar_arrive_expect_tx(&v_full[vst], C::TILE_BYTES);
          if (C::NC > 1 && P.chunked) {
            tma_load_3d(sV + vst * C::V_BYTES, &P.tm_v, 0, krow0 + j * TK, 0, &v_full[vst]);
          } else {
#pragma unroll
            for (int c = 0; c < C::NC; ++c)
              tma_load_2d(sV + vst * C::V_BYTES + c * C::CHUNK_BYTES, &P.tm_v, c * C::CW,
                          krow0 + j * TK, &v_full[vst]);
          }
          if (++vst == C::V_STAGES) {
            vst = 0;
            v_phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    // Lean: descriptors are built once; each product's descriptor is a base plus a
    // constant (the address field is the low 14 bits, in 16-byte units).
    const uint32_t idesc_s = idesc_bf16_f32(TQ, TK);
    const uint32_t idesc_pv = idesc_bf16_f32(TQ, C::N_PV) | (1u << 16);  // B (V) MN-major
    const uint64_t q_desc = smem_desc(smem_u32(sQ), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t k_desc = smem_desc(smem_u32(sK), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t v_desc =
        smem_desc_mn(smem_u32(sV), C::CHUNK_BYTES, 8 * C::ROW_BYTES, C::LAYOUT);
    constexpr uint32_t kKStep = C::TILE_BYTES >> 4;
    constexpr uint32_t kVStep = C::V_BYTES >> 4;
    int kst = 0, vst = 0;
    uint32_t k_phase = 0, v_phase = 0, q_phase = 0;
    uint32_t n_sf = 0, n_p = 0, n_o = 0;  // uses of s_free / p_ready / o_full
    bool ok = true;

    // Order of issue per item: S(0), S(1); then for every tile j, once P(j) is ready, P(j) V
    // and then S(j+2) (as soon as the softmax warps hold S(j+1) in registers). P(j) V is
    // queued behind nothing the softmax warps do not need first, and S(j+2) is still a whole
    // tile ahead of its use.
    // S = Q K^T for the next K tile; its stage is released when the product is done.
    auto issue_s = [&](bool last_s) -> bool {
      if (!warp_wait(&k_full[kst], k_phase, P, abort_flag)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t kd = k_desc + (uint64_t)(kst * kKStep);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t o = (((kk * 16) / C::CW) * C::CHUNK_BYTES + ((kk * 16) % C::CW) * 2) >> 4;
          mma_ss(tmem, q_desc + o, kd + o, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        mma_commit(&k_empty[kst]);
        if (last_s) mma_commit(q_empty);
      }
      __syncwarp();
      if (++kst == C::K_STAGES) {
        kst = 0;
        k_phase ^= 1;
      }
      return true;
    };
    int islot = 0;
    uint32_t iphase = 0;
    while (ok && !*abort_flag) {
      int i;
      if (!next_item(i, islot, iphase)) break;
      if (i < 0) break;
      const Item it = decode(P, i);
      const int nk = it.nkv;
      if (!warp_wait(q_full, q_phase, P, abort_flag)) break;
      q_phase ^= 1;
      if (!issue_s(nk == 1)) break;  // S(0)
      if (nk > 1) {
        if (!warp_wait(s_free, n_sf & 1, P, abort_flag)) break;  // S(0) is in registers
        ++n_sf;
        if (!issue_s(nk == 2)) break;  // S(1)
      }
      for (int j = 0; j < nk; ++j) {
        if (!warp_wait(p_ready, n_p & 1, P, abort_flag)) { ok = false; break; }
        ++n_p;
        if (j == 0 && n_o > 0 && !warp_wait(o_free, (n_o - 1) & 1, P, abort_flag)) {
          ok = false;
          break;
        }
        if (!warp_wait(&v_full[vst], v_phase, P, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool last = j + 1 == nk;
        if (elect_one()) {
          // O += P V (V: the MN-major B operand, N = head dim[+ ones], K = keys; 16 keys
          // are two 8-row groups of every chunk)
          const uint64_t vd = v_desc + (uint64_t)(vst * kVStep);
#pragma unroll
          for (int kk = 0; kk < TK / 16; ++kk)
            mma_ts(tmem + C::O_COL, tmem + C::P_COL + kk * 8,
                   vd + (uint64_t)((kk * 16 * C::ROW_BYTES) >> 4), idesc_pv,
                   (j == 0 && kk == 0) ? 0u : 1u);
          mma_commit(pv_done);
          if (last) mma_commit(o_full);
          mma_commit(&v_empty[vst]);
        }
        __syncwarp();
        if (j + 2 < nk) {
          // then S(j+2), once the softmax warps hold S(j+1) in registers
          if (!warp_wait(s_free, n_sf & 1, P, abort_flag)) { ok = false; break; }
          ++n_sf;
          if (!issue_s(j + 3 == nk)) { ok = false; break; }  // S(j+2)
        }
        if (last) ++n_o;
        if (++vst == C::V_STAGES) {
          vst = 0;
          v_phase ^= 1;
        }
      }
    }
  }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    if constexpr (C::CTAS == 2) setmaxnreg_inc<kLargeRegs>();
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off;
    const uint32_t t_p = tmem + lane_off + C::P_COL;
    const uint32_t t_o = tmem + lane_off + C::O_COL;
    uint32_t n_s = 0, n_o = 0;  // uses of s_full / o_full so far
    const float cs = P.scale_log2;
    int islot = 0;
    uint32_t iphase = 0;
    while (!*abort_flag) {
      int i;
      if (!next_item(i, islot, iphase)) break;
      if (i < 0) break;
      const Item it = decode(P, i);
      const int nkv = it.nkv;
      const int q0 = it.qt * TQ;
      const int q = q0 + row;  // query position within the sequence
      float m_used = 0.f, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        if (!warp_wait(s_full, n_s & 1, P, abort_flag)) { ok = false; break; }
        ++n_s;
        tc_fence_after();
        float s[TK];
        {
          uint32_t r[TK];
          tmem_ld128_wait(t_s, r);
#pragma unroll
          for (int c = 0; c < TK; ++c) s[c] = __uint_as_float(r[c]);
        }
        if (j + 1 < nkv) {
          // S is in registers: the next S may be written.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
        const int kv0 = j * TK;
        if ((P.causal && kv0 + TK - 1 > q0) || (kv0 + TK > P.T)) {
          // keys past the sequence end, and (causal) keys after this query
          const int lim = P.causal ? min(q + 1, P.T) : P.T;
#pragma unroll
          for (int c = 0; c < TK; ++c)
            if (kv0 + c >= lim) s[c] = -INFINITY;
        }
        // Row maximum in two halves of 64 columns: the exponentials of the first half need
        // only its own maximum (and the running reference), so the second half's maximum is
        // formed while they run. A reference moves only when a maximum passes it by more
        // than the threshold; if the second half's does, the first half's P is rescaled
        // (rare after a row's first tiles).
        static_assert(TK == 128, "the row-maximum schedule covers 128 columns");
        float mp[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) mp[x] = fmax3(s[x], s[8 + x], s[16 + x]);        // 0..23
#pragma unroll
        for (int c = 24; c < 56; c += 16)                                           // 24..55
#pragma unroll
          for (int x = 0; x < 8; ++x) mp[x] = fmax3(mp[x], s[c + x], s[c + 8 + x]);
#pragma unroll
        for (int x = 0; x < 8; ++x) mp[x] = fmaxf(mp[x], s[56 + x]);                // 56..63
        const float m_old = m_used;
        {
          const float m_a = fmaxf(fmax3(mp[0], mp[1], mp[2]),
                                  fmax3(fmax3(mp[3], mp[4], mp[5]), mp[6], mp[7])) * cs;
          if (j == 0)
            m_used = m_a == -INFINITY ? 0.f : m_a;  // a half with every key masked
          else if (m_a > m_used + kRescaleThreshold)
            m_used = m_a;
        }
        // p = exp2(s * scale - m) with a packed FMA for the argument; most pairs on MUFU,
        // kFmaPairsOf8 of every 8 on the FMA-pipe polynomial. P is kept in registers as
        // bf16 pairs until the whole tile is done.
        const float2 cs2 = make_float2(cs, cs);
        uint32_t pk[TK / 2];
        float2 lsa[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 lsb[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        {
          const float2 nm2 = make_float2(-m_used, -m_used);
#pragma unroll
          for (int x = 0; x < TK / 4; ++x) {
            const float2 t = fma2(make_float2(s[2 * x], s[2 * x + 1]), cs2, nm2);
            const float2 p = (x & 7) >= 8 - kFmaPairsOf8
                                 ? exp2_fma2(t)
                                 : make_float2(fast_exp2(t.x), fast_exp2(t.y));
            if constexpr (!C::SUM_MMA) lsa[x & 1] = add2(lsa[x & 1], p);
            pk[x] = pack_bf16x2(p.x, p.y);
          }
        }
        // second half's maximum
#pragma unroll
        for (int x = 0; x < 8; ++x) mp[x] = fmax3(s[64 + x], s[72 + x], s[80 + x]);  // 64..87
#pragma unroll
        for (int c = 88; c < 120; c += 16)                                          // 88..119
#pragma unroll
          for (int x = 0; x < 8; ++x) mp[x] = fmax3(mp[x], s[c + x], s[c + 8 + x]);
#pragma unroll
        for (int x = 0; x < 8; ++x) mp[x] = fmaxf(mp[x], s[120 + x]);               // 120..127
        {
          const float m_b = fmaxf(fmax3(mp[0], mp[1], mp[2]),
                                  fmax3(fmax3(mp[3], mp[4], mp[5]), mp[6], mp[7])) * cs;
          if (m_b > m_used + kRescaleThreshold) {
            const float a2 = fast_exp2(m_used - m_b);
#pragma unroll
            for (int x = 0; x < TK / 4; ++x)
              pk[x] = pack_bf16x2(__uint_as_float(pk[x] << 16) * a2,
                                  __uint_as_float(pk[x] & 0xffff0000u) * a2);
            if constexpr (!C::SUM_MMA) {
              lsa[0] = mul2(lsa[0], make_float2(a2, a2));
              lsa[1] = mul2(lsa[1], make_float2(a2, a2));
            }
            m_used = m_b;
          }
        }
        {
          const float2 nm2 = make_float2(-m_used, -m_used);
#pragma unroll
          for (int x = TK / 4; x < TK / 2; ++x) {
            const float2 t = fma2(make_float2(s[2 * x], s[2 * x + 1]), cs2, nm2);
            const float2 p = (x & 7) >= 8 - kFmaPairsOf8
                                 ? exp2_fma2(t)
                                 : make_float2(fast_exp2(t.x), fast_exp2(t.y));
            if constexpr (!C::SUM_MMA) lsb[x & 1] = add2(lsb[x & 1], p);
            pk[x] = pack_bf16x2(p.x, p.y);
          }
        }
        // O is rescaled when this tile moved the reference (never on a row's first tile)
        const bool need = j > 0 && m_used != m_old;
        const float alpha = need ? fast_exp2(m_old - m_used) : 1.f;
        if constexpr (!C::SUM_MMA) {
          const float2 a = add2(add2(lsa[0], lsa[1]), add2(lsb[0], lsb[1]));
          l = l * alpha + (a.x + a.y);
        }
        // S(j) was issued without waiting for P(j-1) V, and the exponentials above did not
        // need it either: only now wait for that product before overwriting P or
        // rescaling O.
        if (j > 0 && !warp_wait(pv_done, (n_s - 2) & 1, P, abort_flag)) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, need)) {
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < C::N_PV; c0 += 16) {
            uint32_t r[16];
            tmem_ld16_wait(t_o + c0, r);
#pragma unroll
            for (int x = 0; x < 16; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
            tmem_st16(t_o + c0, r);
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < TK / 2; c0 += 16) {
          uint32_t r[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) r[x] = pk[c0 + x];
          tmem_st16(t_p + c0, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);
      }
      if (!ok) break;
      // ---- epilogue: O / l into Z
      if (!warp_wait(o_full, n_o & 1, P, abort_flag)) break;
      ++n_o;
      tc_fence_after();
      const bool valid = q < P.T;
      const int64_t tok = (int64_t)it.b * P.T + q;
      if constexpr (C::SUM_MMA) {
        uint32_t r[16];
        tmem_ld16_wait(t_o + DH, r);
        l = __uint_as_float(r[0]);
      }
      float scale = 1.f / l;
      // the row's log2-sum-exp2 of its scaled scores: p = exp2(s * scale_log2 - lse)
      if (valid) P.lse[(int64_t)it.s * P.M + tok] = m_used + __log2f(l);
      int col;
      if (it.s < P.Sr) {
        col = it.s * DH;
        if (P.weighted && valid) scale *= P.psel[tok * P.psel_stride + P.psel_off + it.s];
      } else {
        col = P.shared_col;
      }
      __nv_bfloat16* dst = P.Z + tok * P.Do + col;
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 16) {
        uint32_t r[16];
        tmem_ld16_wait(t_o + c0, r);
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
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // every CTA has taken its last item: the last one to leave resets the counters
  if (threadIdx.x == 0 && atomicAdd(P.next_item + 1, 1) == (int)gridDim.x - 1) {
    P.next_item[0] = 0;
    P.next_item[1] = 0;
  }
}

template <int DH>
int launch_dh(gqe_ctx* h, int B, int T, int S, int shared_col, int weighted, int causal,
              int Do, cudaStream_t st) {
  using C = Cfg<DH>;
  if (!set_smem_limit_once<attn_kernel<DH>>(C::SMEM)) return -1;
  const int M = B * T;
  Params P;
  memset(&P, 0, sizeof(P));
  const CUtensorMapSwizzle sw = C::CW == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : C::CW == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_32B;
  // One copy per tile where the driver accepts the chunked 3D maps, else one per chunk.
  const uint64_t kv_rows = (uint64_t)(h->g1 - h->g0) * M;  // this handle's KV heads
  P.chunked = C::NC > 1 &&
              tmap_bf16_chunked(&P.tm_q, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW, TQ, sw) &&
              tmap_bf16_chunked(&P.tm_k, h->ws.K, DH, kv_rows, DH, C::CW, TK, sw) &&
              tmap_bf16_chunked(&P.tm_v, h->ws.V, DH, kv_rows, DH, C::CW, TK, sw);
  if (!P.chunked &&
      (!tmap_bf16_2d_ext(&P.tm_q, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW, TQ, sw) ||
       !tmap_bf16_2d_ext(&P.tm_k, h->ws.K, DH, kv_rows, DH, C::CW, TK, sw) ||
       !tmap_bf16_2d_ext(&P.tm_v, h->ws.V, DH, kv_rows, DH, C::CW, TK, sw)))
    return -1;
  P.Z = static_cast<__nv_bfloat16*>(h->ws.Z);
  P.lse = h->ws.lse;
  P.psel = h->ws.psel;
  P.M = M;
  P.T = T;
  P.B = B;
  P.S = S;
  P.Sr = (h->g1 - h->g0) * h->k;
  P.k = h->k;
  P.psel_stride = h->G * h->k;
  P.psel_off = h->g0 * h->k;
  P.Do = Do;
  P.shared_col = shared_col;
  P.weighted = weighted;
  P.causal = causal;
  P.nq = (T + TQ - 1) / TQ;
  P.items = B * S * P.nq;
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  P.status = h->ws.status;
  P.spin = h->spin_limit > 0 ? h->spin_limit : (int64_t)1 << 22;
  const int slots = C::CTAS * h->num_sms;
  const int grid = P.items < slots ? P.items : slots;
  P.next_item = h->ws.attn_counter;
  return launch_pdl(attn_kernel<DH>, dim3(grid), dim3(THREADS), C::SMEM, st, P) == cudaSuccess
             ? 1
             : -1;
}

}  // namespace

int launch_tc_attention(gqe_ctx* h, int B, int T, int S, int has_shared, int variant,
                        int causal, int Do, cudaStream_t st) {
  (void)has_shared;
  const int Sr = (h->g1 - h->g0) * h->k;
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
