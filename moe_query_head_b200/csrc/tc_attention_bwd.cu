// Tensor-core (tcgen05) backward pass of the GQE attention: the gradients of the query
// streams, keys and values, given the forward's per-row log2-sum-exp2 (lse), the upstream
// gradient dO of every stream's output and D = rowsum(dO * O).
//
// Stream s < G*k holds the routed queries of group s / k and reads that group's KV head; the
// last stream is the always-on shared head and reads KV head 0 ("GQE: Grouped Query
// Experts" README, Algorithm Overview; gist.science summary, Output Construction). With
// P = softmax(Q K^T / sqrt(d_h)) (causal or not), dP = dO V^T and dS = P * (dP - D):
//   dQ = dS K / sqrt(d_h),   dK = sum over the head's streams of dS^T Q / sqrt(d_h),
//   dV = sum over the head's streams of P^T dO.
//
// Two kernels, neither with atomics (every output row is written by one CTA, so the result
// is the same from run to run). Head dims up to 64 run two CTAs per SM (256 TMEM columns
// each; warpgroup 0 gives registers to the softmax warpgroup), larger ones (80 to 128) one
// CTA per SM with 512 columns and the whole register file:
//   attn_bwd_dq_kernel    work item = (sequence, stream, 128-query tile); per 64-key step
//                         S = Q K^T and dP = dO V^T (both operands from shared memory) into
//                         TMEM, the softmax warpgroup forms dS in bf16 in TMEM, and
//                         dQ += dS K (A from TMEM, K as an MN-major shared-memory operand)
//                         accumulates in TMEM. The routed stream (g, r) of token t lands in
//                         row t of dQ_exp [M, N d_h] at the column block of its expert
//                         g E + sel[t, g, r]; the shared stream in dQ_sh [M, d_h].
//   attn_bwd_dkdv_kernel  work item = (sequence, KV head, 128-key tile); per job (a stream
//                         that reads the head, a tile of 48 queries; 32 at d_h = 64, 64
//                         above),
//                         S^T = K Q^T and dP^T = V dO^T into TMEM, the softmax warpgroup
//                         (one key per thread) forms P^T and dS^T in bf16 in TMEM, and
//                         dV += P^T dO, dK += dS^T Q accumulate in TMEM over all of the
//                         head's streams. dK, dV land token-major in [M, G d_h].
// Warps: 0 TMA loads, 1 TMEM owner and MMA issue, 2-3 idle, 4-7 softmax and epilogue; the
// next tile's S and dP are issued as soon as the softmax warps hold the current ones in
// registers. Persistent CTAs take items heaviest first. Head dims 16 to 128.
#include <cudaTypedefs.h>

#include "gqe_common.cuh"
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

constexpr int THREADS = 256;
constexpr int TQ = 128;  // query rows of a tile
constexpr int TK = 128;  // key rows of a tile

template <int DH>
struct BCfg {
  static_assert(DH % 16 == 0 && DH <= 128, "the backward kernels take head dims up to 128");
  // shared-memory chunking: 64-column chunks (128-byte swizzle) for multiples of 64, else
  // 16-column chunks (32-byte swizzle)
  static constexpr int CW = (DH % 64 == 0) ? 64 : 16;
  static constexpr int NC = DH / CW;
  static constexpr uint32_t LAYOUT = CW == 64 ? kSwizzle128B : kSwizzle32B;
  static constexpr int ROW_BYTES = CW * 2;
  static constexpr int CHUNK_BYTES = 128 * ROW_BYTES;
  static constexpr int TILE_BYTES = 128 * DH * 2;
  // CTAs per SM: two while each CTA's TMEM fits in 256 columns
  static constexpr int CTAS = DH <= 64 ? 2 : 1;
  static constexpr int TMEM_COLS = CTAS == 2 ? 256 : 512;
};

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // Q, dO [S M, d_h]; K, V [G M, d_h]; 128-row boxes
  CUtensorMap tm_k64, tm_v64;           // K, V with 64-row boxes (the dQ kernel)
  CUtensorMap tm_qj, tm_doj;            // Q, dO with job-row boxes (the dK / dV kernel)
  const float* lse;     // [S, M]
  const float* dsum;    // [S, M] rowsum(dO * O)
  const int32_t* sel;   // [M, sel_stride]: stream s's selection at column sel_off + s
  __nv_bfloat16* dq_exp;  // [M, N d_h]
  __nv_bfloat16* dq_sh;   // [M, d_h]
  __nv_bfloat16* dk;      // [M, G d_h]
  __nv_bfloat16* dv;      // [M, G d_h]
  // S, Sr, G, N: this handle's streams, routed streams, KV heads and experts (a group range
  // counts from its first group)
  int M, T, B, S, Sr, k, G, E, N, has_shared, causal, nq, items, chunked;
  int sel_stride, sel_off;
  float scale_log2;  // log2(e) / sqrt(d_h)
  float scale;       // 1 / sqrt(d_h)
  int* counter;      // [2] item counter and exit counter (zero at launch; reset by the last CTA)
  int32_t* status;
  int64_t spin;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const BwdParams& P,
                                          volatile int* abort_flag) {
  const bool ok = !__any_sync(0xffffffffu, !mbar_wait(bar, parity, P.spin));
  if (!ok && (threadIdx.x & 31) == 0) {
    *abort_flag = 1;
    atomicExch(P.status, kStatusTimeout);
  }
  return ok;
}
__device__ __forceinline__ bool lane_wait(uint64_t* bar, uint32_t parity, const BwdParams& P,
                                          volatile int* abort_flag) {
  if (mbar_wait(bar, parity, P.spin)) return true;
  *abort_flag = 1;
  atomicExch(P.status, kStatusTimeout);
  return false;
}

// One tile of ROWS rows (128 or 64): chunk after chunk, each ROWS x CW.
template <int DH, int ROWS = 128>
__device__ __forceinline__ void load_tile(const BwdParams& P, const CUtensorMap* map,
                                          uint8_t* dst, int row, uint64_t* bar) {
  using C = BCfg<DH>;
  if (C::NC > 1 && P.chunked) {
    tma_load_3d(dst, map, 0, row, 0, bar);
  } else {
#pragma unroll
    for (int c = 0; c < C::NC; ++c)
      tma_load_2d(dst + c * ROWS * C::ROW_BYTES, map, c * C::CW, row, bar);
  }
}

// K-major descriptor offset (16-byte units) of head-dim columns kk*16 .. kk*16+15 in a
// tile of ROWS rows.
template <int DH, int ROWS = 128>
__device__ __forceinline__ uint32_t kmajor_off(int kk) {
  using C = BCfg<DH>;
  return (((kk * 16) / C::CW) * ROWS * C::ROW_BYTES + ((kk * 16) % C::CW) * 2) >> 4;
}

// bf16 pairs of the packed row -> 16 TMEM columns at a time
__device__ __forceinline__ void store_packed32(uint32_t taddr, const uint32_t (&pk)[32]) {
#pragma unroll
  for (int c0 = 0; c0 < 32; c0 += 16) {
    uint32_t r[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) r[x] = pk[c0 + x];
    tmem_st16(taddr + c0, r);
  }
}
__device__ __forceinline__ void store_packed64(uint32_t taddr, const uint32_t (&pk)[64]) {
#pragma unroll
  for (int c0 = 0; c0 < 64; c0 += 16) {
    uint32_t r[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) r[x] = pk[c0 + x];
    tmem_st16(taddr + c0, r);
  }
}

struct Shared {
  uint64_t* q_full;   // fixed pair loaded (dq: Q, dO; dkdv: K, V)
  uint64_t* q_empty;
  uint64_t* r_full;   // [STAGES] ring pairs (dq: K, V; dkdv: Q, dO)
  uint64_t* r_empty;  // [STAGES]
  uint64_t* sdp_full;
  uint64_t* s_free;
  uint64_t* d_ready;  // dS (and P^T) written to TMEM
  uint64_t* d_free;   // their MMAs are done
  uint64_t* acc_full;
  uint64_t* acc_free;
  uint64_t* item_full;   // [2]
  uint64_t* item_empty;  // [2]
  uint64_t* l_bar;       // [2] the softmax warpgroup has filled sL / sD buffer 0 / 1
  volatile int* item_ring;
  uint32_t* tmem_holder;
  volatile int* abort_flag;
  float* sL;  // [2][128] lse of the job's queries (dkdv)
  float* sD;  // [2][128]
};

// Shared memory: two fixed tiles of fix_bytes, a ring of `stages` tile pairs of ring_bytes,
// then the barriers and the lse / D buffers.
__device__ __forceinline__ Shared carve(uint8_t* smem, int fix_bytes, int ring_bytes, int stages,
                                        uint8_t*& sFix0, uint8_t*& sFix1, uint8_t*& sR0,
                                        uint8_t*& sR1) {
  sFix0 = smem;
  sFix1 = smem + fix_bytes;
  sR0 = sFix1 + fix_bytes;              // ring: first tile of each pair
  sR1 = sR0 + stages * ring_bytes;      // ring: second tile of each pair
  uint64_t* bar = reinterpret_cast<uint64_t*>(sR1 + stages * ring_bytes);
  Shared sh;
  sh.q_full = bar;
  sh.q_empty = bar + 1;
  sh.r_full = bar + 2;
  sh.r_empty = sh.r_full + stages;
  sh.sdp_full = sh.r_empty + stages;
  sh.s_free = sh.sdp_full + 1;
  sh.d_ready = sh.s_free + 1;
  sh.d_free = sh.d_ready + 1;
  sh.acc_full = sh.d_free + 1;
  sh.acc_free = sh.acc_full + 1;
  sh.item_full = sh.acc_free + 1;
  sh.item_empty = sh.item_full + 2;
  sh.l_bar = sh.item_empty + 2;
  sh.item_ring = reinterpret_cast<volatile int*>(sh.l_bar + 2);
  sh.tmem_holder = reinterpret_cast<uint32_t*>(sh.l_bar + 3);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_holder + 1);
  sh.sL = reinterpret_cast<float*>(sh.l_bar + 4);
  sh.sD = sh.sL + 256;
  return sh;
}

__device__ __forceinline__ void init_shared(const Shared& sh, int stages) {
  mbar_init(sh.q_full, 1);
  mbar_init(sh.q_empty, 1);
  for (int s = 0; s < stages; ++s) {
    mbar_init(&sh.r_full[s], 1);
    mbar_init(&sh.r_empty[s], 1);
  }
  mbar_init(sh.sdp_full, 1);
  mbar_init(sh.s_free, 4);
  mbar_init(sh.d_ready, 4);
  mbar_init(sh.d_free, 1);
  mbar_init(sh.acc_full, 1);
  mbar_init(sh.acc_free, 4);
  for (int r = 0; r < 2; ++r) {
    mbar_init(&sh.item_full[r], 1);
    mbar_init(&sh.item_empty[r], 5);  // the MMA warp and the four softmax warps
    mbar_init(&sh.l_bar[r], 128);     // every softmax thread
  }
  *sh.abort_flag = 0;
  fence_barrier_init();
}

// Claims items for the CTA (lane 0 of warp 0) and publishes them through the two-slot ring;
// -1 ends the CTA's work.
__device__ __forceinline__ bool publish_item(const Shared& sh, const BwdParams& P, int& islot,
                                             uint32_t& iphase, int& i) {
  if (!lane_wait(&sh.item_empty[islot], iphase ^ 1, P, sh.abort_flag)) return false;
  i = atomicAdd(P.counter, 1);
  if (i >= P.items) i = -1;
  sh.item_ring[islot] = i;
  mbar_arrive(&sh.item_full[islot]);
  if (++islot == 2) {
    islot = 0;
    iphase ^= 1;
  }
  return true;
}
__device__ __forceinline__ bool next_item(const Shared& sh, const BwdParams& P, int& islot,
                                          uint32_t& iphase, int& i) {
  if (!warp_wait(&sh.item_full[islot], iphase, P, sh.abort_flag)) return false;
  i = sh.item_ring[islot];
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sh.item_empty[islot]);
  if (++islot == 2) {
    islot = 0;
    iphase ^= 1;
  }
  return true;
}

__device__ __forceinline__ void finish(const BwdParams& P, uint32_t tmem, int warp,
                                       uint32_t cols) {
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, cols);
  }
  if (threadIdx.x == 0 && atomicAdd(P.counter + 1, 1) == (int)gridDim.x - 1) {
    P.counter[0] = 0;
    P.counter[1] = 0;
  }
}

// ---------------------------------------------------------------------------------------
// dQ: item (b, s, query tile), heaviest (last) query tiles first when causal.
// ---------------------------------------------------------------------------------------
struct QItem {
  int b, s, qt, nk;
};
__device__ __forceinline__ QItem decode_q(const BwdParams& P, int i) {
  QItem it;
  const int bs = P.B * P.S;
  it.qt = P.causal ? P.nq - 1 - i / bs : i / bs;
  const int r = i % bs;
  it.s = r % P.S;
  it.b = r / P.S;
  it.nk = P.causal ? it.qt + 1 : P.nq;
  return it;
}

// The dQ kernel runs two CTAs per SM with 64-key steps, so that each CTA's TMEM (S, dP,
// dS, dQ) fits in 256 columns and two softmax warpgroups share an SM; warpgroup 0 (loads,
// MMA, two idle warps) gives most of its registers to the softmax warpgroup.
template <int DH>
struct QCfg {
  using C = BCfg<DH>;
  static constexpr int TKD = 64;                     // keys per step
  static constexpr int KT_BYTES = TKD * DH * 2;      // one 64-row K or V tile
  static constexpr int STAGES = 3;
  static constexpr int SMEM = 2 * C::TILE_BYTES + STAGES * 2 * KT_BYTES + 1024 + 512 + 2048;
  static constexpr int CTAS = C::CTAS;
  static constexpr int TMEM_COLS = C::TMEM_COLS;
  static constexpr int S_COL = 0, DP_COL = 64, DS_COL = 128, DQ_COL = 160;
  static_assert(DQ_COL + DH <= TMEM_COLS, "TMEM budget");
  static_assert(CTAS * (SMEM + 1024) <= 228 * 1024, "shared memory per SM");
};
constexpr int kQSmallRegs = 48, kQLargeRegs = 208;
static_assert(kQSmallRegs * 128 + kQLargeRegs * 128 == THREADS * (65536 / (2 * THREADS)),
              "register split must equal the launch allocation");

template <int DH>
__global__ void __launch_bounds__(THREADS, QCfg<DH>::CTAS)
attn_bwd_dq_kernel(const __grid_constant__ BwdParams P) {
  using C = BCfg<DH>;
  using Q = QCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t *sQ, *sdO, *sK, *sV;
  const Shared sh = carve(smem, C::TILE_BYTES, Q::KT_BYTES, Q::STAGES, sQ, sdO, sK, sV);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) init_shared(sh, Q::STAGES);
  if (warp == 1) {
    tmem_alloc(sh.tmem_holder, Q::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.tm_q);
    prefetch_tmap(&P.tm_k64);
    prefetch_tmap(&P.tm_v64);
    prefetch_tmap(&P.tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_holder;
  pdl_wait();
  pdl_allow_next();

  if (warp < 4) {
  if constexpr (C::CTAS == 2) setmaxnreg_dec<kQSmallRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      int st = 0, islot = 0;
      uint32_t r_phase = 0, q_phase = 0, iphase = 0;
      while (!*sh.abort_flag) {
        int i;
        if (!publish_item(sh, P, islot, iphase, i) || i < 0) break;
        const QItem it = decode_q(P, i);
        if (!lane_wait(sh.q_empty, q_phase ^ 1, P, sh.abort_flag)) break;
        q_phase ^= 1;
        mbar_arrive_expect_tx(sh.q_full, 2 * C::TILE_BYTES);
        const int qrow = it.s * P.M + it.b * P.T + it.qt * TQ;
        load_tile<DH>(P, &P.tm_q, sQ, qrow, sh.q_full);
        load_tile<DH>(P, &P.tm_do, sdO, qrow, sh.q_full);
        const int kvh = it.s < P.Sr ? it.s / P.k : 0;
        const int krow0 = kvh * P.M + it.b * P.T;
        const int nsteps = 2 * it.nk;  // 64-key steps over the item's 128-key tiles
        for (int j = 0; j < nsteps; ++j) {
          if (!lane_wait(&sh.r_empty[st], r_phase ^ 1, P, sh.abort_flag)) break;
          mbar_arrive_expect_tx(&sh.r_full[st], 2 * Q::KT_BYTES);
          load_tile<DH, Q::TKD>(P, &P.tm_k64, sK + st * Q::KT_BYTES, krow0 + j * Q::TKD,
                                &sh.r_full[st]);
          load_tile<DH, Q::TKD>(P, &P.tm_v64, sV + st * Q::KT_BYTES, krow0 + j * Q::TKD,
                                &sh.r_full[st]);
          if (++st == Q::STAGES) {
            st = 0;
            r_phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    const uint32_t idesc_s = idesc_bf16_f32(TQ, Q::TKD);
    const uint32_t idesc_dq = idesc_bf16_f32(TQ, DH) | (1u << 16);  // B (K) MN-major
    const uint64_t q_desc = smem_desc(smem_u32(sQ), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t do_desc = smem_desc(smem_u32(sdO), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t k_desc = smem_desc(smem_u32(sK), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t v_desc = smem_desc(smem_u32(sV), 8 * C::ROW_BYTES, C::LAYOUT);
    // K as the MN-major B operand of dQ: 64-row chunks
    const uint64_t kmn_desc =
        smem_desc_mn(smem_u32(sK), Q::TKD * C::ROW_BYTES, 8 * C::ROW_BYTES, C::LAYOUT);
    constexpr uint32_t kStep = Q::KT_BYTES >> 4;
    int st = 0, islot = 0;
    uint32_t r_phase = 0, q_phase = 0, iphase = 0;
    uint32_t n_sf = 0, n_dr = 0, n_items = 0;
    bool ok = true;
    // S = Q K^T and dP = dO V^T of the next 64-key tile
    auto issue_sdp = [&](int stage, uint32_t phase) -> bool {
      if (!warp_wait(&sh.r_full[stage], phase, P, sh.abort_flag)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t kd = k_desc + (uint64_t)(stage * kStep);
        const uint64_t vd = v_desc + (uint64_t)(stage * kStep);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          mma_ss(tmem + Q::S_COL, q_desc + kmajor_off<DH>(kk), kd + kmajor_off<DH, Q::TKD>(kk),
                 idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          mma_ss(tmem + Q::DP_COL, do_desc + kmajor_off<DH>(kk), vd + kmajor_off<DH, Q::TKD>(kk),
                 idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(sh.sdp_full);
      }
      __syncwarp();
      return true;
    };
    while (ok && !*sh.abort_flag) {
      int i;
      if (!next_item(sh, P, islot, iphase, i) || i < 0) break;
      const QItem it = decode_q(P, i);
      if (!warp_wait(sh.q_full, q_phase, P, sh.abort_flag)) break;
      q_phase ^= 1;
      int st_next = st;
      uint32_t ph_next = r_phase;
      const int nsteps = 2 * it.nk;
      if (!issue_sdp(st_next, ph_next)) break;
      for (int j = 0; j < nsteps; ++j) {
        const int st_j = st_next;
        if (++st_next == Q::STAGES) {
          st_next = 0;
          ph_next ^= 1;
        }
        if (j + 1 < nsteps) {
          // the softmax warps hold S(j), dP(j) in registers: the next pair may be written
          if (!warp_wait(sh.s_free, n_sf & 1, P, sh.abort_flag)) { ok = false; break; }
          ++n_sf;
          if (!issue_sdp(st_next, ph_next)) { ok = false; break; }
        }
        if (!warp_wait(sh.d_ready, n_dr & 1, P, sh.abort_flag)) { ok = false; break; }
        ++n_dr;
        if (j == 0 && n_items > 0 &&
            !warp_wait(sh.acc_free, (n_items - 1) & 1, P, sh.abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          // dQ (+)= dS K: A = dS (queries x 64 keys, TMEM), B = the K tile (N = head dim,
          // K = keys; MN-major)
          const uint64_t kd = kmn_desc + (uint64_t)(st_j * kStep);
#pragma unroll
          for (int kk = 0; kk < Q::TKD / 16; ++kk)
            mma_ts(tmem + Q::DQ_COL, tmem + Q::DS_COL + kk * 8,
                   kd + (uint64_t)((kk * 16 * C::ROW_BYTES) >> 4), idesc_dq,
                   (j == 0 && kk == 0) ? 0u : 1u);
          mma_commit(&sh.r_empty[st_j]);
          mma_commit(sh.d_free);
          if (j + 1 == nsteps) {
            mma_commit(sh.acc_full);
            mma_commit(sh.q_empty);
          }
        }
        __syncwarp();
      }
      st = st_next;
      r_phase = ph_next;
      ++n_items;
    }
  }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    if constexpr (C::CTAS == 2) setmaxnreg_inc<kQLargeRegs>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_base = tmem + lane_off;
    uint32_t n_sdp = 0, n_ds = 0, n_acc = 0;
    int islot = 0;
    uint32_t iphase = 0;
    const float c2 = P.scale_log2;
    while (!*sh.abort_flag) {
      int i;
      if (!next_item(sh, P, islot, iphase, i) || i < 0) break;
      const QItem it = decode_q(P, i);
      const int q0 = it.qt * TQ;
      const int q = q0 + row;
      const bool valid = q < P.T;
      const int64_t tok = (int64_t)it.b * P.T + q;
      const float lse = valid ? P.lse[(int64_t)it.s * P.M + tok] : 0.f;
      const float dsum = valid ? P.dsum[(int64_t)it.s * P.M + tok] : 0.f;
      const int lim = !valid ? 0 : (P.causal ? q + 1 : P.T);  // keys < lim are live
      const int nsteps = 2 * it.nk;
      bool ok = true;
      for (int j = 0; j < nsteps; ++j) {
        if (!warp_wait(sh.sdp_full, n_sdp & 1, P, sh.abort_flag)) { ok = false; break; }
        ++n_sdp;
        tc_fence_after();
        const int kv0 = j * Q::TKD;
        uint32_t pk[32];
        {
          uint32_t sr[64], dr[64];
          tmem_ld64_wait(t_base + Q::S_COL, sr);
          tmem_ld64_wait(t_base + Q::DP_COL, dr);
          if (j + 1 < nsteps) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sh.s_free);
          }
          if (kv0 + Q::TKD <= lim) {
            // every key of the tile is live for this query: no masks
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * x]), c2, -lse));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * x + 1]), c2, -lse));
              pk[x] = pack_bf16x2(p0 * (__uint_as_float(dr[2 * x]) - dsum),
                                  p1 * (__uint_as_float(dr[2 * x + 1]) - dsum));
            }
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const int c = 2 * x;
              float d0 = 0.f, d1 = 0.f;
              if (kv0 + c < lim) {
                const float p = fast_exp2(fmaf(__uint_as_float(sr[2 * x]), c2, -lse));
                d0 = p * (__uint_as_float(dr[2 * x]) - dsum);
              }
              if (kv0 + c + 1 < lim) {
                const float p = fast_exp2(fmaf(__uint_as_float(sr[2 * x + 1]), c2, -lse));
                d1 = p * (__uint_as_float(dr[2 * x + 1]) - dsum);
              }
              pk[x] = pack_bf16x2(d0, d1);
            }
          }
        }
        // the previous dQ product has read dS: it may be overwritten
        if (n_ds > 0 && !warp_wait(sh.d_free, (n_ds - 1) & 1, P, sh.abort_flag)) {
          ok = false;
          break;
        }
        ++n_ds;
        store_packed32(t_base + Q::DS_COL, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.d_ready);
      }
      if (!ok) break;
      // epilogue: dQ / sqrt(d_h) into its destination row
      if (!warp_wait(sh.acc_full, n_acc & 1, P, sh.abort_flag)) break;
      ++n_acc;
      tc_fence_after();
      __nv_bfloat16* dst = nullptr;
      if (valid) {
        if (it.s < P.Sr) {
          const int g = it.s / P.k;
          const int e = g * P.E + P.sel[tok * (int64_t)P.sel_stride + P.sel_off + it.s];
          dst = P.dq_exp + tok * (int64_t)P.N * DH + (int64_t)e * DH;
        } else {
          dst = P.dq_sh + tok * DH;
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 16) {
        uint32_t r[16];
        tmem_ld16_wait(t_base + Q::DQ_COL + c0, r);
        if (valid) {
          uint4 v0, v1;
          const float sc = P.scale;
          v0.x = pack_bf16x2(__uint_as_float(r[0]) * sc, __uint_as_float(r[1]) * sc);
          v0.y = pack_bf16x2(__uint_as_float(r[2]) * sc, __uint_as_float(r[3]) * sc);
          v0.z = pack_bf16x2(__uint_as_float(r[4]) * sc, __uint_as_float(r[5]) * sc);
          v0.w = pack_bf16x2(__uint_as_float(r[6]) * sc, __uint_as_float(r[7]) * sc);
          v1.x = pack_bf16x2(__uint_as_float(r[8]) * sc, __uint_as_float(r[9]) * sc);
          v1.y = pack_bf16x2(__uint_as_float(r[10]) * sc, __uint_as_float(r[11]) * sc);
          v1.z = pack_bf16x2(__uint_as_float(r[12]) * sc, __uint_as_float(r[13]) * sc);
          v1.w = pack_bf16x2(__uint_as_float(r[14]) * sc, __uint_as_float(r[15]) * sc);
          *reinterpret_cast<uint4*>(dst + c0) = v0;
          *reinterpret_cast<uint4*>(dst + c0 + 8) = v1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sh.acc_free);
    }
  }
  finish(P, tmem, warp, QCfg<DH>::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------
// dK, dV: item (b, KV head g, key tile), first key tiles first when causal (they meet the
// most query tiles). Jobs of an item: every (stream reading g, query tile at or after the
// key tile when causal).
// ---------------------------------------------------------------------------------------
// TMEM -> registers, N consecutive 32-bit columns per lane (N = 32, 48 or 64), and the wait
// for them in the same statement.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld48_wait(uint32_t taddr, uint32_t (&r)[48]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%48];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47}, [%49];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
        "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
        "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47])
      : "r"(taddr), "r"(taddr + 32u)
      : "memory");
}
template <int N>
__device__ __forceinline__ void tmem_ldN_wait(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N == 32 || N == 48 || N == 64, "TMEM row widths of a job");
  if constexpr (N == 32) tmem_ld32_wait(taddr, r);
  else if constexpr (N == 48) tmem_ld48_wait(taddr, r);
  else tmem_ld64_wait(taddr, r);
}
// bf16 pairs of a packed row -> TMEM, 8 columns per store
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// The dK / dV kernel runs jobs of TQJ queries small enough that S^T, dP^T, P^T, dS^T, dV
// and dK all have TMEM columns of their own: at two CTAs per SM (256 columns) 48 queries for
// head dims up to 48 and 32 for 64; at one CTA per SM (512 columns, head dims above 64) 64.
// The next job's S^T and dP^T are issued as soon as the softmax warps hold the current
// ones in registers, as in the dQ kernel.
template <int DH>
struct KCfg {
  using C = BCfg<DH>;
  static constexpr int TQJ = DH <= 48 ? 48 : (DH <= 64 ? 32 : 64);  // queries per job
  static constexpr int QT_BYTES = TQJ * DH * 2;     // one Q or dO tile of the job
  static constexpr int STAGES = 3;
  static constexpr int WARP_STAGE = 4 * 2 * 2 * TQJ * 4;  // per-warp lse / D buffers
  static constexpr int SMEM =
      2 * C::TILE_BYTES + STAGES * 2 * QT_BYTES + 1024 + 512 + 2048 + WARP_STAGE;
  static constexpr int CTAS = C::CTAS;
  static constexpr int TMEM_COLS = C::TMEM_COLS;
  static constexpr int S_COL = 0, DP_COL = TQJ, P_COL = 2 * TQJ, DS_COL = 2 * TQJ + TQJ / 2;
  static constexpr int DV_COL = 3 * TQJ, DK_COL = 3 * TQJ + DH;
  static_assert(TQJ % 16 == 0 && TQJ <= 64, "a job's queries: two per lane at most");
  static_assert(DK_COL + DH <= TMEM_COLS, "TMEM budget");
  static_assert(DP_COL % 16 == 0 && DV_COL % 16 == 0 && DK_COL % 16 == 0, "accumulator columns");
  static_assert(CTAS * (SMEM + 1024) <= 228 * 1024, "shared memory per SM");
};

struct KItem {
  int b, g, kt, ns, qt0, nj;
};
// Jobs of an item: (stream si of the head, query tile qt0 + r of TQJ queries) for si < ns,
// r < per; the first tile is the first one reaching a query at or after the key tile.
template <int TQJ>
__device__ __forceinline__ KItem decode_k(const BwdParams& P, int i) {
  KItem it;
  const int bg = P.B * P.G;
  it.kt = i / bg;
  const int r = i % bg;
  it.g = r % P.G;
  it.b = r / P.G;
  it.ns = P.k + ((it.g == 0 && P.has_shared) ? 1 : 0);
  const int nqj = (P.T + TQJ - 1) / TQJ;
  it.qt0 = P.causal ? (it.kt * TK) / TQJ : 0;
  it.nj = it.ns * (nqj - it.qt0);
  return it;
}
template <int TQJ>
__device__ __forceinline__ void job_of(const BwdParams& P, const KItem& it, int j, int& s,
                                       int& qt) {
  const int per = (P.T + TQJ - 1) / TQJ - it.qt0;
  const int si = j / per;
  qt = it.qt0 + j % per;
  s = si < P.k ? it.g * P.k + si : P.Sr;
}

template <int DH>
__global__ void __launch_bounds__(THREADS, KCfg<DH>::CTAS)
attn_bwd_dkdv_kernel(const __grid_constant__ BwdParams P) {
  using C = BCfg<DH>;
  using K = KCfg<DH>;
  constexpr int TQJ = K::TQJ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t *sK, *sV, *sQ, *sdO;
  const Shared sh = carve(smem, C::TILE_BYTES, K::QT_BYTES, K::STAGES, sK, sV, sQ, sdO);
  // per-warp lse / D buffers after the shared lse / D area (unused here)
  float* wstage = sh.sD + 256;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) init_shared(sh, K::STAGES);
  if (warp == 1) {
    tmem_alloc(sh.tmem_holder, K::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.tm_qj);
    prefetch_tmap(&P.tm_k);
    prefetch_tmap(&P.tm_v);
    prefetch_tmap(&P.tm_doj);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_holder;
  pdl_wait();
  pdl_allow_next();

  if (warp < 4) {
  if constexpr (C::CTAS == 2) setmaxnreg_dec<kQSmallRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      int st = 0, islot = 0;
      uint32_t r_phase = 0, q_phase = 0, iphase = 0;
      while (!*sh.abort_flag) {
        int i;
        if (!publish_item(sh, P, islot, iphase, i) || i < 0) break;
        const KItem it = decode_k<TQJ>(P, i);
        if (!lane_wait(sh.q_empty, q_phase ^ 1, P, sh.abort_flag)) break;
        q_phase ^= 1;
        mbar_arrive_expect_tx(sh.q_full, 2 * C::TILE_BYTES);
        const int krow = it.g * P.M + it.b * P.T + it.kt * TK;
        load_tile<DH>(P, &P.tm_k, sK, krow, sh.q_full);
        load_tile<DH>(P, &P.tm_v, sV, krow, sh.q_full);
        for (int j = 0; j < it.nj; ++j) {
          int s, qt;
          job_of<TQJ>(P, it, j, s, qt);
          if (!lane_wait(&sh.r_empty[st], r_phase ^ 1, P, sh.abort_flag)) break;
          mbar_arrive_expect_tx(&sh.r_full[st], 2 * K::QT_BYTES);
          const int qrow = s * P.M + it.b * P.T + qt * TQJ;
          load_tile<DH, TQJ>(P, &P.tm_qj, sQ + st * K::QT_BYTES, qrow, &sh.r_full[st]);
          load_tile<DH, TQJ>(P, &P.tm_doj, sdO + st * K::QT_BYTES, qrow, &sh.r_full[st]);
          if (++st == K::STAGES) {
            st = 0;
            r_phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issue
    const uint32_t idesc_s = idesc_bf16_f32(TK, TQJ);
    const uint32_t idesc_kv = idesc_bf16_f32(TK, DH) | (1u << 16);  // B (Q, dO) MN-major
    const uint64_t k_desc = smem_desc(smem_u32(sK), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t v_desc = smem_desc(smem_u32(sV), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t q_desc = smem_desc(smem_u32(sQ), 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t do_desc = smem_desc(smem_u32(sdO), 8 * C::ROW_BYTES, C::LAYOUT);
    // Q and dO as MN-major B operands: TQJ-row chunks
    const uint64_t qmn_desc =
        smem_desc_mn(smem_u32(sQ), TQJ * C::ROW_BYTES, 8 * C::ROW_BYTES, C::LAYOUT);
    const uint64_t domn_desc =
        smem_desc_mn(smem_u32(sdO), TQJ * C::ROW_BYTES, 8 * C::ROW_BYTES, C::LAYOUT);
    constexpr uint32_t kStep = K::QT_BYTES >> 4;
    int st = 0, islot = 0;
    uint32_t r_phase = 0, q_phase = 0, iphase = 0;
    uint32_t n_sf = 0, n_dr = 0, n_items = 0;
    bool ok = true;
    // S^T = K Q^T and dP^T = V dO^T of the next job
    auto issue_sdp = [&](int stage, uint32_t phase) -> bool {
      if (!warp_wait(&sh.r_full[stage], phase, P, sh.abort_flag)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t qd = q_desc + (uint64_t)(stage * kStep);
        const uint64_t dd = do_desc + (uint64_t)(stage * kStep);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          mma_ss(tmem + K::S_COL, k_desc + kmajor_off<DH>(kk), qd + kmajor_off<DH, TQJ>(kk),
                 idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          mma_ss(tmem + K::DP_COL, v_desc + kmajor_off<DH>(kk), dd + kmajor_off<DH, TQJ>(kk),
                 idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(sh.sdp_full);
      }
      __syncwarp();
      return true;
    };
    while (ok && !*sh.abort_flag) {
      int i;
      if (!next_item(sh, P, islot, iphase, i) || i < 0) break;
      const KItem it = decode_k<TQJ>(P, i);
      if (!warp_wait(sh.q_full, q_phase, P, sh.abort_flag)) break;
      q_phase ^= 1;
      int st_next = st;
      uint32_t ph_next = r_phase;
      if (!issue_sdp(st_next, ph_next)) break;
      for (int j = 0; j < it.nj; ++j) {
        const int st_j = st_next;
        if (++st_next == K::STAGES) {
          st_next = 0;
          ph_next ^= 1;
        }
        if (j + 1 < it.nj) {
          // the softmax warps hold S^T(j), dP^T(j) in registers: the next pair may be written
          if (!warp_wait(sh.s_free, n_sf & 1, P, sh.abort_flag)) { ok = false; break; }
          ++n_sf;
          if (!issue_sdp(st_next, ph_next)) { ok = false; break; }
        }
        if (!warp_wait(sh.d_ready, n_dr & 1, P, sh.abort_flag)) { ok = false; break; }
        ++n_dr;
        if (j == 0 && n_items > 0 &&
            !warp_wait(sh.acc_free, (n_items - 1) & 1, P, sh.abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint64_t dmn = domn_desc + (uint64_t)(st_j * kStep);
          const uint64_t qmn = qmn_desc + (uint64_t)(st_j * kStep);
          // dV (+)= P^T dO and dK (+)= dS^T Q: A from TMEM (keys x TQJ queries), B = the
          // dO / Q tile (N = head dim, K = queries; MN-major)
#pragma unroll
          for (int kk = 0; kk < TQJ / 16; ++kk)
            mma_ts(tmem + K::DV_COL, tmem + K::P_COL + kk * 8,
                   dmn + (uint64_t)((kk * 16 * C::ROW_BYTES) >> 4), idesc_kv,
                   (j == 0 && kk == 0) ? 0u : 1u);
#pragma unroll
          for (int kk = 0; kk < TQJ / 16; ++kk)
            mma_ts(tmem + K::DK_COL, tmem + K::DS_COL + kk * 8,
                   qmn + (uint64_t)((kk * 16 * C::ROW_BYTES) >> 4), idesc_kv,
                   (j == 0 && kk == 0) ? 0u : 1u);
          mma_commit(&sh.r_empty[st_j]);
          mma_commit(sh.d_free);
          if (j + 1 == it.nj) {
            mma_commit(sh.acc_full);
            mma_commit(sh.q_empty);
          }
        }
        __syncwarp();
      }
      st = st_next;
      r_phase = ph_next;
      ++n_items;
    }
  }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    if constexpr (C::CTAS == 2) setmaxnreg_inc<kQLargeRegs>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row of the tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_base = tmem + lane_off;
    // this warp's lse / D buffers: [2][TQJ] each
    float* wL = wstage + quarter * (2 * 2 * TQJ);
    float* wD = wL + 2 * TQJ;
    uint32_t n_sdp = 0, n_pd = 0, n_acc = 0, n_job = 0;
    int islot = 0;
    uint32_t iphase = 0;
    const float c2 = P.scale_log2;
    while (!*sh.abort_flag) {
      int i;
      if (!next_item(sh, P, islot, iphase, i) || i < 0) break;
      const KItem it = decode_k<TQJ>(P, i);
      const int u = it.kt * TK + row;  // key position
      const bool key_ok = u < P.T;
      bool ok = true;
      // a job's lse and D: lane l loads queries l and l + 32 (< TQJ), one job ahead
      auto fetch = [&](int jj, float (&lv)[2], float (&dv)[2]) {
        int ss, qq_t;
        job_of<TQJ>(P, it, jj, ss, qq_t);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = lane + 32 * h;
          const int qq = qq_t * TQJ + c;
          const bool in = c < TQJ && qq < P.T;
          const int64_t idx = (int64_t)ss * P.M + (int64_t)it.b * P.T + qq;
          lv[h] = in ? P.lse[idx] : 0.f;
          dv[h] = in ? P.dsum[idx] : 0.f;
        }
      };
      float nl[2], nd[2];
      fetch(0, nl, nd);
      for (int j = 0; j < it.nj; ++j, ++n_job) {
        int s, qt;
        job_of<TQJ>(P, it, j, s, qt);
        float* sL = wL + (n_job & 1) * TQJ;
        float* sD = wD + (n_job & 1) * TQJ;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = lane + 32 * h;
          if (c < TQJ) {
            sL[c] = nl[h];
            sD[c] = nd[h];
          }
        }
        __syncwarp();  // this warp's buffer is complete (the other buffer is two jobs old)
        if (j + 1 < it.nj) fetch(j + 1, nl, nd);
        if (!warp_wait(sh.sdp_full, n_sdp & 1, P, sh.abort_flag)) { ok = false; break; }
        ++n_sdp;
        tc_fence_after();
        const int q0 = qt * TQJ;
        // live queries of this key: q < T, and q >= u when causal
        const int qlo = P.causal ? u : 0;
        const bool all_live = key_ok && q0 >= qlo && q0 + TQJ <= P.T;
        uint32_t pp[TQJ / 2], pd[TQJ / 2];
        {
          uint32_t sr[TQJ], dr[TQJ];
          tmem_ldN_wait<TQJ>(t_base + K::S_COL, sr);
          tmem_ldN_wait<TQJ>(t_base + K::DP_COL, dr);
          if (j + 1 < it.nj) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sh.s_free);
          }
          if (all_live) {
#pragma unroll
            for (int x4 = 0; x4 < TQJ / 4; ++x4) {
              const float4 L4 = reinterpret_cast<const float4*>(sL)[x4];
              const float4 D4 = reinterpret_cast<const float4*>(sD)[x4];
              const float p0 = fast_exp2(fmaf(__uint_as_float(sr[4 * x4]), c2, -L4.x));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sr[4 * x4 + 1]), c2, -L4.y));
              const float p2 = fast_exp2(fmaf(__uint_as_float(sr[4 * x4 + 2]), c2, -L4.z));
              const float p3 = fast_exp2(fmaf(__uint_as_float(sr[4 * x4 + 3]), c2, -L4.w));
              pp[2 * x4] = pack_bf16x2(p0, p1);
              pp[2 * x4 + 1] = pack_bf16x2(p2, p3);
              pd[2 * x4] = pack_bf16x2(p0 * (__uint_as_float(dr[4 * x4]) - D4.x),
                                       p1 * (__uint_as_float(dr[4 * x4 + 1]) - D4.y));
              pd[2 * x4 + 1] = pack_bf16x2(p2 * (__uint_as_float(dr[4 * x4 + 2]) - D4.z),
                                           p3 * (__uint_as_float(dr[4 * x4 + 3]) - D4.w));
            }
          } else {
#pragma unroll
            for (int x = 0; x < TQJ / 2; ++x) {
              const int c = 2 * x;
              float p0 = 0.f, p1 = 0.f, d0 = 0.f, d1 = 0.f;
              const int qa = q0 + c, qb = q0 + c + 1;
              if (key_ok && qa < P.T && qa >= qlo) {
                p0 = fast_exp2(fmaf(__uint_as_float(sr[2 * x]), c2, -sL[c]));
                d0 = p0 * (__uint_as_float(dr[2 * x]) - sD[c]);
              }
              if (key_ok && qb < P.T && qb >= qlo) {
                p1 = fast_exp2(fmaf(__uint_as_float(sr[2 * x + 1]), c2, -sL[c + 1]));
                d1 = p1 * (__uint_as_float(dr[2 * x + 1]) - sD[c + 1]);
              }
              pp[x] = pack_bf16x2(p0, p1);
              pd[x] = pack_bf16x2(d0, d1);
            }
          }
        }
        // the previous job's products have read P^T and dS^T: they may be overwritten
        if (n_pd > 0 && !warp_wait(sh.d_free, (n_pd - 1) & 1, P, sh.abort_flag)) {
          ok = false;
          break;
        }
        ++n_pd;
#pragma unroll
        for (int c0 = 0; c0 < TQJ / 2; c0 += 8) {
          tmem_st8(t_base + K::P_COL + c0, pp + c0);
          tmem_st8(t_base + K::DS_COL + c0, pd + c0);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.d_ready);
      }
      if (!ok) break;
      // epilogue: dK / sqrt(d_h) and dV into their token-major rows
      if (!warp_wait(sh.acc_full, n_acc & 1, P, sh.abort_flag)) break;
      ++n_acc;
      tc_fence_after();
      const int64_t tok = (int64_t)it.b * P.T + u;
      const int64_t off = tok * (int64_t)P.G * DH + (int64_t)it.g * DH;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst = (which == 0 ? P.dk : P.dv) + off;
        const float sc = which == 0 ? P.scale : 1.f;
        const uint32_t col = which == 0 ? K::DK_COL : K::DV_COL;
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 16) {
          uint32_t r[16];
          tmem_ld16_wait(t_base + col + c0, r);
          if (key_ok) {
            uint4 v0, v1;
            v0.x = pack_bf16x2(__uint_as_float(r[0]) * sc, __uint_as_float(r[1]) * sc);
            v0.y = pack_bf16x2(__uint_as_float(r[2]) * sc, __uint_as_float(r[3]) * sc);
            v0.z = pack_bf16x2(__uint_as_float(r[4]) * sc, __uint_as_float(r[5]) * sc);
            v0.w = pack_bf16x2(__uint_as_float(r[6]) * sc, __uint_as_float(r[7]) * sc);
            v1.x = pack_bf16x2(__uint_as_float(r[8]) * sc, __uint_as_float(r[9]) * sc);
            v1.y = pack_bf16x2(__uint_as_float(r[10]) * sc, __uint_as_float(r[11]) * sc);
            v1.z = pack_bf16x2(__uint_as_float(r[12]) * sc, __uint_as_float(r[13]) * sc);
            v1.w = pack_bf16x2(__uint_as_float(r[14]) * sc, __uint_as_float(r[15]) * sc);
            *reinterpret_cast<uint4*>(dst + c0) = v0;
            *reinterpret_cast<uint4*>(dst + c0 + 8) = v1;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sh.acc_free);
    }
  }
  finish(P, tmem, warp, KCfg<DH>::TMEM_COLS);
}

template <int DH>
int launch_bwd_dh(gqe_ctx* h, const BwdBuffers& bb, int B, int T, int S, int has_shared,
                  int causal, cudaStream_t st) {
  using C = BCfg<DH>;
  if (!set_smem_limit_once<attn_bwd_dq_kernel<DH>>(QCfg<DH>::SMEM)) return -1;
  if (!set_smem_limit_once<attn_bwd_dkdv_kernel<DH>>(KCfg<DH>::SMEM)) return -1;
  const int M = B * T;
  const int Gl = h->g1 - h->g0;  // this handle's KV heads
  const uint64_t kv_rows = (uint64_t)Gl * M;
  BwdParams P;
  memset(&P, 0, sizeof(P));
  const CUtensorMapSwizzle sw = C::CW == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B;
  P.chunked = C::NC > 1 &&
              tmap_bf16_chunked(&P.tm_q, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW, 128, sw) &&
              tmap_bf16_chunked(&P.tm_do, bb.dO, DH, (uint64_t)S * M, DH, C::CW, 128, sw) &&
              tmap_bf16_chunked(&P.tm_k, h->ws.K, DH, kv_rows, DH, C::CW, 128, sw) &&
              tmap_bf16_chunked(&P.tm_v, h->ws.V, DH, kv_rows, DH, C::CW, 128, sw) &&
              tmap_bf16_chunked(&P.tm_k64, h->ws.K, DH, kv_rows, DH, C::CW, 64, sw) &&
              tmap_bf16_chunked(&P.tm_v64, h->ws.V, DH, kv_rows, DH, C::CW, 64, sw) &&
              tmap_bf16_chunked(&P.tm_qj, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW,
                                KCfg<DH>::TQJ, sw) &&
              tmap_bf16_chunked(&P.tm_doj, bb.dO, DH, (uint64_t)S * M, DH, C::CW,
                                KCfg<DH>::TQJ, sw);
  if (!P.chunked &&
      (!tmap_bf16_2d_ext(&P.tm_q, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW, 128, sw) ||
       !tmap_bf16_2d_ext(&P.tm_do, bb.dO, DH, (uint64_t)S * M, DH, C::CW, 128, sw) ||
       !tmap_bf16_2d_ext(&P.tm_k, h->ws.K, DH, kv_rows, DH, C::CW, 128, sw) ||
       !tmap_bf16_2d_ext(&P.tm_v, h->ws.V, DH, kv_rows, DH, C::CW, 128, sw) ||
       !tmap_bf16_2d_ext(&P.tm_k64, h->ws.K, DH, kv_rows, DH, C::CW, 64, sw) ||
       !tmap_bf16_2d_ext(&P.tm_v64, h->ws.V, DH, kv_rows, DH, C::CW, 64, sw) ||
       !tmap_bf16_2d_ext(&P.tm_qj, h->ws.Q, DH, (uint64_t)S * M, DH, C::CW, KCfg<DH>::TQJ,
                         sw) ||
       !tmap_bf16_2d_ext(&P.tm_doj, bb.dO, DH, (uint64_t)S * M, DH, C::CW, KCfg<DH>::TQJ,
                         sw)))
    return -1;
  P.lse = h->ws.lse;
  P.dsum = bb.dsum;
  P.sel = h->ws.sel;
  P.dq_exp = bb.dq_exp;
  P.dq_sh = bb.dq_sh;
  P.dk = bb.dk;
  P.dv = bb.dv;
  P.M = M;
  P.T = T;
  P.B = B;
  P.S = S;
  P.Sr = Gl * h->k;
  P.k = h->k;
  P.G = Gl;
  P.E = h->E;
  P.N = Gl * h->E;
  P.sel_stride = h->G * h->k;
  P.sel_off = h->g0 * h->k;
  P.has_shared = has_shared;
  P.causal = causal;
  P.nq = (T + TQ - 1) / TQ;
  P.scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
  P.scale = 1.f / sqrtf((float)DH);
  P.status = h->ws.status;
  P.spin = h->spin_limit > 0 ? h->spin_limit : (int64_t)1 << 22;
  P.counter = bb.counter;
  // dQ
  P.items = B * S * P.nq;
  const int per_sm = C::CTAS * h->num_sms;  // persistent CTAs
  int grid = P.items < per_sm ? P.items : per_sm;
  if (launch_pdl(attn_bwd_dq_kernel<DH>, dim3(grid), dim3(THREADS), QCfg<DH>::SMEM, st, P) !=
      cudaSuccess)
    return -1;
  // dK, dV
  P.items = B * Gl * P.nq;
  P.counter = bb.counter + 2;
  grid = P.items < per_sm ? P.items : per_sm;
  if (launch_pdl(attn_bwd_dkdv_kernel<DH>, dim3(grid), dim3(THREADS), KCfg<DH>::SMEM, st, P) !=
      cudaSuccess)
    return -1;
  return 2;
}

}  // namespace

bool tc_backward_supported(const gqe_ctx* h) {
  return h->dtype == GQE_BF16 && h->d_h <= 128;
}

int launch_tc_attention_backward(gqe_ctx* h, const BwdBuffers& bb, int B, int T, int S,
                                 int has_shared, int causal, cudaStream_t st) {
  switch (h->d_h) {
    case 16: return launch_bwd_dh<16>(h, bb, B, T, S, has_shared, causal, st);
    case 32: return launch_bwd_dh<32>(h, bb, B, T, S, has_shared, causal, st);
    case 48: return launch_bwd_dh<48>(h, bb, B, T, S, has_shared, causal, st);
    case 64: return launch_bwd_dh<64>(h, bb, B, T, S, has_shared, causal, st);
    case 80: return launch_bwd_dh<80>(h, bb, B, T, S, has_shared, causal, st);
    case 96: return launch_bwd_dh<96>(h, bb, B, T, S, has_shared, causal, st);
    case 112: return launch_bwd_dh<112>(h, bb, B, T, S, has_shared, causal, st);
    case 128: return launch_bwd_dh<128>(h, bb, B, T, S, has_shared, causal, st);
    default: return -1;
  }
}

}  // namespace gqe
