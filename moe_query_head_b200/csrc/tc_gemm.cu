// Tensor-core (tcgen05) GEMMs of the GQE forward pass, bf16 in, fp32 accumulation in TMEM:
//
//   dense projection  x [M, dim] times W_r, W_k, W_v, W_shared ([out, dim] each): router
//                     logits (fp32), K and V [G, M, d_h], and the
//                     shared head's queries. KV heads are dense and routing-independent
//                     ("GQE: Grouped Query Experts" README, Algorithm Overview).
//   routed Q          for each expert e, the rows of x in e's bucket times W_q[e]; row i
//                     lands in query stream g*k + r at its token position, so only the
//                     selected (token, expert) pairs are projected (README, Algorithm
//                     Overview: only the active query-head computation is reduced).
//   output projection Z [M, D_o] times W_o [dim, D_o].
// A handle restricted to a group range (gqe_set_group_range) projects only its heads' K / V
// and its experts' buckets (still routing every group in the dense projection).
//
// One persistent kernel, two CTAs per SM (each CTA's pipeline hand-offs, fills and tail are
// covered by the other CTA's work); grids of at most one CTA per SM (small M) run one CTA per
// SM with a ring twice as deep:
//   producers  dense: one warp issuing TMA tile loads of A and B. Routed projection: three
//              warps gathering A rows through registers into the 128-byte swizzled
//              layout (each warp fills every third stage), B by TMA;
//   MMA warp   allocates TMEM; one lane issues tcgen05.mma (128 x BN x 16) and commits;
//   4 warps    epilogue: tcgen05.ld of the fp32 accumulator, conversion, stores.
// Shared-memory stages are guarded by full/empty mbarriers; two TMEM accumulators let the
// epilogue of one tile overlap the MMAs of the next.
#include <cudaTypedefs.h>

#include <mutex>

#include "gqe_common.cuh"
#include "tc_ptx.cuh"

namespace gqe {

namespace {

using namespace tc;

constexpr int BM = 128;        // tile rows = MMA M = TMEM lanes
constexpr int BN = 128;        // widest tile (MMA N)
constexpr int BK = 64;         // one 128-byte swizzle atom of bf16 along K
constexpr int CTAS_PER_SM = 2;  // shared memory: 2 x ~98 KB; TMEM: 2 x 256 columns
// Warp roles: producers, one MMA-issuing warp, four epilogue warps.
template <bool GATHER>
struct Lay {
  static constexpr int NPROD = GATHER ? 3 : 1;
  static constexpr int MMA = NPROD;
  static constexpr int EPI0 = NPROD + 1;
  static constexpr int THREADS = (NPROD + 5) * 32;
};
// Shared-memory ring: B stages hold up to BN rows, or 64 for the routed projection of a head
// dimension up to 64 (NARROW), whose smaller stages buy a fourth stage in the same space:
// these GEMMs are bound by load latency times the bytes in flight. DEEP: one CTA per SM
// with twice the stages, for grids no larger than the SM count (the small-M GEMMs of a
// decode step), whose few CTAs each walk all of K: fewer round trips over K.
template <bool NARROW, bool DEEP = false>
struct Ring {
  static constexpr int STAGES = (NARROW ? 4 : 3) * (DEEP ? 2 : 1);
  static constexpr int B_ROWS = NARROW ? 64 : BN;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  // stages, 1024-byte alignment, barriers and flags, the routed schedule's scratch
  static constexpr int SMEM =
      STAGES * (A_BYTES + B_BYTES) + 1024 + 256 + 16 * (kMaxExperts + 8) + 4 * kMaxExperts;
};
// Scratch after the barriers (routed schedule): s_cnt [kMaxExperts] and s_t0
// [kMaxExperts + 1] ints, then CTA 0's probability sums, doubles, at kPsOffset.
constexpr int kPsOffset = 528;
static_assert(kPsOffset >= 4 * (2 * kMaxExperts + 1) && kPsOffset % 8 == 0,
              "the probability sums follow the schedule arrays, 8-byte aligned");
template <int STAGES>
constexpr bool scratch_fits() {
  // barriers (full, empty per stage; two accumulators' full and empty), the TMEM holder and
  // abort flag (16 bytes), then the scratch, within the space SMEM reserves after the stages
  return (2 * STAGES + 4) * 8 + 16 + kPsOffset + 8 * kMaxExperts <=
         256 + 16 * (kMaxExperts + 8) + 4 * kMaxExperts;
}
static_assert(scratch_fits<Ring<true, true>::STAGES>() && scratch_fits<Ring<false, true>::STAGES>(),
              "the routed schedule's scratch fits the deepest ring's shared memory");
constexpr int TMEM_COLS = 2 * BN;
constexpr int MAX_PROBLEMS = 4;
constexpr int MAX_COL_TILES = 32;  // column tiles over all problems of one GEMM

struct Problem {
  int N;        // output columns of this problem
  int n_tiles;  // ceil(N / BN)
  int box_n;    // rows of B per TMA box (<= BN, multiple of 16)
  OutMap out;
};

// Outputs of the routing done in the dense projection's router tiles (see route_rows). The
// cursors and probability sums come in two sets used by alternate calls, chosen on the
// device by a flag that the routed projection's last CTA flips when it is done with its set
// (so a captured graph alternates as its calls would): this call's set is zero when it
// starts (the previous call's dense projection cleared it), and this call clears the other
// one, whose last reader (the previous call's routed projection) is done.
struct RouteOut {
  float* logits_out;     // [M, N] problem 0's output (router logits, fp32)
  int32_t* sel;          // [M, G, k]
  float* psel;           // [M, G, k]
  float* gates;          // [M, G, k]
  float* wslot;          // [M, G, k]
  unsigned long long* psum_fx;  // [2][kMaxExperts] probability sums, fixed point
  int32_t* cursor;       // [2][kMaxExperts] bucket cursors
  const int32_t* set_flag;  // the set of this call (0 or 1)
  int32_t* bucket;       // [N * M]
};

// Routing statistics written by the routed projection's CTA 0 when it schedules from the
// cursors ("GQE" README, Algorithm Overview; the Switch-style load-balancing loss).
struct StatsOut {
  int32_t* counts;       // [N]
  float* mean_prob;      // [N]
  int32_t* offsets;      // [N + 1]
  float* aux;            // [1] or null
  int32_t* tile_count;
};

struct Params {
  CUtensorMap tmap_a;                   // A [M, K] (unused when gathering)
  CUtensorMap tmap_b[MAX_PROBLEMS];     // B [N_p, K] per problem
  Problem prob[MAX_PROBLEMS];
  int nprob;
  int M, K;
  int m_tiles;
  int tiles_per_m;                      // column tiles: sum of n_tiles over problems
  int total_tiles;                      // dense: m_tiles * tiles_per_m
  // (problem, first column) of each column tile. Column-major (col_major): tile t covers
  // column tile t / m_tiles of row tile t % m_tiles, so the CTAs' round-robin passes deal
  // out the column tiles in this order (router tiles one per CTA, then the widest) instead
  // of giving some CTAs only narrow tiles and others only full ones. Otherwise row-major:
  // row tile t / tiles_per_m, column tile t % tiles_per_m (neighbouring CTAs share A rows).
  int2 ctile[MAX_COL_TILES];
  int col_major;
  // routed projection (gather mode)
  const __nv_bfloat16* x;               // A rows gathered from x [M, K]
  const int32_t* bucket;                // entries (t << 3) | r
  const int2* tile_list;                // (expert | rows << 8, first bucket slot) per tile
  const int32_t* tile_count;            // number of tiles (device)
  // scheduling from the dense projection's cursors instead of the tile list (rc non-null):
  // expert e's bucket holds rc[set][e] entries for the call's set (*set_flag); CTA 0 also
  // writes the statistics; the last CTA to finish flips *set_flag
  const int32_t* rc;                    // [2][kMaxExperts]
  const unsigned long long* rpsum;      // [2][kMaxExperts] probability sums, fixed point
  int32_t* set_flag;
  int32_t* exit_counter;                // zero between calls
  int nexp;
  // experts whose buckets this projection computes: [e_lo, e_hi) (a group range of the
  // layer, see gqe_set_group_range); W_q holds their rows only and their query streams
  // are numbered from the range's first group
  int e_lo, e_hi;
  StatsOut so;
  __nv_bfloat16* Q;                     // query streams [S, M, d_h]
  // dense projection with routing (the ROUTE instance): problem 0 = W_r
  int G;
  RouteOut ro;
  int E, k, d_h;
  int32_t* status;
  int64_t spin;
};

struct TileInfo {
  int p;       // problem (dense) or expert (gather)
  int m0;      // first row: token row (dense) or bucket slot (gather)
  int rows;    // valid rows in the tile
  int n0;      // first column within the problem
  int n;       // MMA N (multiple of 16)
};

// Routed-projection tile `tile` as (expert | rows << 8, first bucket slot): from the tile
// list, or (scheduling from the cursors) from the per-expert counts s_cnt and first tiles
// s_t0 [nexp + 1] in shared memory (experts in order; each bucket cut into runs of 128).
__device__ __forceinline__ int2 tile_entry(const Params& P, const int* s_cnt, const int* s_t0,
                                           int tile) {
  if (P.rc == nullptr) return P.tile_list[tile];
  int x = 0;
  while (x + 1 < P.nexp && s_t0[x + 1] <= tile) ++x;
  const int i = tile - s_t0[x];
  return make_int2(x | min(BM, s_cnt[x] - BM * i) << 8, x * P.M + i * BM);
}

template <bool GATHER>
__device__ __forceinline__ TileInfo tile_info(const Params& P, int tile, const int* s_cnt,
                                              const int* s_t0) {
  TileInfo ti;
  if constexpr (GATHER) {
    const int2 t = tile_entry(P, s_cnt, s_t0, tile);  // (expert | rows << 8, first slot)
    ti.p = t.x & 255;
    ti.m0 = t.y;
    ti.rows = t.x >> 8;
    ti.n0 = 0;
    ti.n = P.prob[0].box_n;
  } else {
    int j, mt;
    if (P.col_major) {
      j = tile / P.m_tiles;
      mt = tile - j * P.m_tiles;
    } else {
      mt = tile / P.tiles_per_m;
      j = tile - mt * P.tiles_per_m;
    }
    const int2 ct = P.ctile[j];
    const int p = ct.x;
    ti.p = p;
    ti.m0 = mt * BM;
    ti.rows = min(BM, P.M - ti.m0);
    ti.n0 = ct.y;
    const int rem = P.prob[p].N - ti.n0;
    ti.n = min(BN, (rem + 15) / 16 * 16);
  }
  return ti;
}

__device__ __forceinline__ void set_timeout(const Params& P, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicExch(P.status, kStatusTimeout);
}

// Fixed-point scale of the per-expert probability sums (integer additions do not depend on
// their order, so the sums are the same whatever order the warps add them in).
constexpr double kProbFix = 4294967296.0;  // 2^32

// Routing of a router tile's rows, in the dense projection's epilogue ("GQE: Grouped Query
// Experts" README, Algorithm Overview: N experts in G groups, the top k of each group by
// router logit, ties to the lower index; softmax over each group's experts; gist.science
// summary, Load Balancing). One thread per token (its TMEM lane), N and E = N / G fixed at
// compile time so every index is static and the logits never leave registers:
//   - the N fp32 logits come from TMEM; the accumulator is released; the row is stored;
//   - per group: the top k (k passes of an argmax, ties to the lower index), the softmax
//     p, the group's selected mass; sel (ascending expert index), p_sel, the gates
//     p_sel / (group's selected mass) and the slot weights p_sel / (all G k selections);
//   - per expert, over the warp's 32 tokens: the selection count (a ballot) and the
//     probability sum (a butterfly), which lane e adds to the expert's totals: its bucket
//     cursor (the atomic returns the warp's first slot) and, in fixed point, its
//     probability sum;
//   - the bucket entries (token << 3) | rank, in lane order within the warp's run.
// The only memory round trip on this path is that atomic.
template <int N, int E>
__device__ void route_rows(const Params& P, uint32_t t_row, int t, bool valid, int lane,
                           uint64_t* acc_empty, int cset) {
  constexpr int G = N / E;
  constexpr unsigned all = 0xffffffffu;
  const RouteOut& R = P.ro;
  const int k = P.k;
  float lg[N];
#pragma unroll
  for (int c0 = 0; c0 < N; c0 += 16) {
    uint32_t r[16];
    tmem_ld16_wait(t_row + c0, r);
#pragma unroll
    for (int x = 0; x < 16; ++x)
      if (c0 + x < N) lg[c0 + x] = __uint_as_float(r[x]);
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(acc_empty);
  if (valid) {
    float* d = R.logits_out + (int64_t)t * N;
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int c = 0; c < N; c += 4)
        *reinterpret_cast<float4*>(d + c) = make_float4(lg[c], lg[c + 1], lg[c + 2], lg[c + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < N; ++c) d[c] = lg[c];
    }
  }
  // selections and probabilities
  uint32_t hit = 0;  // bit e: expert e selected
  float p[N];
  float psum[G];
  float p_tot = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float* l = lg + g * E;
    uint32_t taken = 0;
    for (int r = 0; r < k; ++r) {
      int best = 0;
      float bv = -INFINITY;
      bool any = false;
#pragma unroll
      for (int j = 0; j < E; ++j) {
        const bool ok = !(taken >> j & 1u) && (!any || l[j] > bv);
        best = ok ? j : best;
        bv = ok ? l[j] : bv;
        any = any || !(taken >> j & 1u);
      }
      taken |= 1u << best;
    }
    float mx = l[0];
#pragma unroll
    for (int j = 1; j < E; ++j) mx = fmaxf(mx, l[j]);
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      p[g * E + j] = expf(l[j] - mx);
      den += p[g * E + j];
    }
    const float inv = 1.f / den;
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      p[g * E + j] *= inv;
      if (taken >> j & 1u) s += p[g * E + j];
    }
    psum[g] = s;
    p_tot += s;
    hit |= (E == 32 ? taken : (taken & ((1u << (E & 31)) - 1u))) << (g * E);
  }
  if (!valid) hit = 0;
  if (valid) {
    const float winv = 1.f / p_tot;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float ginv = 1.f / psum[g];
      int r = 0;
#pragma unroll
      for (int j = 0; j < E; ++j) {
        if (!(hit >> (g * E + j) & 1u)) continue;
        const int64_t o = (int64_t)t * G * k + g * k + r;
        R.sel[o] = j;
        R.psel[o] = p[g * E + j];
        R.gates[o] = p[g * E + j] * ginv;
        R.wslot[o] = p[g * E + j] * winv;
        ++r;
      }
    }
  }
  // per expert over the warp: counts and probability sums; lane e keeps expert e's
  uint32_t bal[N];
  int my_cnt = 0;
  float my_sum = 0.f;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    bal[e] = __ballot_sync(all, hit >> e & 1u);
    float s = valid ? p[e] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(all, s, o);
    if (lane == e) {
      my_cnt = __popc(bal[e]);
      my_sum = s;
    }
  }
  int my_base = 0;
  if (lane < N) {
    if (my_cnt) my_base = atomicAdd(&R.cursor[cset + lane], my_cnt);
    atomicAdd(&R.psum_fx[cset + lane],
              (unsigned long long)__double2ll_rn((double)my_sum * kProbFix));
  }
  const unsigned below = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const int base = __shfl_sync(all, my_base, e);
    if (hit >> e & 1u) {
      const int g0 = (e / E) * E;
      const uint32_t grp_below = hit & ((1u << e) - 1u) & ~((1u << g0) - 1u);
      const int slot = base + __popc(bal[e] & below);
      if (slot < P.M) R.bucket[(int64_t)e * P.M + slot] = (t << 3) | __popc(grp_below);
    }
  }
}

template <int N>
__device__ void route_rows_e(const Params& P, uint32_t t_row, int t, bool valid, int lane,
                             uint64_t* bar, int cset) {
  switch (N / P.G) {
    case 1: route_rows<N, 1>(P, t_row, t, valid, lane, bar, cset); break;
    case 2: if constexpr (N >= 2) route_rows<N, (N >= 2 ? 2 : 1)>(P, t_row, t, valid, lane, bar, cset); break;
    case 4: if constexpr (N >= 4) route_rows<N, (N >= 4 ? 4 : 1)>(P, t_row, t, valid, lane, bar, cset); break;
    case 8: if constexpr (N >= 8) route_rows<N, (N >= 8 ? 8 : 1)>(P, t_row, t, valid, lane, bar, cset); break;
    case 16: if constexpr (N >= 16) route_rows<N, (N >= 16 ? 16 : 1)>(P, t_row, t, valid, lane, bar, cset); break;
    default: if constexpr (N >= 32) route_rows<N, (N >= 32 ? 32 : 1)>(P, t_row, t, valid, lane, bar, cset); break;
  }
}

__device__ void route_rows_any(const Params& P, uint32_t t_row, int t, bool valid, int lane,
                               uint64_t* bar, int cset) {
  switch (P.prob[0].N) {
    case 1: route_rows_e<1>(P, t_row, t, valid, lane, bar, cset); break;
    case 2: route_rows_e<2>(P, t_row, t, valid, lane, bar, cset); break;
    case 4: route_rows_e<4>(P, t_row, t, valid, lane, bar, cset); break;
    case 8: route_rows_e<8>(P, t_row, t, valid, lane, bar, cset); break;
    case 16: route_rows_e<16>(P, t_row, t, valid, lane, bar, cset); break;
    default: route_rows_e<32>(P, t_row, t, valid, lane, bar, cset); break;
  }
}

// The routed projection's schedule from the dense projection's cursors, in every CTA
// (block-wide, shared memory): s_cnt[e] = expert e's entries, s_t0[e] = its first tile
// (each bucket cut into runs of 128 slots), s_t0[nexp] = the number of tiles. CTA 0 also
// writes the routing statistics ("GQE" README, Algorithm Overview; the Switch-style
// load-balancing loss): counts, mean_prob (fixed-point sum / M), offsets (e M) and
//   L = (1/G) sum_e E f_e Pbar_e,  f = count / (M k),  Pbar = prob_sum / M.
__device__ void routed_schedule(const Params& P, int* s_cnt, int* s_t0, double* s_ps) {
  const int N = P.nexp, M = P.M;
  const int tid = threadIdx.x;
  if (tid < N) {
    // the set flag and both sets' counts (and, in CTA 0, probability sums) in one round
    // trip; the flag then picks the call's set
    const int flag = __ldcg(P.set_flag);
    const int c0 = __ldcg(P.rc + tid), c1 = __ldcg(P.rc + kMaxExperts + tid);
    long long p0 = 0, p1 = 0;
    if (blockIdx.x == 0) {
      p0 = __ldcg(reinterpret_cast<const long long*>(P.rpsum) + tid);
      p1 = __ldcg(reinterpret_cast<const long long*>(P.rpsum) + kMaxExperts + tid);
    }
    const bool second = flag & 1;
    // a count above M would mean a cursor set that was not cleared: never reached, but the
    // bucket reads stay inside expert e's M slots whatever the cursors hold
    const int c = second ? c1 : c0;
    s_cnt[tid] = min(max(c, 0), M);
    if (c < 0 || c > M) atomicExch(P.status, kStatusBadState);
    if (blockIdx.x == 0) s_ps[tid] = (double)(second ? p1 : p0) / kProbFix;
  }
  __syncthreads();
  if (tid == 0) {
    int nt = 0;
    for (int x = 0; x < N; ++x) {
      s_t0[x] = nt;
      if (x >= P.e_lo && x < P.e_hi) nt += (s_cnt[x] + BM - 1) / BM;
    }
    s_t0[N] = nt;
  }
  if (blockIdx.x == 0) {
    const StatsOut& S = P.so;
    const int G = N / P.E;
    if (tid < N) {
      S.counts[tid] = s_cnt[tid];
      S.offsets[tid] = tid * M;
      S.mean_prob[tid] = (float)(s_ps[tid] / M);
    }
    if (tid == 0) {
      S.offsets[N] = N * M;
      double L = 0.0;
      for (int x = 0; x < N; ++x)
        L += (double)P.E * ((double)s_cnt[x] / ((double)M * P.k)) * (s_ps[x] / M);
      if (S.aux) S.aux[0] = (float)(L / G);
    }
  }
  __syncthreads();
  if (blockIdx.x == 0 && tid == 0) *P.so.tile_count = s_t0[N];
}

// ROUTE: the dense projection whose router tiles (problem 0) route (route_rows); a separate
// instance, so the plain GEMMs carry none of that code.
template <bool GATHER, bool ROUTE, bool NARROW, bool DEEP>
__global__ void __launch_bounds__(Lay<GATHER>::THREADS, DEEP ? 1 : CTAS_PER_SM)
tc_gemm_kernel(const __grid_constant__ Params P) {
  using L = Lay<GATHER>;
  using R = Ring<NARROW, DEEP>;
  constexpr int STAGES = R::STAGES;
  constexpr int A_STAGE_BYTES = R::A_BYTES;
  constexpr int B_STAGE_BYTES = R::B_BYTES;
  // A producer warp waits only for the stage it fills next; with more producer warps than
  // stages one of them could get two uses of a stage ahead of the MMA warp, and a parity
  // wait cannot tell those phases apart.
  static_assert(L::NPROD <= STAGES, "a producer warp could lap the stage ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  uint8_t* scratch = reinterpret_cast<uint8_t*>(acc_empty + 2) + 16;  // routed schedule

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], GATHER ? 33 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == L::MMA) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.tmap_a);
    for (int p = 0; p < P.nprob; ++p) prefetch_tmap(&P.tmap_b[p]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int KB = (P.K + BK - 1) / BK;
  pdl_wait();  // the previous kernel's outputs (x, the buckets, Z) are complete from here on
  pdl_allow_next();
  int* s_cnt = reinterpret_cast<int*>(scratch);         // [kMaxExperts] routed schedule
  int* s_t0 = s_cnt + kMaxExperts;                      // [kMaxExperts + 1]
  double* s_ps = reinterpret_cast<double*>(scratch + kPsOffset);  // [kMaxExperts] (CTA 0)
  int total = P.total_tiles;
  int cset = 0;  // this call's cursor set, as an offset into the two sets
  if constexpr (ROUTE) {
    // Only the epilogue warps route, so only they read the set flag (the producer and MMA
    // warps start at once). This call's set is zero; two epilogue warps of CTA 0 clear the
    // other one (the previous call's, whose last reader has finished).
    if (warp >= L::EPI0) {
      cset = (__ldcg(P.ro.set_flag) & 1) * kMaxExperts;
      const int e = threadIdx.x - L::EPI0 * 32;
      if (blockIdx.x == 0 && e < kMaxExperts) {
        const int other = kMaxExperts - cset;
        P.ro.cursor[other + e] = 0;
        P.ro.psum_fx[other + e] = 0ull;
      }
    }
  }
  if constexpr (GATHER) {
    if (P.rc != nullptr) {
      routed_schedule(P, s_cnt, s_t0, s_ps);  // block-wide
      total = s_t0[P.nexp];
    } else {
      total = *P.tile_count;
    }
  }

  if (warp < L::NPROD) {
    // ------------------------------------------------------------------ producers
    if constexpr (!GATHER) {
      // One lane issues TMA tile loads of A and B.
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        const TileInfo ti = tile_info<false>(P, tile, nullptr, nullptr);
        const uint32_t b_bytes = (uint32_t)P.prob[ti.p].box_n * BK * 2;
        for (int kb = 0; kb < KB; ++kb) {
          bool ok = mbar_wait(&empty[stage], phase ^ 1, P.spin);
          ok = !__any_sync(0xffffffffu, !ok);
          if (!ok) {
            if (lane == 0) set_timeout(P, abort_flag);
            break;
          }
          if (elect_one()) {
            mbar_arrive_expect_tx(&full[stage], (uint32_t)A_STAGE_BYTES + b_bytes);
            tma_load_2d(sA + stage * A_STAGE_BYTES, &P.tmap_a, kb * BK, ti.m0, &full[stage]);
            tma_load_2d(sB + stage * B_STAGE_BYTES, &P.tmap_b[ti.p], kb * BK, ti.n0, &full[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    } else {
      // NPROD producer warps; warp p fills stages p, p + NPROD, ... of the CTA's stage sequence.
      // A rows are gathered by asynchronous 16-byte copies (cp.async, no registers, many
      // stages in flight): lane l moves chunk l % 8 of rows 4 i + l / 8 (eight lanes per
      // 128-byte row segment: coalesced reads, conflict-free writes into the
      // 128-byte-swizzled slot). B (the expert's W_q rows) comes by TMA. The stage's full
      // barrier takes 33 arrivals: the TMA's, and one per lane when its copies complete.
      const int pw = warp;
      const int c = lane & 7;
      uint32_t g = 0;  // position in the CTA's stage sequence
      // Index pipeline: the tile-list entry two tiles ahead and the bucket entries (source
      // rows) of the next tile are loaded while this tile's rows stream, and only used a
      // tile later, so no tile boundary waits for an index load.
      const int stride = gridDim.x;
      int tile = blockIdx.x;
      int2 t = tile < total ? tile_entry(P, s_cnt, s_t0, tile) : make_int2(0, 0);
      int2 t_nxt = tile + stride < total ? tile_entry(P, s_cnt, s_t0, tile + stride)
                                         : make_int2(0, 0);
      // raw bucket entries of this lane's source rows r = 4 i + lane / 8 (rows past the
      // tile's end repeat its first row: computed, never stored)
      int raw[BM / 4], raw0;
      auto load_rows = [&](int2 tt, int (&dst)[BM / 4], int& d0) {
        const int n = tt.x >> 8;
        d0 = P.bucket[tt.y];
#pragma unroll
        for (int i = 0; i < BM / 4; ++i) {
          const int r = 4 * i + (lane >> 3);
          dst[i] = r < n ? P.bucket[tt.y + r] : 0;
        }
      };
      if (tile < total) load_rows(t, raw, raw0);
      for (; tile < total && !*abort_flag; tile += stride) {
        const int2 t_nn =
            tile + 2 * stride < total ? tile_entry(P, s_cnt, s_t0, tile + 2 * stride)
                                      : make_int2(0, 0);
        int nraw[BM / 4], nraw0 = 0;
        if (tile + stride < total) load_rows(t_nxt, nraw, nraw0);
        const int n = t.x >> 8;
        const int e = t.x & 255;
        const uint32_t b_bytes = (uint32_t)P.prob[0].box_n * BK * 2;
        // (token indices are clamped to the call's rows: defence against a bucket that a
        // failed routing pass left stale; a complete pass never needs it)
        const int first = min(raw0 >> 3, P.M - 1);
        int src[BM / 4];
#pragma unroll
        for (int i = 0; i < BM / 4; ++i) {
          const int r = 4 * i + (lane >> 3);
          src[i] = r < n ? min(raw[i] >> 3, P.M - 1) : first;
        }
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++g) {
          if ((int)(g % L::NPROD) != pw) continue;
          const int stage = (int)(g % STAGES);
          const uint32_t phase = (g / STAGES) & 1;
          ok = !__any_sync(0xffffffffu, !mbar_wait(&empty[stage], phase ^ 1, P.spin));
          if (!ok) {
            if (lane == 0) set_timeout(P, abort_flag);
            break;
          }
          if (elect_one()) {
            mbar_arrive_expect_tx(&full[stage], b_bytes);
            tma_load_2d(sB + stage * B_STAGE_BYTES, &P.tmap_b[0], kb * BK,
                        (e - P.e_lo) * P.d_h, &full[stage]);
          }
          const uint32_t dst = smem_u32(sA + stage * A_STAGE_BYTES);
          const int kcol = kb * BK + c * 8;
          // columns past K are zero-filled (nothing is read; the address stays in range)
          const uint32_t nbytes = kcol < P.K ? 16u : 0u;
          const int kc = kcol < P.K ? kcol : 0;
#pragma unroll
          for (int i = 0; i < BM / 4; ++i) {
            const int r = 4 * i + (lane >> 3);
            cp_async_16(dst + r * 128 + ((c ^ (r & 7)) << 4), P.x + (int64_t)src[i] * P.K + kc,
                        nbytes);
          }
          cp_async_mbar_arrive_noinc(&full[stage]);
        }
        if (!ok) break;
        t = t_nxt;
        t_nxt = t_nn;
        raw0 = nraw0;
#pragma unroll
        for (int i = 0; i < BM / 4; ++i) raw[i] = nraw[i];
      }
      // no copy of this warp may still be writing when the CTA leaves
      cp_async_wait<0>();
    }
  } else if (warp == L::MMA) {
    // ------------------------------------------------------------------ MMA issuer
    const uint64_t a_desc0 = smem_desc(smem_u32(sA), 1024, kSwizzle128B);
    const uint64_t b_desc0 = smem_desc(smem_u32(sB), 1024, kSwizzle128B);
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++it) {
      // Only the MMA width is needed here: constant for the routed projection, so no
      // tile-list load sits on this warp's path.
      int n_mma;
      if constexpr (GATHER) {
        n_mma = P.prob[0].box_n;
      } else {
        n_mma = tile_info<false>(P, tile, nullptr, nullptr).n;
      }
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      bool ok = true;
      ok = mbar_wait(&acc_empty[acc], acc_phase ^ 1, P.spin);
      ok = !__any_sync(0xffffffffu, !ok);
      if (!ok) {
        if (lane == 0) set_timeout(P, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      const uint32_t idesc = idesc_bf16_f32(BM, n_mma);
      for (int kb = 0; kb < KB; ++kb) {
        ok = mbar_wait(&full[stage], phase, P.spin);
        ok = !__any_sync(0xffffffffu, !ok);
        if (!ok) {
          if (lane == 0) set_timeout(P, abort_flag);
          break;
        }
        // gathered rows were written by the generic proxy (cp.async): make them visible
        // to the tensor core's reads
        if constexpr (GATHER) fence_async_shared();
        tc_fence_after();
        if (elect_one()) {
          // descriptor = base + offset in 16-byte units (K step: 32 bytes inside the atom)
          const uint64_t ad = a_desc0 + (uint64_t)(stage * (A_STAGE_BYTES >> 4));
          const uint64_t bd = b_desc0 + (uint64_t)(stage * (B_STAGE_BYTES >> 4));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(&empty[stage]);  // frees the stage when these MMAs finish
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&acc_full[acc]);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 belong to this warp
    const int row = quarter * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++it) {
      const TileInfo ti = tile_info<GATHER>(P, tile, s_cnt, s_t0);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const bool valid = row < ti.rows;
      // gather mode: this row's bucket entry, loaded before the wait
      const int ent = (GATHER && valid) ? P.bucket[ti.m0 + row] : 0;
      bool ok = true;
      ok = mbar_wait(&acc_full[acc], acc_phase, P.spin);
      ok = !__any_sync(0xffffffffu, !ok);
      if (!ok) {
        if (lane == 0) set_timeout(P, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if constexpr (GATHER) {
        __nv_bfloat16* dst = nullptr;
        if (valid) {
          const int g = (ti.p - P.e_lo) / P.E;  // the group within the range
          const int64_t s = (int64_t)g * P.k + min(ent & 7, P.k - 1);
          dst = P.Q + (s * P.M + min(ent >> 3, P.M - 1)) * P.d_h;
        }
        for (int c0 = 0; c0 < ti.n; c0 += 16) {
          uint32_t r[16];
          tmem_ld16_wait(t_row + c0, r);
          if (valid && c0 < P.d_h) {
            uint4 v0, v1;
            v0.x = pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1]));
            v0.y = pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3]));
            v0.z = pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5]));
            v0.w = pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]));
            v1.x = pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9]));
            v1.y = pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11]));
            v1.z = pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13]));
            v1.w = pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15]));
            *reinterpret_cast<uint4*>(dst + c0) = v0;
            *reinterpret_cast<uint4*>(dst + c0 + 8) = v1;
          }
        }
      } else if (ROUTE && ti.p == 0) {
        // router tile: the logits stay in registers for the routing, which also releases
        // the accumulator and stores the logits
        route_rows_any(P, t_row, ti.m0 + row, valid, lane, &acc_empty[acc], cset);
      } else {
        const Problem& pr = P.prob[ti.p];
        const OutMap& o = pr.out;
        const int64_t m = ti.m0 + row;
        for (int c0 = 0; c0 < ti.n; c0 += 16) {
          uint32_t r[16];
          tmem_ld16_wait(t_row + c0, r);
          if (!valid) continue;
#pragma unroll
          for (int g8 = 0; g8 < 2; ++g8) {
            const int c = ti.n0 + c0 + g8 * 8;  // column within the problem
            if (c >= pr.N) continue;
            const int head = c / o.head_w, col = c % o.head_w;
            const int64_t idx = head * o.head_stride + m * o.row_stride + (int64_t)col * o.col_stride;
            const uint32_t* rv = r + g8 * 8;
            if (o.f32) {
              float* d = static_cast<float*>(o.base) + idx;
              if (o.col_stride == 1 && c + 8 <= pr.N && ((reinterpret_cast<uintptr_t>(d) & 15) == 0)) {
                *reinterpret_cast<uint4*>(d) = make_uint4(rv[0], rv[1], rv[2], rv[3]);
                *reinterpret_cast<uint4*>(d + 4) = make_uint4(rv[4], rv[5], rv[6], rv[7]);
              } else {
                for (int j = 0; j < 8 && c + j < pr.N; ++j)
                  d[(int64_t)j * o.col_stride] = __uint_as_float(rv[j]);
              }
            } else {
              __nv_bfloat16* d = static_cast<__nv_bfloat16*>(o.base) + idx;
              if (o.col_stride == 1 && c + 8 <= pr.N && ((reinterpret_cast<uintptr_t>(d) & 15) == 0)) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(rv[0]), __uint_as_float(rv[1]));
                v.y = pack_bf16x2(__uint_as_float(rv[2]), __uint_as_float(rv[3]));
                v.z = pack_bf16x2(__uint_as_float(rv[4]), __uint_as_float(rv[5]));
                v.w = pack_bf16x2(__uint_as_float(rv[6]), __uint_as_float(rv[7]));
                *reinterpret_cast<uint4*>(d) = v;
              } else {
                for (int j = 0; j < 8 && c + j < pr.N; ++j)
                  d[(int64_t)j * o.col_stride] = __float2bfloat16_rn(__uint_as_float(rv[j]));
              }
            }
          }
        }
      }
      if (!(ROUTE && ti.p == 0)) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == L::MMA) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  // routed projection scheduled from the cursors: once every CTA has read this call's set,
  // the next call takes the other one
  if (GATHER && P.rc != nullptr && threadIdx.x == 0 &&
      atomicAdd(P.exit_counter, 1) == (int)gridDim.x - 1) {
    *P.set_flag ^= 1;
    *P.exit_counter = 0;
  }
}

// ---------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cudaGetLastError();
  });
  return g_encode != nullptr;
}

// 2-D bf16 tensor map: `cols` contiguous elements per row, `rows` rows `ld` elements apart;
// box of box_cols x box_rows with 128-byte swizzle (box_cols * 2 must be <= 128).
bool tmap_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t ld,
                  uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  if (!encoder()) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GATHER, bool ROUTE, bool NARROW, bool DEEP>
int launch_ring(const Params& P, int grid, cudaStream_t st) {
  constexpr int smem = Ring<NARROW, DEEP>::SMEM;
  if (!set_smem_limit_once<tc_gemm_kernel<GATHER, ROUTE, NARROW, DEEP>>(smem)) return -1;
  return launch_pdl(tc_gemm_kernel<GATHER, ROUTE, NARROW, DEEP>, dim3(grid),
                    dim3(Lay<GATHER>::THREADS), smem, st, P) == cudaSuccess
             ? 1
             : -1;
}

template <bool GATHER, bool ROUTE = false, bool NARROW = false>
int launch(gqe_ctx* h, const Params& P, int grid, cudaStream_t st) {
  return grid <= h->num_sms ? launch_ring<GATHER, ROUTE, NARROW, true>(P, grid, st)
                            : launch_ring<GATHER, ROUTE, NARROW, false>(P, grid, st);
}

Problem make_problem(int N, OutMap out) {
  Problem p;
  p.N = N;
  p.n_tiles = (N + BN - 1) / BN;
  p.box_n = N >= BN ? BN : (N + 15) / 16 * 16;
  p.out = out;
  return p;
}

// Column tiles of all problems, widest first (stable: problem order within a width). With
// `prob0_first` problem 0's tiles lead instead (the router tiles, whose epilogue routes:
// that work then overlaps the wide tiles' products rather than trailing them).
bool set_col_tiles(Params& P, bool prob0_first) {
  int n = 0;
  auto width = [&](int p, int t) {
    const int rem = P.prob[p].N - t * BN;
    return rem >= BN ? BN : (rem + 15) / 16 * 16;
  };
  if (prob0_first)
    for (int t = 0; t < P.prob[0].n_tiles && n < MAX_COL_TILES; ++t)
      P.ctile[n++] = make_int2(0, t * BN);
  for (int w = BN; w >= 16; w -= 16)
    for (int p = prob0_first ? 1 : 0; p < P.nprob; ++p)
      for (int t = 0; t < P.prob[p].n_tiles; ++t) {
        if (width(p, t) != w) continue;
        if (n == MAX_COL_TILES) return false;
        P.ctile[n++] = make_int2(p, t * BN);
      }
  P.tiles_per_m = n;
  P.total_tiles = P.m_tiles * n;
  return true;
}

int64_t spin_limit(const gqe_ctx* h) { return h->spin_limit > 0 ? h->spin_limit : (int64_t)1 << 22; }

}  // namespace

bool tmap_bf16_2d_ext(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                      uint64_t ld, uint32_t box_cols, uint32_t box_rows,
                      CUtensorMapSwizzle sw) {
  return tmap_bf16_2d(m, ptr, cols, rows, ld, box_cols, box_rows, sw);
}

// A row-major [rows, cols] bf16 matrix seen as chunks of `chunk_cols` columns: dimensions
// (column within the chunk, row, chunk), so one box of (chunk_cols, box_rows, cols /
// chunk_cols) lands in shared memory chunk after chunk, each chunk box_rows x chunk_cols --
// the layout the per-chunk 2D boxes produce, in one copy. Returns false if the driver does
// not accept the map (the caller then issues one 2D box per chunk).
bool tmap_bf16_chunked(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                       uint64_t ld, uint32_t chunk_cols, uint32_t box_rows,
                       CUtensorMapSwizzle sw) {
  if (!encoder() || cols % chunk_cols != 0) return false;
  cuuint64_t dims[3] = {chunk_cols, rows, cols / chunk_cols};
  cuuint64_t strides[2] = {ld * 2, (cuuint64_t)chunk_cols * 2};
  cuuint32_t box[3] = {chunk_cols, box_rows, (cuuint32_t)(cols / chunk_cols)};
  cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The dense projection routes (see route_rows) for N a power of two up to 32.
bool tc_dense_routes(const gqe_ctx* h) { return h->N <= 32 && (h->N & (h->N - 1)) == 0; }

// Also routes when tc_dense_routes(h): the router tiles' epilogue selects the experts and
// fills the buckets, and the last CTA forms the statistics, the aux loss (if aux_out) and
// the routed-projection tiles.
int launch_tc_dense_proj(gqe_ctx* h, const void* x, int M, const void* W_r, const void* W_k,
                         const void* W_v, const void* W_shared, cudaStream_t st) {
  const int d_h = h->d_h, G = h->g1 - h->g0, dim = h->dim;  // this handle's KV heads
  const int S = G * h->k + (W_shared ? 1 : 0);
  Params P;
  memset(&P, 0, sizeof(P));
  if (!tmap_bf16_2d(&P.tmap_a, x, dim, M, dim, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B)) return -1;
  const void* Bs[4] = {W_r, W_k, W_v, W_shared};
  const int Ns[4] = {h->N, G * d_h, G * d_h, d_h};
  OutMap outs[4] = {
      OutMap{h->ws.logits, 0, h->N, 1, 1 << 30, 1},
      OutMap{h->ws.K, (int64_t)M * d_h, d_h, 1, d_h, 0},
      OutMap{h->ws.V, (int64_t)M * d_h, d_h, 1, d_h, 0},
      OutMap{static_cast<char*>(h->ws.Q) + (int64_t)(S - 1) * M * d_h * 2, 0, d_h, 1, d_h, 0}};
  int np = 0;
  for (int i = 0; i < 4; ++i) {
    if (!Bs[i]) continue;
    P.prob[np] = make_problem(Ns[i], outs[i]);
    if (!tmap_bf16_2d(&P.tmap_b[np], Bs[i], dim, Ns[i], dim, BK, P.prob[np].box_n,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return -1;
    ++np;
  }
  P.nprob = np;
  P.M = M;
  P.K = dim;
  P.m_tiles = (M + BM - 1) / BM;
  const bool route = tc_dense_routes(h);
  if (!set_col_tiles(P, route)) return -1;
  P.col_major = 1;
  P.status = h->ws.status;
  P.spin = spin_limit(h);
  P.G = h->G;  // routing covers every group
  P.k = h->k;
  const Workspace& w = h->ws;
  P.ro = RouteOut{w.logits, w.sel, w.psel, w.gates, w.w, w.rpsum, w.rcur,
                  w.rcur + kRouteFlag, w.bucket};
  const int grid = min(P.total_tiles, CTAS_PER_SM * h->num_sms);
  return route ? launch<false, true>(h, P, grid, st) : launch<false>(h, P, grid, st);
}

// The tile list (expert | rows << 8, first bucket slot) and its length come from the routing.
// from_cursors: schedule from the dense projection's cursors (the call's set) and write the
// routing statistics (aux_out if non-null); otherwise from the routing kernel's tile list.
int launch_tc_qproj(gqe_ctx* h, const void* x, int M, const void* W_q, bool from_cursors,
                    float* aux_out, cudaStream_t st) {
  Params P;
  memset(&P, 0, sizeof(P));
  // A: rows of x gathered four at a time (box one row high, 128 bytes wide)
  if (!tmap_bf16_2d(&P.tmap_a, x, h->dim, M, h->dim, BK, 1, CU_TENSOR_MAP_SWIZZLE_128B))
    return -1;
  P.prob[0] = make_problem(h->d_h, OutMap{});
  P.e_lo = h->g0 * h->E;
  P.e_hi = h->g1 * h->E;
  if (!tmap_bf16_2d(&P.tmap_b[0], W_q, h->dim, (uint64_t)(P.e_hi - P.e_lo) * h->d_h, h->dim,
                    BK, P.prob[0].box_n, CU_TENSOR_MAP_SWIZZLE_128B))
    return -1;
  P.nprob = 1;
  P.M = M;
  P.K = h->dim;
  P.x = static_cast<const __nv_bfloat16*>(x);
  P.bucket = h->ws.bucket;
  P.tile_list = h->ws.tile_list;
  P.tile_count = h->ws.tile_count;
  if (from_cursors) {
    P.rc = h->ws.rcur;
    P.rpsum = h->ws.rpsum;
    P.set_flag = h->ws.rcur + kRouteFlag;
    P.exit_counter = h->ws.rcur + kRouteFlag + 1;
    P.so = StatsOut{h->ws.counts, h->ws.mean_prob, h->ws.offsets, aux_out, h->ws.tile_count};
  }
  P.nexp = h->N;
  P.Q = static_cast<__nv_bfloat16*>(h->ws.Q);
  P.E = h->E;
  P.k = h->k;
  P.d_h = h->d_h;
  P.status = h->ws.status;
  P.spin = spin_limit(h);
  const int max_tiles = (int)(((int64_t)M * h->G * h->k + BM - 1) / BM) + h->N;
  const int grid = min(max_tiles, CTAS_PER_SM * h->num_sms);
  return P.prob[0].box_n <= Ring<true>::B_ROWS ? launch<true, false, true>(h, P, grid, st)
                                                : launch<true>(h, P, grid, st);
}

int launch_tc_oproj(gqe_ctx* h, int M, int Do, const void* W_o, void* out, cudaStream_t st) {
  Params P;
  memset(&P, 0, sizeof(P));
  if (!tmap_bf16_2d(&P.tmap_a, h->ws.Z, Do, M, Do, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B)) return -1;
  P.prob[0] = make_problem(h->dim, OutMap{out, 0, h->dim, 1, 1 << 30, 0});
  if (!tmap_bf16_2d(&P.tmap_b[0], W_o, Do, h->dim, Do, BK, P.prob[0].box_n,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return -1;
  P.nprob = 1;
  P.M = M;
  P.K = Do;
  P.m_tiles = (M + BM - 1) / BM;
  if (!set_col_tiles(P, false)) return -1;
  P.status = h->ws.status;
  P.spin = spin_limit(h);
  const int grid = min(P.total_tiles, CTAS_PER_SM * h->num_sms);
  return launch<false>(h, P, grid, st);
}

}  // namespace gqe
