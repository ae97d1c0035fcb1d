// Router: per-group softmax, top-k, gates, slot weights, load statistics, expert buckets.
//
// "GQE: Grouped Query Experts" README, Algorithm Overview: a softmax over the experts of
// each GQA group, then top-k; a Switch-style load-balancing loss. gist.science summary,
// Output Construction: a renormalised weighted sum of the selected outputs using the
// router probabilities (the slot weights w below).
#include "gqe_common.cuh"

namespace gqe {

// Selection for one block of kRouteBlock tokens, one thread per token. The block's logits
// [128, N] are staged in shared memory (one coalesced copy) and every per-token array lives
// there too, so nothing spills to local memory. Writes sel / p_sel / gates / w [M, G, k] and
// this block's per-expert token counts and probability sums to part_counts / part_prob
// [blk, N] (summed later in a fixed order, so the result does not depend on scheduling).
// Leaves the block's selection flags in s_hit.
__device__ void select_block(const float* __restrict__ logits, int blk, int M, int N, int G,
                             int k, int32_t* __restrict__ sel, float* __restrict__ psel,
                             float* __restrict__ gates, float* __restrict__ wslot,
                             int32_t* __restrict__ part_counts, float* __restrict__ part_prob,
                             float (*s_p)[kMaxExperts + 1],
                             unsigned char (*s_hit)[kMaxExperts + 1]) {
  const int E = N / G;
  const int t0 = blk * kRouteBlock;
  const int tid = threadIdx.x;
  const int t = t0 + tid;
  const bool valid = t < M;
  const int rows = min(kRouteBlock, M - t0);
  for (int i = tid; i < kRouteBlock * N; i += kRouteBlock) {
    const int r = i / N, e = i % N;
    s_p[r][e] = r < rows ? logits[(int64_t)t0 * N + i] : 0.f;
    s_hit[r][e] = 0;
  }
  __syncthreads();
  float* p = s_p[tid];
  unsigned char* hit = s_hit[tid];
  float p_tot = 0.f;
  for (int g = 0; g < G; ++g) {
    float* lg = p + g * E;
    // top-k on the logits: k passes of argmax over the experts not yet taken; a strict
    // comparison keeps the lowest index among equal maxima.
    uint64_t taken = 0;
    for (int r = 0; r < k; ++r) {
      int best = -1;
      float bv = 0.f;
      for (int j = 0; j < E; ++j) {
        if (taken >> j & 1ull) continue;
        if (best < 0 || lg[j] > bv) {
          best = j;
          bv = lg[j];
        }
      }
      taken |= 1ull << best;
    }
    // softmax within the group, fp32 with max subtraction (in place)
    float mx = lg[0];
    for (int j = 1; j < E; ++j) mx = fmaxf(mx, lg[j]);
    float den = 0.f;
    for (int j = 0; j < E; ++j) {
      const float z = expf(lg[j] - mx);
      lg[j] = z;
      den += z;
    }
    const float inv = 1.f / den;
    float psum = 0.f;
    for (int j = 0; j < E; ++j) {
      lg[j] *= inv;
      if (taken >> j & 1ull) psum += lg[j];
    }
    // the selected set in ascending expert index
    const float ginv = 1.f / psum;
    int r = 0;
    for (int j = 0; j < E; ++j) {
      if (!(taken >> j & 1ull)) continue;
      hit[g * E + j] = 1;
      if (valid) {
        const int64_t o = (int64_t)t * G * k + g * k + r;
        sel[o] = j;
        psel[o] = lg[j];
        gates[o] = lg[j] * ginv;
      }
      ++r;
    }
    p_tot += psum;
  }
  // slot weights: p of each selection renormalised over all G*k selections
  if (valid) {
    const float winv = 1.f / p_tot;
    for (int g = 0; g < G; ++g) {
      int r = 0;
      for (int j = 0; j < E; ++j)
        if (hit[g * E + j]) wslot[(int64_t)t * G * k + g * k + r++] = p[g * E + j] * winv;
    }
  } else {
    for (int e = 0; e < N; ++e) {
      p[e] = 0.f;
      hit[e] = 0;
    }
  }
  __syncthreads();
  if (tid < N) {
    float ps = 0.f;
    int c = 0;
    for (int i = 0; i < kRouteBlock; ++i) {
      ps += s_p[i][tid];
      c += s_hit[i][tid];
    }
    part_prob[(int64_t)blk * N + tid] = ps;
    part_counts[(int64_t)blk * N + tid] = c;
  }
}

__global__ void __launch_bounds__(kRouteBlock)
route_select_kernel(const float* __restrict__ logits, int M, int N, int G, int k,
                    int32_t* __restrict__ sel, float* __restrict__ psel,
                    float* __restrict__ gates, float* __restrict__ wslot,
                    int32_t* __restrict__ part_counts, float* __restrict__ part_prob) {
  __shared__ float s_p[kRouteBlock][kMaxExperts + 1];          // logits, then probabilities
  __shared__ unsigned char s_hit[kRouteBlock][kMaxExperts + 1];  // selected experts
  select_block(logits, blockIdx.x, M, N, G, k, sel, psel, gates, wslot, part_counts, part_prob,
               s_p, s_hit);
}

// One block of 32 warps; warp w handles experts w and w + 32. Lane l sums a contiguous run
// of router blocks; counts are combined by a warp prefix scan and probabilities (double) by
// a fixed shuffle tree, so the result does not depend on scheduling. Writes counts /
// mean_prob / the bucket offsets, turns part_counts into each (block, expert)'s first
// bucket slot, and computes the Switch loss
//   L = (1/G) sum_g E sum_j f_{g,j} Pbar_{g,j},  f = c / (M k),  Pbar = prob_sum / M.
__global__ void __launch_bounds__(1024)
route_scan_aux_kernel(int32_t* __restrict__ part_counts, const float* __restrict__ part_prob,
                      int nblk, int M, int N, int G, int k, int32_t* __restrict__ counts,
                      float* __restrict__ mean_prob, int32_t* __restrict__ offsets,
                      float* __restrict__ aux_out) {
  __shared__ int s_cnt[kMaxExperts];
  __shared__ double s_term[kMaxExperts];
  __shared__ int s_off[kMaxExperts + 1];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int chunk = (nblk + 31) / 32;
  const int b0 = min(nblk, lane * chunk), b1 = min(nblk, b0 + chunk);
  int my_count[2] = {0, 0};
  int my_prefix[2] = {0, 0};
  for (int h = 0; h < 2; ++h) {
    const int e = warp + 32 * h;
    if (e >= N) break;
    int c = 0;
    double ps = 0.0;
    for (int b = b0; b < b1; ++b) {
      c += part_counts[(int64_t)b * N + e];
      ps += (double)part_prob[(int64_t)b * N + e];
    }
    // exclusive prefix of c over lanes, and the total
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    my_count[h] = c;
    my_prefix[h] = incl - c;
    if (lane == 0) {
      counts[e] = total;
      mean_prob[e] = (float)(ps / M);
      s_cnt[e] = total;
      s_term[e] = (double)(N / G) * ((double)total / ((double)M * k)) * (ps / M);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0;
    for (int e = 0; e < N; ++e) {
      s_off[e] = off;
      offsets[e] = off;
      off += s_cnt[e];
    }
    offsets[N] = off;
    if (aux_out != nullptr) {
      double L = 0.0;
      for (int e = 0; e < N; ++e) L += s_term[e];
      aux_out[0] = (float)(L / G);
    }
  }
  __syncthreads();
  for (int h = 0; h < 2; ++h) {
    const int e = warp + 32 * h;
    if (e >= N) break;
    int run = s_off[e] + my_prefix[h];
    for (int b = b0; b < b1; ++b) {
      const int v = part_counts[(int64_t)b * N + e];
      part_counts[(int64_t)b * N + e] = run;
      run += v;
    }
  }
}

// Grid (nblk, N): block (b, e) writes the entries of expert e for the tokens of router
// block b, in token order, starting at the slot the scan assigned. Entry = (t << 3) | r,
// r = the rank of e among token t's selections in its group (its query stream g*k + r).
__global__ void __launch_bounds__(kRouteBlock)
bucket_kernel(const int32_t* __restrict__ sel, const int32_t* __restrict__ base, int M, int N,
              int G, int k, int32_t* __restrict__ bucket) {
  __shared__ int s_warp[kRouteBlock / 32];
  const int e = blockIdx.y;
  const int E = N / G;
  const int g = e / E, j = e % E;
  const int t = blockIdx.x * kRouteBlock + threadIdx.x;
  int rank = -1;
  if (t < M) {
    for (int r = 0; r < k; ++r)
      if (sel[(int64_t)t * G * k + g * k + r] == j) rank = r;
  }
  const unsigned ball = __ballot_sync(0xffffffffu, rank >= 0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_warp[warp] = __popc(ball);
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += s_warp[w];
  before += __popc(ball & ((1u << lane) - 1u));
  if (rank >= 0) {
    const int slot = base[(int64_t)blockIdx.x * N + e] + before;
    bucket[slot] = (t << 3) | rank;
  }
}

// ---------------------------------------------------------------------------------------
// The whole routing stage in one pass, without a grid barrier: selection, the expert
// buckets, the per-expert statistics and Switch loss, and the routed-projection tile list.
// CTAs of kFusedThreads take blocks of kRouteBlock tokens. Per token and group the
// arithmetic is that of select_block (same operations in the same order), so selections,
// gates and statistics equal route_select_kernel's; the work is spread over one thread per
// (token, group).
//
// Buckets: expert e owns slots [e M, e M + count_e) of the bucket array (room for every
// token). A block claims a contiguous run of each expert's slots with one integer atomic on
// the expert's cursor, so the order of tokens inside a bucket depends on scheduling; every
// routed query row is computed on its own (its value does not depend on which rows share
// its tile), so the results do not. The last CTA to finish (an atomic ticket) turns the
// cursors into counts, reduces the per-block probability sums in block order (the same
// arithmetic as the scan of route_scan_aux_kernel), writes the Switch loss and the tile
// list, and sets the cursors and the ticket back to zero for the next call.
// ---------------------------------------------------------------------------------------
constexpr int kFusedThreads = 512;

// Scratch after the selection arrays: the bucket phase's arrays, the block's counts, and
// the last CTA's reduction arrays.
__host__ __device__ inline int fused_bucket_bytes(int N) {
  return ((kRouteBlock * N + 15) / 16 * 16 + 4 * N + 4 * N * (kRouteBlock / 32) + 15) / 16 * 16;
}
constexpr int kStatsBytes = 8 * kFusedThreads + 8 * kMaxExperts + 4 * kFusedThreads +
                            4 * kMaxExperts + 2 * 4 * (kMaxExperts + 1);
__host__ __device__ inline int fused_smem_bytes(int N, int G) {
  const int sel_bytes = kRouteBlock * N * 4 + kRouteBlock * G * 4 + kRouteBlock * N;
  return (sel_bytes + 15) / 16 * 16 + fused_bucket_bytes(N) + 4 * kMaxExperts + kStatsBytes + 64;
}

// Selection of one token block, one thread per (token, group). Leaves the probabilities in
// s_p [128][N], the chosen experts' ranks + 1 in s_hit [128][N] (0 = not chosen) and the
// block's per-expert token counts in s_count [N]; writes sel / p_sel / gates / w and the
// block's part_counts / part_prob.
__device__ void fused_select(const float* __restrict__ logits, int blk, int M, int N, int G,
                             int k, int32_t* __restrict__ sel, float* __restrict__ psel,
                             float* __restrict__ gates, float* __restrict__ wslot,
                             int32_t* __restrict__ part_counts, float* __restrict__ part_prob,
                             float* s_p, unsigned char* s_hit, float* s_psum, int* s_count) {
  const int E = N / G;
  const int tid = threadIdx.x;
  const int t0 = blk * kRouteBlock;
  const int rows = min(kRouteBlock, M - t0);
  const float* src = logits + (int64_t)t0 * N;
#pragma unroll 4
  for (int i = tid; i < kRouteBlock * N; i += kFusedThreads) {
    s_p[i] = i < rows * N ? __ldcg(src + i) : 0.f;
    s_hit[i] = 0;
  }
  __syncthreads();
  for (int pi = tid; pi < kRouteBlock * G; pi += kFusedThreads) {
    const int tl = pi / G, g = pi % G;
    const int t = t0 + tl;
    float* lg = s_p + tl * N + g * E;
    unsigned char* hit = s_hit + tl * N + g * E;
    if (t >= M) {
      for (int j = 0; j < E; ++j) lg[j] = 0.f;
      s_psum[tl * G + g] = 0.f;
      continue;
    }
    // top-k on the logits (ties: the lowest index), then the group softmax in place
    uint64_t taken = 0;
    for (int r = 0; r < k; ++r) {
      int best = -1;
      float bv = 0.f;
      for (int j = 0; j < E; ++j) {
        if (taken >> j & 1ull) continue;
        if (best < 0 || lg[j] > bv) {
          best = j;
          bv = lg[j];
        }
      }
      taken |= 1ull << best;
    }
    float mx = lg[0];
    for (int j = 1; j < E; ++j) mx = fmaxf(mx, lg[j]);
    float den = 0.f;
    for (int j = 0; j < E; ++j) {
      const float z = expf(lg[j] - mx);
      lg[j] = z;
      den += z;
    }
    const float inv = 1.f / den;
    float psum = 0.f;
    for (int j = 0; j < E; ++j) {
      lg[j] *= inv;
      if (taken >> j & 1ull) psum += lg[j];
    }
    const float ginv = 1.f / psum;
    int r = 0;
    for (int j = 0; j < E; ++j) {
      if (!(taken >> j & 1ull)) continue;
      hit[j] = (unsigned char)(r + 1);
      const int64_t o = (int64_t)t * G * k + g * k + r;
      sel[o] = j;
      psel[o] = lg[j];
      gates[o] = lg[j] * ginv;
      ++r;
    }
    s_psum[tl * G + g] = psum;
  }
  __syncthreads();
  // slot weights: p of each selection renormalised over the token's G*k selections
  for (int pi = tid; pi < kRouteBlock * G; pi += kFusedThreads) {
    const int tl = pi / G, g = pi % G;
    const int t = t0 + tl;
    if (t >= M) continue;
    float p_tot = 0.f;
    for (int gg = 0; gg < G; ++gg) p_tot += s_psum[tl * G + gg];
    const float winv = 1.f / p_tot;
    int r = 0;
    for (int j = 0; j < E; ++j)
      if (s_hit[tl * N + g * E + j])
        wslot[(int64_t)t * G * k + g * k + r++] = s_p[tl * N + g * E + j] * winv;
  }
  // per-expert sums over the block's tokens, in token order
  if (tid < N) {
    float ps = 0.f;
    int c = 0;
    for (int i = 0; i < kRouteBlock; ++i) {
      ps += s_p[i * N + tid];
      c += s_hit[i * N + tid] != 0;
    }
    part_prob[(int64_t)blk * N + tid] = ps;
    part_counts[(int64_t)blk * N + tid] = c;
    s_count[tid] = c;
  }
  __syncthreads();
}

// Bucket entries of one token block: entry (t << 3) | r for every selection, at the
// expert's base slot for this block plus the number of earlier tokens of the block that
// chose the same expert; one warp ballot per expert gives those counts. s_hit holds the
// block's ranks + 1 if `have_hits`, else they are read back from sel; the bases are in
// shared memory if `have_bases`, else read from `base` [blk][N].
__device__ void fused_bucket(const int32_t* __restrict__ sel, const int32_t* __restrict__ base,
                             int blk, int M, int N, int G, int k, int32_t* __restrict__ bucket,
                             unsigned char* s_hit, bool have_hits, bool have_bases,
                             uint8_t* scratch) {
  constexpr int kWarps = kRouteBlock / 32;
  unsigned char* s_lb = scratch;                                      // [128][N] lanes before
  int* s_base = reinterpret_cast<int*>(scratch + ((kRouteBlock * N + 15) / 16 * 16));  // [N]
  int* s_warp = s_base + N;                                           // [N][kWarps]
  const int E = N / G;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int t = blk * kRouteBlock + tid;
  if (!have_hits) {
    for (int i = tid; i < kRouteBlock * N; i += kFusedThreads) s_hit[i] = 0;
    __syncthreads();
    for (int pi = tid; pi < kRouteBlock * G; pi += kFusedThreads) {
      const int tl = pi / G, g = pi % G;
      const int tt = blk * kRouteBlock + tl;
      if (tt >= M) continue;
      for (int r = 0; r < k; ++r)
        s_hit[tl * N + g * E + __ldcg(sel + (int64_t)tt * G * k + g * k + r)] =
            (unsigned char)(r + 1);
    }
  }
  if (!have_bases && tid < N) s_base[tid] = __ldcg(base + (int64_t)blk * N + tid);
  __syncthreads();
  if (tid < kRouteBlock) {
    for (int e = 0; e < N; ++e) {
      const unsigned ball = __ballot_sync(0xffffffffu, s_hit[tid * N + e] != 0);
      s_lb[tid * N + e] = (unsigned char)__popc(ball & ((1u << lane) - 1u));
      if (lane == 0) s_warp[e * kWarps + warp] = __popc(ball);
    }
  }
  __syncthreads();
  if (tid < kRouteBlock && t < M) {
    for (int e = 0; e < N; ++e) {
      const int r1 = s_hit[tid * N + e];
      if (!r1) continue;
      int before = s_lb[tid * N + e];
      for (int w = 0; w < warp; ++w) before += s_warp[e * kWarps + w];
      bucket[s_base[e] + before] = (t << 3) | (r1 - 1);
    }
  }
  __syncthreads();
}

// The last CTA's reduction. Thread (e, c) sums a fixed run of router blocks for expert e
// (kFusedThreads / N threads per expert, loads in batches of eight); the runs combine in run
// order (probabilities in double), so the result does not depend on scheduling. Writes
// counts (the cursors' final values), mean_prob, offsets (e M), the Switch loss
//   L = (1/G) sum_g E sum_j f_{g,j} Pbar_{g,j},  f = c / (M k),  Pbar = prob_sum / M,
// and the routed-projection tiles (each expert's bucket cut into runs of 128 slots:
// (expert | rows << 8, first slot)), then zeroes the cursors.
__device__ void finalize_routing(const float* __restrict__ part_prob, int nblk, int M, int N,
                                 int G, int k, int32_t* __restrict__ cursor,
                                 int32_t* __restrict__ counts, float* __restrict__ mean_prob,
                                 int32_t* __restrict__ offsets, float* __restrict__ aux_out,
                                 int2* __restrict__ tile_list, int32_t* __restrict__ tile_count,
                                 uint8_t* st) {
  double* s_ppart = reinterpret_cast<double*>(st);                   // [kFusedThreads]
  double* s_term = s_ppart + kFusedThreads;                          // [kMaxExperts]
  int* s_cnt = reinterpret_cast<int*>(s_term + kMaxExperts);        // [kMaxExperts]
  int* s_nt = s_cnt + kMaxExperts;                                   // [kMaxExperts + 1]
  const int tid = threadIdx.x;
  const int tpe = max(1, kFusedThreads / N);
  const int e = tid / tpe, c = tid % tpe;
  const bool act = e < N;
  const int chunk = (nblk + tpe - 1) / tpe;
  const int b0 = min(nblk, c * chunk), b1 = min(nblk, b0 + chunk);
  if (act) {
    double ps = 0.0;
    for (int b = b0; b < b1; b += 8) {
      float pv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        pv[u] = b + u < b1 ? __ldcg(part_prob + (int64_t)(b + u) * N + e) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (b + u < b1) ps += (double)pv[u];
    }
    s_ppart[tid] = ps;
  }
  if (tid < N) s_cnt[tid] = __ldcg(cursor + tid);
  __syncthreads();
  if (act && c == 0) {
    double ps = 0.0;
    for (int i = 0; i < tpe; ++i) ps += s_ppart[tid + i];
    const int tot = s_cnt[e];
    counts[e] = tot;
    offsets[e] = e * M;
    mean_prob[e] = (float)(ps / M);
    s_term[e] = (double)(N / G) * ((double)tot / ((double)M * k)) * (ps / M);
    cursor[e] = 0;  // ready for the next call
  }
  __syncthreads();
  if (tid == 0) {
    int nt = 0;
    for (int x = 0; x < N; ++x) {
      s_nt[x] = nt;
      nt += (s_cnt[x] + 127) / 128;
    }
    offsets[N] = N * M;
    *tile_count = nt;
    if (aux_out != nullptr) {
      double L = 0.0;
      for (int x = 0; x < N; ++x) L += s_term[x];
      aux_out[0] = (float)(L / G);
    }
  }
  __syncthreads();
  for (int x = tid; x < N; x += kFusedThreads) {
    const int nt = (s_cnt[x] + 127) / 128;
    for (int i = 0; i < nt; ++i)
      tile_list[s_nt[x] + i] = make_int2(x | min(128, s_cnt[x] - 128 * i) << 8, x * M + i * 128);
  }
}

__global__ void __launch_bounds__(kFusedThreads)
route_fused_kernel(const float* __restrict__ logits, int M, int N, int G, int k,
                   int32_t* __restrict__ sel, float* __restrict__ psel,
                   float* __restrict__ gates, float* __restrict__ wslot,
                   int32_t* __restrict__ part_counts, float* __restrict__ part_prob,
                   int32_t* __restrict__ counts, float* __restrict__ mean_prob,
                   int32_t* __restrict__ offsets, float* __restrict__ aux_out,
                   int32_t* __restrict__ bucket, int2* __restrict__ tile_list,
                   int32_t* __restrict__ tile_count, int32_t* __restrict__ cursor,
                   int32_t* __restrict__ ticket) {
  extern __shared__ __align__(16) uint8_t dsmem[];
  __shared__ int s_last;
  pdl_wait();  // the router logits are complete from here on
  pdl_allow_next();
  float* s_p = reinterpret_cast<float*>(dsmem);                         // [128][N]
  float* s_psum = s_p + kRouteBlock * N;                                // [128][G]
  unsigned char* s_hit = reinterpret_cast<unsigned char*>(s_psum + kRouteBlock * G);  // [128][N]
  uint8_t* scratch = dsmem + ((kRouteBlock * N * 4 + kRouteBlock * G * 4 + kRouteBlock * N + 15) / 16 * 16);
  int* s_base = reinterpret_cast<int*>(scratch + ((kRouteBlock * N + 15) / 16 * 16));  // [N]
  int* s_count = reinterpret_cast<int*>(scratch + fused_bucket_bytes(N));             // [N]
  uint8_t* st = scratch + fused_bucket_bytes(N) + 4 * kMaxExperts;
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    fused_select(logits, blk, M, N, G, k, sel, psel, gates, wslot, part_counts, part_prob, s_p,
                 s_hit, s_psum, s_count);
    // claim this block's run of slots in every expert's bucket
    if (threadIdx.x < N)
      s_base[threadIdx.x] = threadIdx.x * M + atomicAdd(&cursor[threadIdx.x], s_count[threadIdx.x]);
    __syncthreads();
    fused_bucket(sel, nullptr, blk, M, N, G, k, bucket, s_hit, true, true, scratch);
  }
  // the last CTA to get here finishes the statistics
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  finalize_routing(part_prob, nblk, M, N, G, k, cursor, counts, mean_prob, offsets, aux_out,
                   tile_list, tile_count, st);
  if (threadIdx.x == 0) *ticket = 0;
}

int launch_route_fused(gqe_ctx* h, int M, float* aux_out, cudaStream_t st) {
  const int smem = fused_smem_bytes(h->N, h->G);
  // the largest size any shape can ask for, so that one setting serves every handle
  if (!set_smem_limit_once<route_fused_kernel>(fused_smem_bytes(kMaxExperts, kMaxExperts)))
    return -1;
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  const int grid = nblk < 4 * h->num_sms ? nblk : 4 * h->num_sms;
  const float* logits = h->ws.logits;
  return launch_pdl(route_fused_kernel, dim3(grid), dim3(kFusedThreads), smem, st, logits, M,
                    h->N, h->G, h->k, h->ws.sel, h->ws.psel, h->ws.gates, h->ws.w,
                    h->ws.part_counts, h->ws.part_prob, h->ws.counts, h->ws.mean_prob,
                    h->ws.offsets, aux_out, h->ws.bucket, h->ws.tile_list, h->ws.tile_count,
                    h->ws.cursor, h->ws.cursor + kMaxExperts) == cudaSuccess
             ? 1
             : -1;
}

int launch_route_select(gqe_ctx* h, int M, cudaStream_t st) {
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  route_select_kernel<<<nblk, kRouteBlock, 0, st>>>(
      h->ws.logits, M, h->N, h->G, h->k, h->ws.sel, h->ws.psel, h->ws.gates, h->ws.w,
      h->ws.part_counts, h->ws.part_prob);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_route_scan_aux(gqe_ctx* h, int M, float* aux_out, cudaStream_t st) {
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  route_scan_aux_kernel<<<1, 1024, 0, st>>>(h->ws.part_counts, h->ws.part_prob, nblk,
                                                   M, h->N, h->G, h->k, h->ws.counts,
                                                   h->ws.mean_prob, h->ws.offsets, aux_out);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_bucket(gqe_ctx* h, int M, cudaStream_t st) {
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  bucket_kernel<<<dim3(nblk, h->N), kRouteBlock, 0, st>>>(h->ws.sel, h->ws.part_counts, M,
                                                          h->N, h->G, h->k, h->ws.bucket);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace gqe
