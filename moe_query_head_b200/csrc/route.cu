// Router: per-group softmax, top-k, gates, slot weights, load statistics, expert buckets.
//
// "GQE: Grouped Query Experts" README, Algorithm Overview: a softmax over the experts of
// each GQA group, then top-k; a Switch-style load-balancing loss. gist.science summary,
// Output Construction: a renormalised weighted sum of the selected outputs using the
// router probabilities (the slot weights w below).
#include "gqe_common.cuh"

namespace gqe {

// One thread per token. Reads the fp32 logits [M, N]; writes sel / p_sel / gates / w
// [M, G, k]; writes this block's per-expert token counts and probability sums to
// part_counts / part_prob [blockIdx, N] (summed later in a fixed order, so the result
// does not depend on scheduling).
__global__ void __launch_bounds__(kRouteBlock)
route_select_kernel(const float* __restrict__ logits, int M, int N, int G, int k,
                    int32_t* __restrict__ sel, float* __restrict__ psel,
                    float* __restrict__ gates, float* __restrict__ wslot,
                    int32_t* __restrict__ part_counts, float* __restrict__ part_prob) {
  __shared__ float s_prob[kRouteBlock][kMaxExperts + 1];
  __shared__ unsigned char s_hit[kRouteBlock][kMaxExperts + 1];
  const int E = N / G;
  const int t = blockIdx.x * kRouteBlock + threadIdx.x;
  const bool valid = t < M;
  float l[kMaxExperts];
  float p_all[kMaxExperts];
  float p_tot = 0.f;
  int sel_j[kMaxExperts];    // [G][k] selected j, ascending (G*k <= N <= 64)
  float sel_p[kMaxExperts];  // [G][k] their probabilities
#pragma unroll 1
  for (int e = 0; e < N; ++e) l[e] = valid ? logits[(int64_t)t * N + e] : 0.f;
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    const float* lg = l + g * E;
    // softmax within the group, fp32 with max subtraction
    float mx = lg[0];
    for (int j = 1; j < E; ++j) mx = fmaxf(mx, lg[j]);
    float den = 0.f;
    for (int j = 0; j < E; ++j) {
      float z = expf(lg[j] - mx);
      p_all[g * E + j] = z;
      den += z;
    }
    const float inv = 1.f / den;
    for (int j = 0; j < E; ++j) p_all[g * E + j] *= inv;
    // top-k on the logits: k passes of argmax over the experts not yet taken; a strict
    // comparison keeps the lowest index among equal maxima.
    uint64_t taken = 0;
    for (int r = 0; r < k; ++r) {
      int best = -1;
      float bv = 0.f;
      for (int j = 0; j < E; ++j) {
        if (taken >> j & 1ull) continue;
        if (best < 0 || lg[j] > bv) { best = j; bv = lg[j]; }
      }
      taken |= 1ull << best;
    }
    // list the selected set in ascending expert index
    int r = 0;
    float psum = 0.f;
    for (int j = 0; j < E; ++j) {
      if (taken >> j & 1ull) {
        sel_j[g * k + r] = j;
        sel_p[g * k + r] = p_all[g * E + j];
        psum += p_all[g * E + j];
        ++r;
      }
    }
    const float ginv = 1.f / psum;
    if (valid) {
      for (int rr = 0; rr < k; ++rr) {
        const int64_t o = (int64_t)t * G * k + g * k + rr;
        sel[o] = sel_j[g * k + rr];
        psel[o] = sel_p[g * k + rr];
        gates[o] = sel_p[g * k + rr] * ginv;
      }
    }
    p_tot += psum;
  }
  const float winv = 1.f / p_tot;
  if (valid) {
    for (int s = 0; s < G * k; ++s) wslot[(int64_t)t * G * k + s] = sel_p[s] * winv;
  }
  // per-block statistics
  for (int e = 0; e < N; ++e) {
    s_prob[threadIdx.x][e] = valid ? p_all[e] : 0.f;
    s_hit[threadIdx.x][e] = 0;
  }
  if (valid) {
    for (int g = 0; g < G; ++g)
      for (int rr = 0; rr < k; ++rr) s_hit[threadIdx.x][g * E + sel_j[g * k + rr]] = 1;
  }
  __syncthreads();
  if (threadIdx.x < N) {
    const int e = threadIdx.x;
    float ps = 0.f;
    int c = 0;
    for (int i = 0; i < kRouteBlock; ++i) {
      ps += s_prob[i][e];
      c += s_hit[i][e];
    }
    part_prob[(int64_t)blockIdx.x * N + e] = ps;
    part_counts[(int64_t)blockIdx.x * N + e] = c;
  }
}

// One block of kMaxExperts threads. Sums the per-block statistics in block order (double
// accumulation), writes counts / mean_prob / the bucket offsets, turns part_counts into
// each (block, expert)'s first bucket slot, and computes the Switch loss
//   L = (1/G) sum_g E sum_j f_{g,j} Pbar_{g,j},  f = c / (M k),  Pbar = prob_sum / M.
__global__ void route_scan_aux_kernel(int32_t* __restrict__ part_counts,
                                      const float* __restrict__ part_prob, int nblk, int M,
                                      int N, int G, int k, int32_t* __restrict__ counts,
                                      float* __restrict__ mean_prob,
                                      int32_t* __restrict__ offsets, float* __restrict__ aux_out) {
  __shared__ int s_cnt[kMaxExperts];
  __shared__ double s_term[kMaxExperts];
  const int e = threadIdx.x;
  int c = 0;
  double ps = 0.0;
  if (e < N) {
    for (int b = 0; b < nblk; ++b) {
      c += part_counts[(int64_t)b * N + e];
      ps += (double)part_prob[(int64_t)b * N + e];
    }
    counts[e] = c;
    mean_prob[e] = (float)(ps / M);
    s_cnt[e] = c;
    const int E = N / G;
    s_term[e] = (double)E * ((double)c / ((double)M * k)) * (ps / M);
  }
  __syncthreads();
  if (e < N) {
    int off = 0;
    for (int i = 0; i < e; ++i) off += s_cnt[i];
    offsets[e] = off;
    if (e == N - 1) offsets[N] = off + s_cnt[e];
    // exclusive scan over blocks: first slot of (block b, expert e)
    int run = off;
    for (int b = 0; b < nblk; ++b) {
      const int v = part_counts[(int64_t)b * N + e];
      part_counts[(int64_t)b * N + e] = run;
      run += v;
    }
  }
  if (e == 0 && aux_out != nullptr) {
    double L = 0.0;
    for (int i = 0; i < N; ++i) L += s_term[i];
    aux_out[0] = (float)(L / G);
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

int launch_route_select(gqe_ctx* h, int M, cudaStream_t st) {
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  route_select_kernel<<<nblk, kRouteBlock, 0, st>>>(
      h->ws.logits, M, h->N, h->G, h->k, h->ws.sel, h->ws.psel, h->ws.gates, h->ws.w,
      h->ws.part_counts, h->ws.part_prob);
  return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

int launch_route_scan_aux(gqe_ctx* h, int M, float* aux_out, cudaStream_t st) {
  const int nblk = (M + kRouteBlock - 1) / kRouteBlock;
  route_scan_aux_kernel<<<1, kMaxExperts, 0, st>>>(h->ws.part_counts, h->ws.part_prob, nblk,
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
