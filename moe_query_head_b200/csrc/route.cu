// Router: per-group softmax, top-k, gates, slot weights, load statistics, expert buckets.
//
// "GQE: Grouped Query Experts" README, Algorithm Overview: a softmax over the experts of
// each GQA group, then top-k; a Switch-style load-balancing loss. gist.science summary,
// Output Construction: a renormalised weighted sum of the selected outputs using the
// router probabilities (the slot weights w below).
#include "gqe_common.cuh"

namespace gqe {

// One thread per token; the block's logits [128, N] are staged in shared memory (one
// coalesced copy) and every per-token array lives there too, so nothing spills to local
// memory. Writes sel / p_sel / gates / w [M, G, k] and this block's per-expert token
// counts and probability sums to part_counts / part_prob [blockIdx, N] (summed later in a
// fixed order, so the result does not depend on scheduling).
__global__ void __launch_bounds__(kRouteBlock)
route_select_kernel(const float* __restrict__ logits, int M, int N, int G, int k,
                    int32_t* __restrict__ sel, float* __restrict__ psel,
                    float* __restrict__ gates, float* __restrict__ wslot,
                    int32_t* __restrict__ part_counts, float* __restrict__ part_prob) {
  __shared__ float s_p[kRouteBlock][kMaxExperts + 1];          // logits, then probabilities
  __shared__ unsigned char s_hit[kRouteBlock][kMaxExperts + 1];  // selected experts
  const int E = N / G;
  const int t0 = blockIdx.x * kRouteBlock;
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
    part_prob[(int64_t)blockIdx.x * N + tid] = ps;
    part_counts[(int64_t)blockIdx.x * N + tid] = c;
  }
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
