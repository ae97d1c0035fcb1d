// C ABI of the GQE attention library (forward, decode step, group range): argument checks,
// the workspace, and the launch sequence on the caller's stream. The backward pass's entry
// points are in backward.cu. The layer it computes is the one described in
// "GQE: Grouped Query Experts" (FrontiersMindAI/GQE README, Algorithm Overview and
// Parameters) with the output construction of the gist.science summary (Methodology,
// Output Construction).
#include <stdlib.h>
#include <string.h>

#include <new>

#include "gqe_common.cuh"

using namespace gqe;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool head_dim_ok(int d_h) { return d_h >= 16 && d_h <= 128 && d_h % 16 == 0; }

gqe_status check_shape(int dim, int N, int G, int k, int d_h, int dtype, int64_t max_tokens) {
  if (dim < 16 || N < 1 || G < 1 || k < 1 || d_h < 1 || max_tokens < 1)
    return GQE_ERR_INVALID_ARG;
  if (N % G != 0) return GQE_ERR_INVALID_ARG;  // README Parameters: N divisible by G
  const int E = N / G;
  if (k > E) return GQE_ERR_INVALID_ARG;
  if (dtype != GQE_BF16 && dtype != GQE_F32) return GQE_ERR_INVALID_ARG;
  if (N > kMaxExperts || k > kMaxTopK) return GQE_ERR_UNSUPPORTED;
  if (!head_dim_ok(d_h)) return GQE_ERR_UNSUPPORTED;
  if (dim % 16 != 0) return GQE_ERR_UNSUPPORTED;
  if (max_tokens > (int64_t(1) << 27)) return GQE_ERR_UNSUPPORTED;  // (t << 3) in int32
  return GQE_OK;
}

// Lays out the workspace; with base == nullptr only computes the size.
size_t layout(Workspace& w, char* base, int dim, int N, int G, int k, int d_h, int esz,
              int64_t M) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const int64_t S = (int64_t)G * k + 1;
  const int64_t Do = ((int64_t)G * k + 2) * d_h;
  const int64_t nblk = (M + kRouteBlock - 1) / kRouteBlock;
  const int64_t Gk = (int64_t)G * k;
  w.K = take((size_t)G * M * d_h * esz);
  w.V = take((size_t)G * M * d_h * esz);
  w.Q = take((size_t)S * M * d_h * esz);
  w.Z = take((size_t)M * Do * esz);
  w.lse = (float*)take((size_t)S * M * 4);
  w.logits = (float*)take((size_t)M * N * 4);
  w.sel = (int32_t*)take((size_t)M * Gk * 4);
  w.psel = (float*)take((size_t)M * Gk * 4);
  w.gates = (float*)take((size_t)M * Gk * 4);
  w.w = (float*)take((size_t)M * Gk * 4);
  w.part_counts = (int32_t*)take((size_t)nblk * N * 4);
  w.part_prob = (float*)take((size_t)nblk * N * 4);
  w.counts = (int32_t*)take((size_t)N * 4);
  w.mean_prob = (float*)take((size_t)N * 4);
  w.offsets = (int32_t*)take((size_t)(N + 1) * 4);
  w.bucket = (int32_t*)take((size_t)M * N * 4);  // expert e owns slots [e M, (e + 1) M)
  w.tile_list = (int2*)take((size_t)((M * Gk + 127) / 128 + N + 1) * sizeof(int2));
  w.tile_count = (int32_t*)take(16);
  w.attn_counter = (int32_t*)take(16);
  w.cursor = (int32_t*)take((kMaxExperts + 4) * 4);
  w.rcur = (int32_t*)take((kRouteFlag + 2) * 4);
  w.rpsum = (unsigned long long*)take(2 * kMaxExperts * 8);
  w.dec_part = (float*)take((size_t)kDecodeSlots * (k + 1) * (d_h + 2) * 4);
  w.status = (int32_t*)take(16);
  (void)dim;
  return off;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A call that launched the dense projection's routing but not the routed projection leaves
// a cursor set written and the set flag unflipped: both sets and the flag go back to zero so
// the next call starts clean.
void reset_route_sets(gqe_ctx* h, cudaStream_t st) {
  cudaMemsetAsync(h->ws.rcur, 0, (kRouteFlag + 2) * sizeof(int32_t), st);
  cudaMemsetAsync(h->ws.rpsum, 0, 2 * kMaxExperts * sizeof(unsigned long long), st);
}

}  // namespace

extern "C" {

const char* gqe_status_str(int s) {
  switch (s) {
    case GQE_OK: return "GQE_OK";
    case GQE_ERR_INVALID_ARG: return "GQE_ERR_INVALID_ARG: invalid argument";
    case GQE_ERR_UNSUPPORTED: return "GQE_ERR_UNSUPPORTED: shape not supported by this build";
    case GQE_ERR_WORKSPACE: return "GQE_ERR_WORKSPACE: B*T exceeds the handle's max_tokens";
    case GQE_ERR_CUDA: return "GQE_ERR_CUDA: a CUDA call failed";
    case GQE_ERR_TIMEOUT: return "GQE_ERR_TIMEOUT: a device-side wait gave up";
    default: return "unknown gqe_status";
  }
}

int64_t gqe_workspace_bytes(int dim, int N, int G, int k, int d_h, gqe_dtype dtype,
                            int64_t max_tokens) {
  if (check_shape(dim, N, G, k, d_h, dtype, max_tokens) != GQE_OK) return -1;
  Workspace w;
  return (int64_t)layout(w, nullptr, dim, N, G, k, d_h, dtype == GQE_F32 ? 4 : 2, max_tokens);
}

gqe_status gqe_create(gqe_handle* out, int dim, int N, int G, int k, int d_h, gqe_dtype dtype,
                      int64_t max_tokens) {
  if (!out) return GQE_ERR_INVALID_ARG;
  *out = nullptr;
  gqe_status st = check_shape(dim, N, G, k, d_h, dtype, max_tokens);
  if (st != GQE_OK) return st;
  gqe_ctx* h = new (std::nothrow) gqe_ctx();
  if (!h) return GQE_ERR_CUDA;
  h->dim = dim;
  h->N = N;
  h->G = G;
  h->k = k;
  h->d_h = d_h;
  h->E = N / G;
  h->g0 = 0;
  h->g1 = G;
  h->dtype = dtype;
  h->max_tokens = max_tokens;
  h->esz = dtype == GQE_F32 ? 4 : 2;
  h->spin_limit = 0;
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) !=
          cudaSuccess) {
    delete h;
    return GQE_ERR_CUDA;
  }
  const size_t bytes = layout(h->ws, nullptr, dim, N, G, k, d_h, h->esz, max_tokens);
  void* base = nullptr;
  if (cudaMalloc(&base, bytes) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return GQE_ERR_CUDA;
  }
  layout(h->ws, static_cast<char*>(base), dim, N, G, k, d_h, h->esz, max_tokens);
  h->ws.base = base;
  h->ws.bytes = bytes;
  // Everything starts at zero: counters, the status word, and index arrays (so no stale
  // value can ever name a token or expert outside the current call's range).
  if (cudaMemset(base, 0, bytes) != cudaSuccess) {
    cudaFree(base);
    delete h;
    return GQE_ERR_CUDA;
  }
  *out = h;
  return GQE_OK;
}

void gqe_destroy(gqe_handle h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaFree(h->ws.base);
  backward_release(h);
  delete h;
}

gqe_status gqe_set_group_range(gqe_handle h, int g0, int g1) {
  if (!h || g0 < 0 || g1 > h->G || g0 >= g1) return GQE_ERR_INVALID_ARG;
  // a part of the layer needs the routing inside the dense projection (it routes every
  // group, so slot weights and the aux loss stay the whole layer's)
  if ((g0 != 0 || g1 != h->G) && !(h->dtype == GQE_BF16 && tc_dense_routes(h)))
    return GQE_ERR_UNSUPPORTED;
  h->g0 = g0;
  h->g1 = g1;
  return GQE_OK;
}

gqe_status gqe_set_spin_limit(gqe_handle h, int64_t limit) {
  if (!h || limit < 0) return GQE_ERR_INVALID_ARG;
  h->spin_limit = limit;
  return GQE_OK;
}

int gqe_kernel_launches(gqe_handle h) { return h ? h->last_launches : -1; }

gqe_status gqe_set_stage_events(gqe_handle h, void* const* events, int count) {
  if (!h) return GQE_ERR_INVALID_ARG;
  if (count == 0) {
    h->n_stage_events = 0;
    return GQE_OK;
  }
  if (count != GQE_NUM_STAGES + 1 || !events) return GQE_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!events[i]) return GQE_ERR_INVALID_ARG;
    h->stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  h->n_stage_events = count;
  return GQE_OK;
}

const char* gqe_stage_name(int i) {
  static const char* names[GQE_NUM_STAGES] = {"dense_proj", "route", "qproj",
                                               "attention", "combine", "oproj"};
  return (i >= 0 && i < GQE_NUM_STAGES) ? names[i] : nullptr;
}

gqe_status gqe_forward(gqe_handle h, const void* x, int B, int T, const void* W_r,
                       const void* W_q, const void* W_k, const void* W_v, const void* W_shared,
                       const void* W_o, int N, int G, int k, int d_h, int variant, int causal,
                       void* out, float* aux_loss, void* stream) {
  if (!h) return GQE_ERR_INVALID_ARG;
  if (N != h->N || G != h->G || k != h->k || d_h != h->d_h) return GQE_ERR_INVALID_ARG;
  if (B < 1 || T < 1) return GQE_ERR_INVALID_ARG;
  if (variant < GQE_VARIANT_GQE || variant > GQE_VARIANT_HARD_CONCAT) return GQE_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return GQE_ERR_INVALID_ARG;
  if (!x || !W_r || !W_q || !W_k || !W_v || !W_o || !out) return GQE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_r, W_q, W_k, W_v, W_o, out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GQE_ERR_INVALID_ARG;
  if (W_shared && !aligned16(W_shared)) return GQE_ERR_INVALID_ARG;
  if (aux_loss && (reinterpret_cast<uintptr_t>(aux_loss) & 3u)) return GQE_ERR_INVALID_ARG;
  // the shared head reads KV head 0: only the group range that holds group 0 computes it
  if (W_shared && h->g0 != 0) return GQE_ERR_INVALID_ARG;
  const int64_t M64 = (int64_t)B * T;
  if (M64 > h->max_tokens) return GQE_ERR_WORKSPACE;
  const int M = (int)M64;
  const int has_shared = W_shared != nullptr;
  const int Gl = h->g1 - h->g0;  // the groups this handle computes
  const int S = Gl * k + has_shared;
  const int Do = (Gl * k + (variant == GQE_VARIANT_GQE ? 1 : 0) + has_shared) * d_h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  int launches = 0;
  int stage = 0;
  auto add = [&](int n) -> bool {
    if (h->n_stage_events) cudaEventRecord(h->stage_events[stage], st);
    ++stage;
    if (n < 0) return false;
    launches += n;
    return true;
  };
  auto mark = [&]() {
    if (h->n_stage_events) cudaEventRecord(h->stage_events[stage], st);
    ++stage;
    return true;
  };
  // mark() records stage event 0; each add() records the next event after its stage's
  // launches (the arguments are evaluated first), so event i precedes stage i.
  // bf16: tensor-core (tcgen05) kernels for the projections; fp32: CUDA-core kernels.
  const bool tc = h->dtype == GQE_BF16;
  // bf16 with N a power of two up to 32: the routing runs in the dense projection's router
  // tiles, and the routed projection schedules from its cursors (the two cursor sets
  // alternate between calls on a flag the kernels keep in device memory, so the call can be
  // captured in a CUDA graph and replayed)
  const bool fused = tc && tc_dense_routes(h);
  int dense = -1;
  bool ok = mark() &&
            add(dense = tc ? launch_tc_dense_proj(h, x, M, W_r, W_k, W_v, W_shared, st)
                           : launch_simt_dense_proj(h, x, M, W_r, W_k, W_v, W_shared, st)) &&
            add(fused ? 0 : launch_route_fused(h, M, aux_loss, st)) &&
            add(tc ? launch_tc_qproj(h, x, M, W_q, fused, aux_loss, st)
                   : launch_simt_qproj(h, x, M, W_q, st)) &&
            add(tc ? launch_tc_attention(h, B, T, S, has_shared, variant, causal, Do, st)
                   : launch_simt_attention(h, B, T, S, has_shared, variant, causal, Do, st)) &&
            add(launch_combine(h, M, variant, Do, st)) &&
            add(tc ? launch_tc_oproj(h, M, Do, W_o, out, st)
                   : launch_simt_oproj(h, M, Do, W_o, out, st));
  if (fused && dense >= 0 && !ok) reset_route_sets(h, st);
  h->last_M = M;
  h->last_S = S;
  h->last_Do = Do;
  h->last_launches = launches;
  h->last_kind = ok ? 1 : 0;
  h->last_B = B;
  h->last_T = T;
  h->last_variant = variant;
  h->last_causal = causal;
  h->last_shared = has_shared;
  h->last_g0 = h->g0;
  h->last_g1 = h->g1;
  h->bwd_begun = 0;
  return ok ? GQE_OK : GQE_ERR_CUDA;
}

gqe_status gqe_decode(gqe_handle h, const void* x, int B, void* k_cache, void* v_cache,
                      int L_max, const int32_t* lengths, const void* W_r, const void* W_q,
                      const void* W_k, const void* W_v, const void* W_shared, const void* W_o,
                      int N, int G, int k, int d_h, int variant, void* out, float* aux_loss,
                      void* stream) {
  if (!h) return GQE_ERR_INVALID_ARG;
  if (N != h->N || G != h->G || k != h->k || d_h != h->d_h) return GQE_ERR_INVALID_ARG;
  if (B < 1 || L_max < 1) return GQE_ERR_INVALID_ARG;
  if (variant < GQE_VARIANT_GQE || variant > GQE_VARIANT_HARD_CONCAT) return GQE_ERR_INVALID_ARG;
  if (!x || !W_r || !W_q || !W_k || !W_v || !W_o || !out || !k_cache || !v_cache || !lengths)
    return GQE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W_r, W_q, W_k, W_v, W_o, out, k_cache, v_cache};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GQE_ERR_INVALID_ARG;
  if (W_shared && !aligned16(W_shared)) return GQE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lengths) & 3u) return GQE_ERR_INVALID_ARG;
  if (aux_loss && (reinterpret_cast<uintptr_t>(aux_loss) & 3u)) return GQE_ERR_INVALID_ARG;
  if (h->dtype != GQE_BF16) return GQE_ERR_UNSUPPORTED;
  // the shared head reads KV head 0: only the group range that holds group 0 computes it
  if (W_shared && h->g0 != 0) return GQE_ERR_INVALID_ARG;
  if (B > 65535) return GQE_ERR_UNSUPPORTED;  // one grid row per sequence
  if (B > h->max_tokens) return GQE_ERR_WORKSPACE;
  const int M = B;
  const int has_shared = W_shared != nullptr;
  const int Gl = h->g1 - h->g0;  // the groups this handle computes (their caches)
  const int S = Gl * k + has_shared;
  const int Do = (Gl * k + (variant == GQE_VARIANT_GQE ? 1 : 0) + has_shared) * d_h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  int launches = 0;
  int stage = 0;
  auto add = [&](int n) -> bool {
    if (h->n_stage_events) cudaEventRecord(h->stage_events[stage], st);
    ++stage;
    if (n < 0) return false;
    launches += n;
    return true;
  };
  auto mark = [&]() {
    if (h->n_stage_events) cudaEventRecord(h->stage_events[stage], st);
    ++stage;
    return true;
  };
  // the forward's stages on the B new tokens, with the cache attention in place of the
  // prefill attention
  const bool fused = tc_dense_routes(h);
  int dense = -1;
  bool ok = mark() &&
            add(dense = launch_tc_dense_proj(h, x, M, W_r, W_k, W_v, W_shared, st)) &&
            add(fused ? 0 : launch_route_fused(h, M, aux_loss, st)) &&
            add(launch_tc_qproj(h, x, M, W_q, fused, aux_loss, st)) &&
            add(launch_tc_decode_attention(h, B, S, has_shared, variant, Do, k_cache, v_cache,
                                           L_max, lengths, st)) &&
            add(0) &&  // the combine (gqe slot) runs in the cache attention's finish kernel
            add(launch_tc_oproj(h, M, Do, W_o, out, st));
  if (fused && dense >= 0 && !ok) reset_route_sets(h, st);
  h->last_M = M;
  h->last_S = S;
  h->last_Do = Do;
  h->last_launches = launches;
  h->last_kind = ok ? 2 : 0;
  h->bwd_begun = 0;
  return ok ? GQE_OK : GQE_ERR_CUDA;
}

gqe_status gqe_get_routing(gqe_handle h, int32_t* sel, float* gates, int32_t* counts,
                           float* mean_prob, void* stream) {
  if (!h || h->last_M == 0) return GQE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t mgk = (size_t)h->last_M * h->G * h->k;
  cudaError_t e = cudaSuccess;
  if (sel && e == cudaSuccess)
    e = cudaMemcpyAsync(sel, h->ws.sel, mgk * 4, cudaMemcpyDeviceToDevice, st);
  if (gates && e == cudaSuccess)
    e = cudaMemcpyAsync(gates, h->ws.gates, mgk * 4, cudaMemcpyDeviceToDevice, st);
  if (counts && e == cudaSuccess)
    e = cudaMemcpyAsync(counts, h->ws.counts, (size_t)h->N * 4, cudaMemcpyDeviceToDevice, st);
  if (mean_prob && e == cudaSuccess)
    e = cudaMemcpyAsync(mean_prob, h->ws.mean_prob, (size_t)h->N * 4, cudaMemcpyDeviceToDevice,
                        st);
  return e == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}

gqe_status gqe_get_tensor(gqe_handle h, int which, void* dst, size_t bytes, void* stream) {
  if (!h || !dst || h->last_M == 0) return GQE_ERR_INVALID_ARG;
  const size_t M = (size_t)h->last_M;
  const void* src = nullptr;
  size_t n = 0;
  switch (which) {
    case GQE_T_K: src = h->ws.K; n = (size_t)(h->g1 - h->g0) * M * h->d_h * h->esz; break;
    case GQE_T_V: src = h->ws.V; n = (size_t)(h->g1 - h->g0) * M * h->d_h * h->esz; break;
    case GQE_T_Q: src = h->ws.Q; n = (size_t)h->last_S * M * h->d_h * h->esz; break;
    case GQE_T_Z: src = h->ws.Z; n = M * h->last_Do * h->esz; break;
    case GQE_T_PSEL: src = h->ws.psel; n = M * h->G * h->k * 4; break;
    case GQE_T_W: src = h->ws.w; n = M * h->G * h->k * 4; break;
    case GQE_T_LOGITS: src = h->ws.logits; n = M * h->N * 4; break;
    default: return GQE_ERR_INVALID_ARG;
  }
  if (bytes < n) return GQE_ERR_INVALID_ARG;
  // Q: the shared stream sits at index G*k of an S-stream buffer sized for G*k+1.
  return cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToDevice,
                         static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GQE_OK
             : GQE_ERR_CUDA;
}

gqe_status gqe_check_device_status(gqe_handle h, void* stream) {
  if (!h) return GQE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return GQE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, h->ws.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return GQE_ERR_CUDA;
  if (v != kStatusOk) {
    cudaMemset(h->ws.status, 0, 4);
    return v == kStatusBadInput ? GQE_ERR_INVALID_ARG
           : v == kStatusBadState ? GQE_ERR_CUDA
                                  : GQE_ERR_TIMEOUT;
  }
  return GQE_OK;
}

}  // extern "C"
