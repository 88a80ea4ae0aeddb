// api.cu -- the extern "C" boundary of libkvscan: argument checks on the host
// (nothing is launched or written when a check fails), workspace carving, and
// the launches, all on the caller's stream. No allocation, no synchronisation.
#include <cstring>

#include "internal.cuh"
#include "scan_core.cuh"

namespace kvs {

namespace {
thread_local char g_err[512] = "";
}

kvs_status fail(kvs_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

const char* g_err_text() { return g_err; }

kvs_status ok() {
  g_err[0] = 0;
  return KVS_OK;
}

kvs_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVS_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return KVS_OK;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = v > 0 ? v : 148;
  }
  return cached[dev];
}

}  // namespace kvs

using namespace kvs;

namespace {

kvs_status check_index(const kvs_fathom_index* ix, int n_max) {
  KVS_REQUIRE(ix != nullptr, KVS_EINVAL, "index descriptor is null");
  KVS_REQUIRE(ix->planes && ix->kmin && ix->kstep && ix->kvar, KVS_EINVAL,
              "index: planes/kmin/kstep/kvar must be non-null");
  KVS_REQUIRE(ix->R >= 1 && ix->G >= 1, KVS_EINVAL, "index: R=%d G=%d", ix->R, ix->G);
  KVS_REQUIRE(ix->D == kD, KVS_EUNSUPPORTED, "index: head dim D=%d (only 128 is built)", ix->D);
  KVS_REQUIRE(ix->W >= 4 && ix->W % 4 == 0, KVS_EINVAL,
              "index: W=%d words per plane must be a positive multiple of 4", ix->W);
  KVS_REQUIRE(static_cast<int64_t>(ix->W) * 32 >= n_max, KVS_EINVAL,
              "index: W=%d words hold %d keys < n_max=%d", ix->W, ix->W * 32, n_max);
  KVS_REQUIRE(aligned16(ix->planes), KVS_EINVAL, "index: planes must be 16-byte aligned");
  return KVS_OK;
}

kvs_status check_plan(const kvs_plan* plan, int D) {
  KVS_REQUIRE(plan != nullptr, KVS_EINVAL, "plan descriptor is null");
  KVS_REQUIRE(plan->B >= 0 && plan->B <= 4 * D, KVS_EINVAL, "bit budget B=%d outside 0..%d",
              plan->B, 4 * D);
  KVS_REQUIRE(plan->t && plan->C && (plan->B == 0 || (plan->plane_idx && plan->plane_w)),
              KVS_EINVAL, "plan: t/plane_idx/plane_w/C must be non-null");
  return KVS_OK;
}

}  // namespace

extern "C" {

int32_t kvs_abi_version(void) { return KVS_ABI_VERSION; }

const char* kvs_last_error(void) { return kvs::g_err_text(); }

size_t kvs_build_index_workspace_size(int32_t R, int32_t G, int32_t D) {
  return build_index_ws_bytes(R, G, D);
}

kvs_status kvs_build_fathom_index(const uint16_t* K, const int32_t* n, int32_t R, int32_t G,
                                  int32_t n_max, int32_t D, int32_t W, uint32_t* planes,
                                  float* kmin, float* kstep, float* kvar, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream) {
  (void)dev_status;
  KVS_REQUIRE(K && n && planes && kmin && kstep && kvar, KVS_EINVAL,
              "build_fathom_index: null pointer argument");
  KVS_REQUIRE(R >= 1 && G >= 1 && n_max >= 0, KVS_EINVAL, "build_fathom_index: R=%d G=%d n_max=%d",
              R, G, n_max);
  KVS_REQUIRE(D == kD, KVS_EUNSUPPORTED, "build_fathom_index: D=%d (only 128 is built)", D);
  KVS_REQUIRE(W >= 4 && W % 4 == 0 && static_cast<int64_t>(W) * 32 >= n_max, KVS_EINVAL,
              "build_fathom_index: W=%d must be a multiple of 4 with 32*W >= n_max=%d", W, n_max);
  KVS_REQUIRE(aligned16(K) && aligned16(planes), KVS_EINVAL,
              "build_fathom_index: K and planes must be 16-byte aligned");
  KVS_REQUIRE(ws && ws_bytes >= build_index_ws_bytes(R, G, D), KVS_EWORKSPACE,
              "build_fathom_index: workspace %zu < %zu bytes", ws_bytes,
              build_index_ws_bytes(R, G, D));
  kvs_status st = build_index_launch(K, n, R, G, n_max, W, planes, kmin, kstep, kvar, ws,
                                     static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

kvs_status fathom_plan_bits(const float* q, int32_t H, const kvs_fathom_index* ix, int32_t B,
                            const kvs_plan* plan, int32_t* dev_status, void* stream) {
  (void)dev_status;
  KVS_REQUIRE(q != nullptr, KVS_EINVAL, "fathom_plan_bits: q is null");
  KVS_REQUIRE(H >= 1 && H <= 8, KVS_EINVAL, "fathom_plan_bits: H=%d (1..8)", H);
  kvs_status st = check_index(ix, 0);
  if (st != KVS_OK) return st;
  st = check_plan(plan, ix->D);
  if (st != KVS_OK) return st;
  KVS_REQUIRE(plan->B == B, KVS_EINVAL, "fathom_plan_bits: B=%d but plan->B=%d", B, plan->B);
  st = plan_bits_launch(q, H, ix->kmin, ix->kstep, ix->kvar, ix->R * ix->G, B, plan->t,
                        plan->plane_idx, plan->plane_w, plan->C, static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

kvs_status index_scan(const kvs_scan_args* a, float* scores, int32_t* dev_status, void* stream) {
  KVS_REQUIRE(a != nullptr && scores != nullptr, KVS_EINVAL, "index_scan: null argument");
  KVS_REQUIRE(a->n != nullptr && a->R >= 1 && a->n_max >= 0, KVS_EINVAL,
              "index_scan: n must be non-null, R >= 1, n_max >= 0");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->kind == KVS_SCAN_FATHOM) {
    kvs_status st = check_index(a->ix, a->n_max);
    if (st != KVS_OK) return st;
    st = check_plan(a->plan, a->ix->D);
    if (st != KVS_OK) return st;
    KVS_REQUIRE(a->ix->R == a->R, KVS_EINVAL, "index_scan: index R=%d != R=%d", a->ix->R, a->R);
    st = fathom_scan_dispatch(a->ix, a->plan, a->n, a->n_max, scores, dev_status, s);
    return st == KVS_OK ? ok() : st;
  }
  if (a->kind == KVS_SCAN_LIGHTNING) {
    kvs_status st = lightning_scan_dispatch(a, scores, dev_status, s);
    return st == KVS_OK ? ok() : st;
  }
  return fail(KVS_EINVAL, "index_scan: unknown kind %d", a->kind);
}

kvs_status kvs_selftest_scan_timeout(const kvs_fathom_index* ix, const kvs_plan* plan, const int32_t* n,
                                     int32_t n_max, float* scores, int64_t wait_cycles,
                                     int32_t* dev_status, void* stream) {
  kvs_status st = check_index(ix, n_max);
  if (st != KVS_OK) return st;
  st = check_plan(plan, ix->D);
  if (st != KVS_OK) return st;
  KVS_REQUIRE(n && scores && dev_status && n_max >= 1, KVS_EINVAL,
              "kvs_selftest_scan_timeout: n, scores and dev_status are required, n_max >= 1");
  KVS_REQUIRE(!ix->host_mapped && plan->B >= 1 && plan->B <= 144, KVS_EUNSUPPORTED,
              "kvs_selftest_scan_timeout: an index in HBM and a plan of 1..144 planes");
  KVS_REQUIRE(wait_cycles >= 1000 && wait_cycles <= 2000000000LL, KVS_EINVAL,
              "kvs_selftest_scan_timeout: wait_cycles=%lld (1e3 .. 2e9)", static_cast<long long>(wait_cycles));
  ScanParams p{};
  p.planes = ix->planes;
  p.W = ix->W;
  p.RG = ix->R * ix->G;
  p.Gheads = ix->G;
  p.plane_idx = plan->plane_idx;
  p.plane_w = plan->plane_w;
  p.C = plan->C;
  p.B = plan->B;
  p.n = n;
  p.n_max = n_max;
  scan_schedule(plan->B, p.G, p.b, p.nsets);
  p.scores = scores;
  p.dev_status = dev_status;
  p.wait_cycles = wait_cycles;
  p.withhold_arrive = 1;
  st = fathom_scan_lut_launch(p, static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

size_t kvs_topk_workspace_size(int32_t R, int32_t G, int32_t n_max, int32_t k, int32_t block) {
  return topk_ws_bytes(R, G, n_max, k, block);
}

kvs_status topk_select(const float* scores, int64_t ld, const int32_t* n, int32_t R, int32_t G,
                       int32_t k, int32_t block, int32_t* idx, float* vals, void* ws,
                       size_t ws_bytes, int32_t* dev_status, void* stream) {
  (void)dev_status;
  (void)ws;
  KVS_REQUIRE(scores && n && idx, KVS_EINVAL, "topk_select: null pointer argument");
  KVS_REQUIRE(R >= 1 && G >= 1 && k >= 1 && ld >= 1, KVS_EINVAL,
              "topk_select: R=%d G=%d k=%d ld=%lld", R, G, k, static_cast<long long>(ld));
  KVS_REQUIRE(block == 1 || (block > 1 && block <= 1024 && k % block == 0), KVS_EINVAL,
              "topk_select: block=%d must be 1, or divide k=%d", block, k);
  KVS_REQUIRE(ws_bytes >= topk_ws_bytes(R, G, static_cast<int>(ld), k, block), KVS_EWORKSPACE,
              "topk_select: workspace too small");
  kvs_status st = topk_launch(scores, ld, n, R, G, k, block, idx, vals, static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

kvs_status sparse_gather(const int32_t* idx, int32_t k, const int32_t* slot_map,
                         const uint16_t* hotK, const uint16_t* hotV, int32_t S,
                         const uint16_t* fullK, const uint16_t* fullV, const int32_t* n,
                         int32_t n_max, int32_t R, int32_t G, int32_t D, uint16_t* gK,
                         uint16_t* gV, int32_t* slots, int32_t* misses, int32_t* dev_status,
                         void* stream) {
  (void)dev_status;
  (void)n;
  KVS_REQUIRE(idx && slot_map && hotK && hotV && fullK && fullV && gK && gV && slots && misses,
              KVS_EINVAL, "sparse_gather: null pointer argument");
  KVS_REQUIRE(R >= 1 && G >= 1 && k >= 1 && S >= 1 && n_max >= 1, KVS_EINVAL,
              "sparse_gather: R=%d G=%d k=%d S=%d n_max=%d", R, G, k, S, n_max);
  KVS_REQUIRE(D == kD, KVS_EUNSUPPORTED, "sparse_gather: D=%d (only 128 is built)", D);
  KVS_REQUIRE(aligned16(hotK) && aligned16(hotV) && aligned16(fullK) && aligned16(fullV) &&
                  aligned16(gK) && aligned16(gV),
              KVS_EINVAL, "sparse_gather: K/V buffers must be 16-byte aligned");
  kvs_status st = sparse_gather_launch(idx, k, slot_map, hotK, hotV, S, fullK, fullV, n_max, R * G,
                                       gK, gV, slots, misses, static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

kvs_status kvs_append_token(const uint16_t* Knew, const uint16_t* Vnew, int32_t* n, int32_t R,
                            int32_t G, int32_t D, int32_t n_max, uint32_t* planes, int32_t W,
                            const float* kmin, const float* kstep, uint16_t* fullK, uint16_t* fullV,
                            int32_t* slot_map, const int32_t* hot_slot, int32_t* hot_tok,
                            uint16_t* hotK, uint16_t* hotV, int32_t S, int32_t* dev_status,
                            void* stream) {
  KVS_REQUIRE(Knew && Vnew && n && planes && kmin && kstep && fullK && fullV, KVS_EINVAL,
              "kvs_append_token: null pointer argument");
  KVS_REQUIRE(R >= 1 && G >= 1 && G <= 8 && n_max >= 1, KVS_EINVAL,
              "kvs_append_token: R=%d G=%d (1..8) n_max=%d", R, G, n_max);
  KVS_REQUIRE(D == kD, KVS_EUNSUPPORTED, "kvs_append_token: D=%d (only 128 is built)", D);
  KVS_REQUIRE(W >= 4 && W % 4 == 0 && 32LL * W >= n_max, KVS_EINVAL,
              "kvs_append_token: W=%d must be a multiple of 4 with 32*W >= n_max=%d", W, n_max);
  KVS_REQUIRE(!hot_slot || (slot_map && hot_tok && hotK && hotV && S >= 1), KVS_EINVAL,
              "kvs_append_token: hot_slot needs slot_map, hot_tok, hotK, hotV and S >= 1");
  kvs_status st = append_token_launch(Knew, Vnew, n, R, G, n_max, planes, W, kmin, kstep, fullK, fullV,
                                      slot_map, hot_slot, hot_tok, hotK, hotV, S, dev_status,
                                      static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

size_t kvs_attn_workspace_size(int32_t R, int32_t G, int32_t H, int32_t k) {
  return attn_ws_bytes(R * G, H, k);
}

kvs_status sparse_decode_attn(const void* q, int32_t q_dtype, const uint16_t* K,
                              const uint16_t* V, const int32_t* k_eff, int32_t R, int32_t G,
                              int32_t H, int32_t D, int32_t k, float scale, float* out,
                              float* lse, void* ws, size_t ws_bytes, int32_t* dev_status,
                              void* stream) {
  (void)dev_status;
  KVS_REQUIRE(q && K && V && out, KVS_EINVAL, "sparse_decode_attn: null pointer argument");
  KVS_REQUIRE(q_dtype == KVS_F32 || q_dtype == KVS_BF16, KVS_EINVAL,
              "sparse_decode_attn: q_dtype=%d", q_dtype);
  KVS_REQUIRE(R >= 1 && G >= 1 && k >= 1 && H >= 1 && H <= 8, KVS_EINVAL,
              "sparse_decode_attn: R=%d G=%d H=%d k=%d", R, G, H, k);
  KVS_REQUIRE(D == kD, KVS_EUNSUPPORTED, "sparse_decode_attn: D=%d (only 128 is built)", D);
  KVS_REQUIRE(aligned16(K) && aligned16(V) && aligned16(out), KVS_EINVAL,
              "sparse_decode_attn: K, V and out must be 16-byte aligned");
  const size_t need = attn_ws_bytes(R * G, H, k);
  KVS_REQUIRE(need == 0 || (ws && ws_bytes >= need), KVS_EWORKSPACE,
              "sparse_decode_attn: workspace %zu < %zu bytes", ws_bytes, need);
  RowSrc src{};
  src.mode = kRowsStaged;
  src.K = K;
  src.V = V;
  src.k_eff = k_eff;
  src.G = G;
  src.k = k;
  kvs_status st = attn_launch(q, q_dtype == KVS_BF16, src, R * G, H, scale, out, lse, ws,
                              static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}

size_t kvs_decode_step_workspace_size_host(int32_t R, int32_t G, int32_t H, int32_t n_max, int32_t k,
                                           int32_t B) {
  return decode_ws_bytes_host(R, G, H, n_max, k, B);
}

size_t kvs_decode_step_workspace_size(int32_t R, int32_t G, int32_t H, int32_t n_max, int32_t k,
                                      int32_t B) {
  return decode_ws_bytes(R, G, H, n_max, k, B);
}

static kvs_status decode_step_checked(const kvs_decode_args* a, void* ws, size_t ws_bytes,
                                      int32_t* dev_status, void* stream, cudaEvent_t const* ev) {
  KVS_REQUIRE(a != nullptr, KVS_EINVAL, "decode_step: args is null");
  KVS_REQUIRE(a->q && a->out && a->fullK && a->fullV && a->n, KVS_EINVAL,
              "decode_step: q/out/fullK/fullV/n must be non-null");
  KVS_REQUIRE(a->q_dtype == KVS_F32 || a->q_dtype == KVS_BF16, KVS_EINVAL,
              "decode_step: q_dtype=%d", a->q_dtype);
  KVS_REQUIRE(a->H >= 1 && a->H <= 8 && a->k >= 1 && a->n_max >= 1, KVS_EINVAL,
              "decode_step: H=%d k=%d n_max=%d", a->H, a->k, a->n_max);
  KVS_REQUIRE(a->ix != nullptr, KVS_EINVAL, "decode_step: index descriptor is null");
  KVS_REQUIRE(aligned16(a->fullK) && aligned16(a->fullV) && aligned16(a->out), KVS_EINVAL,
              "decode_step: fullK, fullV and out must be 16-byte aligned");
  if (a->slot_map) {
    KVS_REQUIRE(a->hotK && a->hotV && a->S >= 1, KVS_EINVAL,
                "decode_step: a slot map needs hotK/hotV and S >= 1");
    KVS_REQUIRE(aligned16(a->hotK) && aligned16(a->hotV), KVS_EINVAL,
                "decode_step: hotK/hotV must be 16-byte aligned");
  }
  if (a->idx_in == nullptr) {
    kvs_status st = check_index(a->ix, a->n_max);
    if (st != KVS_OK) return st;
    st = check_plan(a->plan, a->ix->D);
    if (st != KVS_OK) return st;
    KVS_REQUIRE(a->idx != nullptr, KVS_EINVAL, "decode_step: idx output is null");
    KVS_REQUIRE(a->q_dtype == KVS_F32, KVS_EINVAL,
                "decode_step: the bit allocation takes f32 queries");
  } else {
    KVS_REQUIRE(a->ix->R >= 1 && a->ix->G >= 1, KVS_EINVAL, "decode_step: index R/G");
  }
  // a full store in host memory also needs the staging of the fetched misses
  const bool host_full = a->fullK && host_resident(a->fullK);
  KVS_REQUIRE(!host_full || host_resident(a->fullV), KVS_EINVAL,
              "decode_step: fullK is host memory but fullV is not");
  const size_t need = host_full ? decode_ws_bytes_host(a->ix->R, a->ix->G, a->H, a->n_max, a->k,
                                                       a->plan ? a->plan->B : 0)
                                : decode_ws_bytes(a->ix->R, a->ix->G, a->H, a->n_max, a->k,
                                                  a->plan ? a->plan->B : 0);
  KVS_REQUIRE(ws && ws_bytes >= need, KVS_EWORKSPACE, "decode_step: workspace %zu < %zu bytes",
              ws_bytes, need);
  kvs_status st = decode_step_run(a, ws, dev_status, static_cast<cudaStream_t>(stream), ev);
  return st == KVS_OK ? ok() : st;
}

kvs_status decode_step(const kvs_decode_args* a, void* ws, size_t ws_bytes, int32_t* dev_status,
                       void* stream) {
  return decode_step_checked(a, ws, ws_bytes, dev_status, stream, nullptr);
}

kvs_status decode_step_timed(const kvs_decode_args* a, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream, void* const* events,
                             int32_t n_events) {
  KVS_REQUIRE(events != nullptr && n_events == KVS_DECODE_STAGES + 1, KVS_EINVAL,
              "decode_step_timed: %d events given, %d needed", n_events, KVS_DECODE_STAGES + 1);
  for (int i = 0; i < n_events; ++i)
    KVS_REQUIRE(events[i] != nullptr, KVS_EINVAL, "decode_step_timed: event %d is null", i);
  return decode_step_checked(a, ws, ws_bytes, dev_status, stream,
                             reinterpret_cast<cudaEvent_t const*>(events));
}

}  // extern "C"
