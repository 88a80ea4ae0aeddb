// decode.cu -- a6: one fused decode step for every (request, KV head), and
// the dispatch of the index scans.
//
// Step order (all on the caller's stream, nothing synchronised):
//   plan_bits -> Fathom scan -> top-k -> slots + misses -> attention over
//   the selected rows read through the slot map.
// With a selection given (idx_in), the first three are skipped: the layer
// group sharing of "MiniMax-M3: share the sparse index top-k across layers and
// reuse the decode top-k buffer" (description), where the group's first layer
// selects and the others reuse the selection.
#include <algorithm>

#include "internal.cuh"
#include "scan_core.cuh"

namespace kvs {

kvs_status fathom_scan_dispatch(const kvs_fathom_index* ix, const kvs_plan* plan,
                                const int32_t* n, int n_max, float* scores, int32_t* dev_status,
                                cudaStream_t s) {
  if (ix->host_mapped || plan->B == 0)
    return fathom_scan_simple_launch(ix->planes, ix->W, ix->R, ix->G, plan->plane_idx,
                                     plan->plane_w, plan->C, plan->B, n, n_max, scores, s);
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
  return fathom_scan_lut_launch(p, s);
}

size_t decode_ws_bytes(int R, int G, int H, int n_max, int k, int B) {
  WsCarver c(nullptr);
  c.take<int32_t>(static_cast<size_t>(R) * G * k);  // slots when the caller passes none
  c.take<unsigned char>(attn_ws_bytes(R * G, H, k));
  const size_t unfused = static_cast<size_t>(R) * G * n_max * sizeof(float);  // scores
  // the larger of the HBM and the host-mapped layouts (the index's residence
  // is not known here)
  const size_t fused = fused_topk_supported(n_max, k, B)
                           ? std::max(fused_ws_bytes(R * G, n_max, k, B),
                                      fused_ws_bytes(R * G, n_max, k, B, true)) : 0;
  c.take<unsigned char>(unfused > fused ? unfused : fused);
  return c.used;
}

// With the full K/V store in host memory: the above, then the staging
// buffers of the fetched misses (K and V, [RG][k][D] each).
size_t decode_ws_bytes_host(int R, int G, int H, int n_max, int k, int B) {
  WsCarver c(nullptr);
  c.take<unsigned char>(decode_ws_bytes(R, G, H, n_max, k, B));
  c.take<uint16_t>(static_cast<size_t>(R) * G * k * kD);
  c.take<uint16_t>(static_cast<size_t>(R) * G * k * kD);
  return c.used;
}

kvs_status decode_step_run(const kvs_decode_args* a, void* ws, int32_t* dev_status,
                           cudaStream_t s, cudaEvent_t const* ev) {
  const int R = a->ix->R, G = a->ix->G, RG = R * G;
  // stage boundaries: 0 start, 1 allocation, 2 scan, 3 selection, 4 attention
  auto mark = [&](int i) {
    if (ev) cudaEventRecord(ev[i], s);
  };
  mark(0);
  WsCarver c(ws);
  int32_t* slots_ws = c.take<int32_t>(static_cast<size_t>(RG) * a->k);
  void* attn_ws = c.take<unsigned char>(attn_ws_bytes(RG, a->H, a->k));
  void* rest = c.take<unsigned char>(0);
  int32_t* slots = a->slots ? a->slots : slots_ws;
  kvs_status st;
  const int32_t* sel = a->idx_in;
  int shared = a->idx_in ? a->idx_shared : 0;
  bool have_slots = false;
  if (!sel) {
    const int B = a->plan->B;
    st = plan_bits_launch(static_cast<const float*>(a->q), a->H, a->ix->kmin, a->ix->kstep,
                          a->ix->kvar, RG, B, a->plan->t, a->plan->plane_idx, a->plan->plane_w,
                          a->plan->C, s);
    if (st != KVS_OK) return st;
    mark(1);
    if (fused_topk_supported(a->n_max, a->k, B)) {
      // plans of <= 144 planes or an index in mapped host memory: the scan
      // writes scores and 16-key maxima, then the per-row top-k over them;
      // longer plans: the scan keeps top-k candidates on chip, then the
      // per-row merge (both write the slots and misses)
      ScanParams p{};
      p.planes = a->ix->planes;
      p.W = a->ix->W;
      p.RG = RG;
      p.Gheads = G;
      p.plane_idx = a->plan->plane_idx;
      p.plane_w = a->plan->plane_w;
      p.C = a->plan->C;
      p.B = B;
      p.n = a->n;
      p.n_max = a->n_max;
      scan_schedule(B, p.G, p.b, p.nsets);
      p.dev_status = dev_status;
      p.k = a->k;
      st = fathom_scan_topk_launch(p, rest, a->slot_map, a->idx, slots, a->misses, s,
                                   ev ? ev[2] : nullptr, a->ix->host_mapped != 0);
      if (st != KVS_OK) return st;
      have_slots = true;
    } else {
      float* scores = static_cast<float*>(rest);
      st = fathom_scan_dispatch(a->ix, a->plan, a->n, a->n_max, scores, dev_status, s);
      if (st != KVS_OK) return st;
      mark(2);
      st = topk_launch(scores, a->n_max, a->n, R, G, a->k, 1, a->idx, nullptr, s);
      if (st != KVS_OK) return st;
    }
    sel = a->idx;
  } else {
    mark(1);
    mark(2);
  }
  if (!have_slots) {
    st = select_slots_launch(sel, shared, G, a->k, a->slot_map, a->n_max, RG, slots, a->misses, s);
    if (st != KVS_OK) return st;
  }
  mark(3);
  RowSrc src{};
  src.mode = a->slot_map ? kRowsSlot : kRowsDirect;
  if (host_resident(a->fullK)) {
    // the full store lives in host memory: bring the misses into HBM first
    WsCarver h(ws);
    h.take<unsigned char>(decode_ws_bytes(R, G, a->H, a->n_max, a->k, a->plan ? a->plan->B : 0));
    uint16_t* stageK = h.take<uint16_t>(static_cast<size_t>(RG) * a->k * kD);
    uint16_t* stageV = h.take<uint16_t>(static_cast<size_t>(RG) * a->k * kD);
    st = fetch_misses_launch(sel, shared, G, a->k, slots, a->fullK, a->fullV, a->n_max, RG, stageK,
                             stageV, s);
    if (st != KVS_OK) return st;
    src.mode = kRowsSlotStaged;
    src.K = stageK;
    src.V = stageV;
  }
  if (src.mode != kRowsSlotStaged) {
    src.K = a->fullK;
    src.V = a->fullV;
  }
  src.hotK = a->hotK;
  src.hotV = a->hotV;
  src.idx = sel;
  src.idx_shared = shared;
  src.slots = slots;
  src.slot_map = a->slot_map;
  src.n_max = a->n_max;
  src.S = a->S;
  src.G = G;
  src.k = a->k;
  // q may be read before the wait on the preceding kernel when this step ran
  // the plan kernel: it waits for everything before the step before it lets
  // the chain go on, and no kernel of the step writes q
  st = attn_launch(a->q, a->q_dtype == KVS_BF16, src, RG, a->H, a->scale, a->out, a->lse,
                   attn_ws, s, /*q_early=*/a->idx_in == nullptr);
  if (st != KVS_OK) return st;
  mark(4);
  return KVS_OK;
}


}  // namespace kvs
