// internal.cuh -- declarations shared between the launch layer (api.cu,
// decode.cu) and the kernel files of libkvscan.
#pragma once

#include "common.cuh"

namespace kvs {

// ---- attention row sources (attn.cu) ----
// kRowsSlotStaged: hits from the hot slots, misses from a staging buffer
// [RG][k][D] at the entry's position j (the rows fetched from a full store in
// host memory, fetch.cu)
enum RowMode { kRowsStaged = 0, kRowsSlot = 1, kRowsDirect = 2, kRowsSlotStaged = 3 };

struct RowSrc {
  int mode;
  const uint16_t* K;  // staged [RG][k][D] or full store [RG][n_max][D]
  const uint16_t* V;
  const uint16_t* hotK;  // [RG][S][D]
  const uint16_t* hotV;
  const int32_t* idx;  // [RG][k] or, with idx_shared, [R][k]
  int idx_shared;
  const int32_t* slots;     // [RG][k] slot of each selected key (nullable)
  const int32_t* slot_map;  // [RG][n_max] (used when slots is null)
  const int32_t* k_eff;     // staged mode: valid rows per (r, g) (nullable)
  int n_max, S, G, k;
};

// ---- launchers ----
size_t build_index_ws_bytes(int R, int G, int D);
kvs_status build_index_launch(const uint16_t* K, const int32_t* n, int R, int G, int n_max, int W,
                              uint32_t* planes, float* kmin, float* kstep, float* kvar, void* ws,
                              cudaStream_t s);
kvs_status plan_bits_launch(const float* q, int H, const float* kmin, const float* kstep,
                            const float* kvar, int RG, int B, uint8_t* t, uint16_t* plane_idx,
                            float* plane_w, float* C, cudaStream_t s);
kvs_status fathom_scan_simple_launch(const uint32_t* planes, int W, int R, int G,
                                     const uint16_t* plane_idx, const float* plane_w,
                                     const float* C, int B, const int32_t* n, int n_max,
                                     float* scores, cudaStream_t s, float* gmax = nullptr);
struct ScanParams;
kvs_status fathom_scan_lut_launch(const ScanParams& p, cudaStream_t s);
bool fused_topk_supported(int n_max, int k, int B);
size_t fused_ws_bytes(int RG, int n_max, int k, int B, bool host_mapped = false);
kvs_status fathom_scan_topk_launch(ScanParams p, void* ws, const int32_t* slot_map, int32_t* idx,
                                   int32_t* slots, int32_t* misses, cudaStream_t s,
                                   cudaEvent_t after_scan = nullptr, bool host_mapped = false);
kvs_status fathom_scan_dispatch(const kvs_fathom_index* ix, const kvs_plan* plan,
                                const int32_t* n, int n_max, float* scores, int32_t* dev_status,
                                cudaStream_t s);
kvs_status lightning_scan_dispatch(const kvs_scan_args* a, float* scores, int32_t* dev_status,
                                   cudaStream_t s);
size_t topk_ws_bytes(int R, int G, int n_max, int k, int block);
kvs_status topk_launch(const float* scores, int64_t ld, const int32_t* n, int R, int G, int k,
                       int block, int32_t* idx, float* vals, cudaStream_t s);
kvs_status sparse_gather_launch(const int32_t* idx, int k, const int32_t* slot_map,
                                const uint16_t* hotK, const uint16_t* hotV, int S,
                                const uint16_t* fullK, const uint16_t* fullV, int n_max, int RG,
                                uint16_t* gK, uint16_t* gV, int32_t* slots, int32_t* misses,
                                cudaStream_t s);
kvs_status select_slots_launch(const int32_t* idx, int idx_shared, int G, int k,
                               const int32_t* slot_map, int n_max, int RG, int32_t* slots,
                               int32_t* misses, cudaStream_t s);
void attn_split(int RG, int k, int& nsplit, int& rows_per_split);
size_t attn_ws_bytes(int RG, int H, int k);
// q_early: q may be read before the wait on the preceding kernel (no kernel of
// the launch chain writes it).
kvs_status attn_launch(const void* q, int q_bf16, const RowSrc& src, int RG, int H, float scale,
                       float* out, float* lse, void* ws, cudaStream_t s, bool q_early = false);
kvs_status attn_launch_fit(const void* q, int q_bf16, const RowSrc& src, int RG, int H,
                           float scale, float* out, float* lse, float* part, size_t part_bytes,
                           size_t* need, cudaStream_t s);
size_t decode_ws_bytes(int R, int G, int H, int n_max, int k, int B);
bool host_resident(const void* p);
kvs_status fetch_misses_launch(const int32_t* idx, int idx_shared, int G, int k, const int32_t* slots,
                               const uint16_t* fullK, const uint16_t* fullV, int n_max, int RG,
                               uint16_t* stageK, uint16_t* stageV, cudaStream_t s);
size_t decode_ws_bytes_host(int R, int G, int H, int n_max, int k, int B);
kvs_status append_token_launch(const uint16_t* Knew, const uint16_t* Vnew, int32_t* n, int R, int G,
                               int n_max, uint32_t* planes, int W, const float* kmin, const float* kstep,
                               uint16_t* fullK, uint16_t* fullV, int32_t* slot_map, const int32_t* hot_slot,
                               int32_t* hot_tok, uint16_t* hotK, uint16_t* hotV, int S, int32_t* dev_status,
                               cudaStream_t s);
kvs_status decode_step_run(const kvs_decode_args* a, void* ws, int32_t* dev_status,
                           cudaStream_t s,
                           cudaEvent_t const* ev = nullptr);

const char* g_err_text();

}  // namespace kvs
