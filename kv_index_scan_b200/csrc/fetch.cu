// fetch.cu -- the miss fetch from the host tier, between the selection and
// the attention of decode_step ("XM-Sparse: Pushing the Throughput Frontier of
// Sparse Attention with Netpreme X-Mem", Figure 1 and the request-lifecycle
// item on fetching selected KV: the GPU keeps a hot KV buffer in HBM and
// brings in only the selected entries that are absent from it, from the full
// store in external memory, over the host link).
//
// When decode_step's full K/V store is pinned host memory (mapped into the
// device's address space), each selected entry whose slot is -1 (a miss) has
// its K and V rows (256 bytes each) read over the host link with 16-byte
// loads into a staging buffer [RG][k][D] at its position j; the attention then
// reads hits from the hot slots and misses from the staging buffer, all in
// HBM. A warp looks at 32 entries at once (one ballot finds the misses) and
// moves up to 8 missing entries together -- lanes 0-15 a K row, 16-31 the V
// row, all 8 reads issued before any store -- so that each warp keeps 4 KB of
// host reads in flight; a block of 8 warps walks one (request, KV head) row.
#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kFetchWarps = 8;

__global__ void __launch_bounds__(32 * kFetchWarps) fetch_misses_kernel(
    const int32_t* __restrict__ idx, int idx_shared, int G, int k, const int32_t* __restrict__ slots,
    const uint16_t* fullK, const uint16_t* fullV, int n_max, uint16_t* __restrict__ stageK,
    uint16_t* __restrict__ stageV) {
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* irow = idx + (idx_shared ? static_cast<size_t>(u / G) : static_cast<size_t>(u)) * k;
  const int32_t* srow = slots + static_cast<size_t>(u) * k;
  const bool isv = lane >= 16;
  const int ch = lane & 15;
  const uint16_t* src_base = (isv ? fullV : fullK) + static_cast<size_t>(u) * n_max * kD + ch * 8;
  uint16_t* dst_base = (isv ? stageV : stageK) + static_cast<size_t>(u) * k * kD + ch * 8;
  constexpr int kBatch = 8;
  for (int j0 = 32 * warp; j0 < k; j0 += 32 * kFetchWarps) {
    const int jl = j0 + lane;
    const bool miss = jl < k && irow[jl] >= 0 && srow[jl] < 0;
    unsigned mask = __ballot_sync(0xFFFFFFFFu, miss);
    while (mask) {
      int js[kBatch];
      uint4 v[kBatch];
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        js[e] = -1;
        if (mask) {
          js[e] = j0 + __ffs(mask) - 1;
          mask &= mask - 1;
        }
      }
#pragma unroll
      for (int e = 0; e < kBatch; ++e)
        if (js[e] >= 0) v[e] = *reinterpret_cast<const uint4*>(src_base + static_cast<size_t>(irow[js[e]]) * kD);
#pragma unroll
      for (int e = 0; e < kBatch; ++e)
        if (js[e] >= 0) *reinterpret_cast<uint4*>(dst_base + static_cast<size_t>(js[e]) * kD) = v[e];
    }
  }
}

}  // namespace

// Page-locked host memory (mapped into the device's address space).
bool host_resident(const void* p) {
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();  // a pointer the runtime does not know is not host memory it registered
    return false;
  }
  return attr.type == cudaMemoryTypeHost;
}

kvs_status fetch_misses_launch(const int32_t* idx, int idx_shared, int G, int k, const int32_t* slots,
                               const uint16_t* fullK, const uint16_t* fullV, int n_max, int RG,
                               uint16_t* stageK, uint16_t* stageV, cudaStream_t s) {
  launch_chained(fetch_misses_kernel, dim3(RG), dim3(32 * kFetchWarps), 0, s, idx, idx_shared, G, k,
                 slots, fullK, fullV, n_max, stageK, stageV);
  return check_launch("decode_step(miss fetch from host memory)");
}

}  // namespace kvs
