// gather.cu -- a4: fetch the selected K/V rows through the hot-buffer slot map
// ("XM-Sparse: Pushing the Throughput Frontier of Sparse Attention with
// Netpreme X-Mem", Figure 1 and the request-lifecycle item on fetching selected
// KV: each selected entry is looked up in the GPU's hot buffer, and only the
// absent ones come from the full store; the miss rate counts those).
//
// slot_map[r][g][i] >= 0 is the hot slot holding key i (a hit); -1 means the
// key is absent (a miss: row from the full store). One block per (r, g); a
// half-warp moves one 256-byte K row and one V row with 16-byte accesses; the
// miss count is a block reduction (no atomics, no pre-zeroing).
#include "internal.cuh"

namespace kvs {

namespace {

__global__ void __launch_bounds__(256) sparse_gather_kernel(
    const int32_t* __restrict__ idx, int k, const int32_t* __restrict__ slot_map,
    const uint16_t* __restrict__ hotK, const uint16_t* __restrict__ hotV, int S,
    const uint16_t* __restrict__ fullK, const uint16_t* __restrict__ fullV, int n_max,
    uint16_t* __restrict__ gK, uint16_t* __restrict__ gV, int32_t* __restrict__ slots,
    int32_t* __restrict__ misses) {
  const int u = blockIdx.x;
  const int half = threadIdx.x >> 4, l16 = threadIdx.x & 15;
  int my_misses = 0;
  for (int j = half; j < k; j += blockDim.x / 16) {
    const int i = idx[static_cast<size_t>(u) * k + j];
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    int slot = -2;
    if (i >= 0) {
      slot = slot_map[static_cast<size_t>(u) * n_max + i];
      const uint16_t *ks, *vs;
      if (slot >= 0) {
        ks = hotK + (static_cast<size_t>(u) * S + slot) * kD;
        vs = hotV + (static_cast<size_t>(u) * S + slot) * kD;
      } else {
        ks = fullK + (static_cast<size_t>(u) * n_max + i) * kD;
        vs = fullV + (static_cast<size_t>(u) * n_max + i) * kD;
        if (l16 == 0) ++my_misses;
      }
      kv = reinterpret_cast<const uint4*>(ks)[l16];
      vv = reinterpret_cast<const uint4*>(vs)[l16];
    }
    reinterpret_cast<uint4*>(gK + (static_cast<size_t>(u) * k + j) * kD)[l16] = kv;
    reinterpret_cast<uint4*>(gV + (static_cast<size_t>(u) * k + j) * kD)[l16] = vv;
    if (l16 == 0) slots[static_cast<size_t>(u) * k + j] = slot;
  }
  __shared__ int warp_sum[8];
  const int w = __reduce_add_sync(0xFFFFFFFFu, my_misses);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = w;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int e = 0; e < 8; ++e) t += warp_sum[e];
    misses[u] = t;
  }
}

// The slot of every selected key and the miss count of each (r, g), without
// moving rows: the attention kernel then reads K/V through these slots. With
// vec (k a multiple of 4, idx and slots 16-byte aligned) each thread handles
// four entries per 16-byte load and store.
__global__ void __launch_bounds__(256) select_slots_kernel(
    const int32_t* __restrict__ idx, int idx_shared, int G, int k,
    const int32_t* __restrict__ slot_map, int n_max, int32_t* __restrict__ slots,
    int32_t* __restrict__ misses, int vec) {
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x;
  const int32_t* irow = idx + (idx_shared ? static_cast<size_t>(u / G) : static_cast<size_t>(u)) * k;
  const int32_t* smap = slot_map ? slot_map + static_cast<size_t>(u) * n_max : nullptr;
  int32_t* srow = slots ? slots + static_cast<size_t>(u) * k : nullptr;
  auto slot_of = [&](int i) { return i < 0 ? -2 : (smap ? smap[i] : -1); };
  int my_misses = 0;
  if (vec) {
    for (int j4 = threadIdx.x; j4 < k / 4; j4 += blockDim.x) {
      const int4 iv = *reinterpret_cast<const int4*>(irow + 4 * j4);
      const int4 sv = make_int4(slot_of(iv.x), slot_of(iv.y), slot_of(iv.z), slot_of(iv.w));
      my_misses += (iv.x >= 0 && sv.x < 0) + (iv.y >= 0 && sv.y < 0) + (iv.z >= 0 && sv.z < 0) +
                   (iv.w >= 0 && sv.w < 0);
      if (srow) *reinterpret_cast<int4*>(srow + 4 * j4) = sv;
    }
  } else {
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
      const int i = irow[j];
      const int slot = slot_of(i);
      my_misses += (i >= 0 && slot < 0) ? 1 : 0;
      if (srow) srow[j] = slot;
    }
  }
  __shared__ int warp_sum[8];
  const int w = __reduce_add_sync(0xFFFFFFFFu, my_misses);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = w;
  __syncthreads();
  if (threadIdx.x == 0 && misses) {
    int t = 0;
    for (int e = 0; e < 8; ++e) t += warp_sum[e];
    misses[u] = t;
  }
}

}  // namespace

kvs_status select_slots_launch(const int32_t* idx, int idx_shared, int G, int k,
                               const int32_t* slot_map, int n_max, int RG, int32_t* slots,
                               int32_t* misses, cudaStream_t s) {
  const int vec = (k % 4 == 0) && aligned16(idx) && (slots == nullptr || aligned16(slots)) ? 1 : 0;
  launch_chained(select_slots_kernel, dim3(RG), dim3(256), 0, s, idx, idx_shared, G, k, slot_map, n_max, slots,
                 misses, vec);
  return check_launch("select_slots");
}

kvs_status sparse_gather_launch(const int32_t* idx, int k, const int32_t* slot_map,
                                const uint16_t* hotK, const uint16_t* hotV, int S,
                                const uint16_t* fullK, const uint16_t* fullV, int n_max, int RG,
                                uint16_t* gK, uint16_t* gV, int32_t* slots, int32_t* misses,
                                cudaStream_t s) {
  sparse_gather_kernel<<<RG, 256, 0, s>>>(idx, k, slot_map, hotK, hotV, S, fullK, fullV, n_max, gK,
                                          gV, slots, misses);
  return check_launch("sparse_gather");
}

}  // namespace kvs
