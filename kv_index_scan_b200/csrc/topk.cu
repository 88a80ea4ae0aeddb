// topk.cu -- a3: exact top-k of a score row ("XM-Sparse: Pushing the
// Throughput Frontier of Sparse Attention with Netpreme X-Mem", modelled
// study: 2,048 KV entries are picked per layer and step; "MiniMax-M3: share the
// sparse index top-k across layers and reuse the decode top-k buffer",
// description: the selection is made over 64-token KV blocks).
//
// Order: (score desc, index asc). Scores become order-preserving u32 keys; a
// three-pass radix select (11 + 11 + 10 bits, shared-memory histograms with
// warp-aggregated atomics) finds the k-th key tau and how many tau-valued
// entries to take; an ordered block-wide compaction then emits every entry
// above tau plus the first (lowest-index) tau-valued ones, which leaves the
// output ascending by index. Block mode selects k/block blocks and expands
// them to their tokens. One 1024-thread block per (request, KV head) row.
#include <cub/block/block_scan.cuh>

#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kNT = 1024;

struct RadixState {
  uint32_t prefix, mask;
  int krem;
};

// Finds the key of rank keff (1-based, from the top) among the ne keys given by
// key_of(i). Returns tau and, in krem, how many keys equal to tau belong to
// the top keff.
template <typename KeyOf>
__device__ void radix_select(KeyOf key_of, int ne, int keff, uint32_t& tau, int& take_eq) {
  __shared__ unsigned hist[2048];
  __shared__ RadixState st;
  if (threadIdx.x == 0) st = {0u, 0u, keff};
  const int lane = threadIdx.x & 31;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t dmask = (1u << widths[pass]) - 1u;
    for (int b = threadIdx.x; b < 2048; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = st.prefix, mask = st.mask;
    for (int base = 0; base < ne; base += blockDim.x) {
      const int i = base + threadIdx.x;
      int bin = -1;
      if (i < ne) {
        const uint32_t key = key_of(i);
        if ((key & mask) == prefix) bin = static_cast<int>((key >> shift) & dmask);
      }
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // find the bin holding rank krem counting from the top: warp-parallel
      // over chunks of 64 bins from the highest
      int krem = st.krem;
      const int nbins = static_cast<int>(dmask) + 1;
      int digit = 0;
      int above = 0;
      for (int top = nbins; top > 0; top -= 64) {
        const int b0 = top - 1 - 2 * lane, b1 = b0 - 1;
        const int c0 = b0 >= 0 ? static_cast<int>(hist[b0]) : 0;
        const int c1 = b1 >= 0 ? static_cast<int>(hist[b1]) : 0;
        const int mine = c0 + c1;
        int incl = mine;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
          if (lane >= d) incl += o;
        }
        const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        if (above + total >= krem) {
          const unsigned hit = __ballot_sync(0xFFFFFFFFu, above + incl >= krem);
          const int l = __ffs(hit) - 1;
          const int ex = __shfl_sync(0xFFFFFFFFu, incl - mine, l);
          const int cb0 = __shfl_sync(0xFFFFFFFFu, c0, l);
          const int bb0 = top - 1 - 2 * l;
          if (above + ex + cb0 >= krem) {
            digit = bb0;
            krem -= above + ex;
          } else {
            digit = bb0 - 1;
            krem -= above + ex + cb0;
          }
          break;
        }
        above += total;
      }
      if (lane == 0) {
        st.prefix = prefix | (static_cast<uint32_t>(digit) << shift);
        st.mask = mask | (dmask << shift);
        st.krem = krem;
      }
    }
    __syncthreads();
  }
  tau = st.prefix;
  take_eq = st.krem;
}

__global__ void __launch_bounds__(kNT) topk_rows_kernel(const float* __restrict__ scores,
                                                       int64_t ld, const int32_t* __restrict__ n,
                                                       int G, int k, int block,
                                                       int32_t* __restrict__ idx,
                                                       float* __restrict__ vals) {
  using BlockScan = cub::BlockScan<int, kNT>;
  __shared__ typename BlockScan::TempStorage scan_tmp;
  const int u = blockIdx.x;
  const int nr = n[u / G];
  const int64_t ne64 = block == 1 ? nr : (nr + block - 1) / block;
  const int ne = static_cast<int>(ne64 < ld ? ne64 : ld);
  const int kk = k / block;
  const int keff = min(kk, ne);
  const float* row = scores + static_cast<size_t>(u) * ld;
  int32_t* irow = idx + static_cast<size_t>(u) * k;
  float* vrow = vals ? vals + static_cast<size_t>(u) * k : nullptr;
  for (int j = threadIdx.x; j < k; j += kNT) {
    irow[j] = -1;
    if (vrow) vrow[j] = -__int_as_float(0x7f800000);
  }
  __syncthreads();
  if (keff <= 0) return;
  uint32_t tau;
  int take_eq;
  radix_select([row](int i) { return ordered_key(row[i]); }, ne, keff, tau, take_eq);
  int eq_base = 0, out_base = 0;
  for (int base = 0; base < ne && out_base < keff; base += kNT) {
    const int i = base + threadIdx.x;
    uint32_t key = 0;
    float f = 0.f;
    if (i < ne) {
      f = row[i];
      key = ordered_key(f);
    }
    const int gt = (i < ne && key > tau) ? 1 : 0;
    const int eq = (i < ne && key == tau) ? 1 : 0;
    int eq_ex, eq_tot;
    BlockScan(scan_tmp).ExclusiveSum(eq, eq_ex, eq_tot);
    __syncthreads();
    const int take = gt | (eq && eq_base + eq_ex < take_eq ? 1 : 0);
    int t_ex, t_tot;
    BlockScan(scan_tmp).ExclusiveSum(take, t_ex, t_tot);
    __syncthreads();
    if (take) {
      const int q = out_base + t_ex;
      if (block == 1) {
        irow[q] = i;
        if (vrow) vrow[q] = f;
      } else {
        for (int t = 0; t < block; ++t) {
          const int tok = i * block + t;
          if (tok < nr) {
            irow[q * block + t] = tok;
            if (vrow) vrow[q * block + t] = f;
          }
        }
      }
    }
    eq_base += eq_tot;
    out_base += t_tot;
  }
}

}  // namespace

size_t topk_ws_bytes(int, int, int, int, int) { return 0; }

kvs_status topk_launch(const float* scores, int64_t ld, const int32_t* n, int R, int G, int k,
                       int block, int32_t* idx, float* vals, cudaStream_t s) {
  topk_rows_kernel<<<R * G, kNT, 0, s>>>(scores, ld, n, G, k, block, idx, vals);
  return check_launch("topk_select");
}

}  // namespace kvs
