// append.cu -- the per-step write-back after the decode path: the token just
// generated joins every (request, KV head) row ("XM-Sparse: Pushing the
// Throughput Frontier of Sparse Attention with Netpreme X-Mem", the request
// lifecycle list: the KV generated at each step is written back; "Fathom:
// Per-Query Read Depth for Sparse Decoding over Offloaded KV Caches",
// abstract: the 4-bit channel-major bit-plane K copy the scan reads).
//
// For request r the new token takes position i = n[r]. Channel c of KV head g
// gets the code u = clamp(floor((k - m_c) / s_c + 1/2), 0, 15), computed in
// fp64 from the bf16 key with the row's stored m_c and s_c (s_c = 0 -> u = 0):
// the quantiser of the index build, not re-fitted (kmin, kstep and kvar are
// unchanged). The four plane bits of key i are set (or cleared) to u's bits,
// the K and V rows are stored in the full store at i, and, when a hot slot is
// given, the rows are copied into it, the slot's previous token leaves the
// slot map and the new one enters it. Finally n[r] grows by one. One block
// per request (G x 128 threads): every head of a request reads n[r] before
// the block's thread 0 advances it.
#include "internal.cuh"

namespace kvs {

namespace {

__global__ void append_token_kernel(const uint16_t* __restrict__ Knew, const uint16_t* __restrict__ Vnew,
                                    int32_t* __restrict__ n, int G, int n_max, uint32_t* __restrict__ planes,
                                    int W, const float* __restrict__ kmin, const float* __restrict__ kstep,
                                    uint16_t* __restrict__ fullK, uint16_t* __restrict__ fullV,
                                    int32_t* __restrict__ slot_map, const int32_t* __restrict__ hot_slot,
                                    int32_t* __restrict__ hot_tok, uint16_t* __restrict__ hotK,
                                    uint16_t* __restrict__ hotV, int S, int32_t* dev_status) {
  pdl_wait();
  const int r = blockIdx.x;
  const int g = threadIdx.x / kD, c = threadIdx.x % kD;
  const int i = n[r];
  __syncthreads();  // every thread has read n[r] before it is advanced
  if (i < 0 || i >= n_max) {
    if (threadIdx.x == 0) set_status(dev_status, KVS_EBOUNDS);
    return;
  }
  const int u = r * G + g;
  const size_t row = static_cast<size_t>(u) * kD + c;
  const double k = static_cast<double>(bf16_bits_to_float(Knew[row]));
  const double m = static_cast<double>(kmin[row]);
  const double s = static_cast<double>(kstep[row]);
  int code = 0;
  if (s != 0.0) {
    const double x = floor(__dadd_rn(__ddiv_rn(__dsub_rn(k, m), s), 0.5));
    code = x < 0.0 ? 0 : (x > 15.0 ? 15 : static_cast<int>(x));
  }
  const uint32_t bit = 1u << (i & 31);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t* word = planes + (row * 4 + p) * static_cast<size_t>(W) + (i >> 5);
    if ((code >> (3 - p)) & 1) atomicOr(word, bit);
    else atomicAnd(word, ~bit);
  }
  const size_t at = (static_cast<size_t>(u) * n_max + i) * kD + c;
  fullK[at] = Knew[row];
  fullV[at] = Vnew[row];
  const int slot = hot_slot ? hot_slot[u] : -1;
  if (slot >= 0 && slot < S) {
    const size_t h = (static_cast<size_t>(u) * S + slot) * kD + c;
    hotK[h] = Knew[row];
    hotV[h] = Vnew[row];
  }
  if (c == 0 && slot_map) {
    int32_t* sm = slot_map + static_cast<size_t>(u) * n_max;
    if (slot >= 0 && slot < S) {
      const int old = hot_tok[static_cast<size_t>(u) * S + slot];
      if (old >= 0 && old < n_max) sm[old] = -1;
      hot_tok[static_cast<size_t>(u) * S + slot] = i;
      sm[i] = slot;
    } else {
      sm[i] = -1;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) n[r] = i + 1;
}

}  // namespace

kvs_status append_token_launch(const uint16_t* Knew, const uint16_t* Vnew, int32_t* n, int R, int G,
                               int n_max, uint32_t* planes, int W, const float* kmin, const float* kstep,
                               uint16_t* fullK, uint16_t* fullV, int32_t* slot_map, const int32_t* hot_slot,
                               int32_t* hot_tok, uint16_t* hotK, uint16_t* hotV, int S, int32_t* dev_status,
                               cudaStream_t s) {
  launch_chained(append_token_kernel, dim3(R), dim3(G * kD), 0, s, Knew, Vnew, n, G, n_max, planes, W, kmin,
                 kstep, fullK, fullV, slot_map, hot_slot, hot_tok, hotK, hotV, S, dev_status);
  return check_launch("kvs_append_token");
}

}  // namespace kvs
