// scan_topk.cu -- a2 + a3 for decode_step: the Fathom scan followed by the
// per-row top-k, with the hot-buffer slot lookup of every selected key.
//
// Selection order is (score desc, index asc) ("XM-Sparse: Pushing the
// Throughput Frontier of Sparse Attention with Netpreme X-Mem", modelled
// study: 2,048 entries are picked per layer and step).
//
// Plans of at most 144 planes: the byte-indexed scan writes every score and
// the maximum of every 16 keys; topk_scores_kernel (below) selects from them,
// one block per row, reading only the groups whose maximum can reach the
// row's k-th score.
//
// Larger plans: the group-table scan keeps each row's candidates on chip.
// Each block walks a contiguous range of chunks; the part of one (request, KV
// head) row inside a block is a "segment". Per segment the block appends to a
// buffer in L2 every key whose score is at least a running threshold tau (all
// keys, until a threshold exists), as (order-preserving score key, index).
// When the buffer may not hold another chunk, two histogram passes over the
// held keys (bits 31..21, then 20..10) find the cell holding the k-th largest
// key; tau becomes that cell's lower edge and every held key below it is
// dropped. The held set always contains the segment's top-k (at least k keys
// are >= tau), so nothing of the answer is ever lost. A merge kernel, one
// block per row, gathers the segments' candidates as distinct 53-bit
// composites (score key << 21 | (2^21 - 1 - index)), selects exactly the k
// largest (radix passes), emits their indices in ascending order through a
// bitmap over the row, and looks every selected key up in the hot-buffer slot
// map (slots; misses = the number absent from the hot buffer).
#include "internal.cuh"
#include "scan_core.cuh"
#include "scan_prmt.cuh"

namespace kvs {

namespace {

constexpr int kIdxBits = 21;
constexpr uint32_t kIdxMask = (1u << kIdxBits) - 1u;
constexpr int kCandCap = 16384;  // per-block candidate buffer entries in global memory

__device__ __forceinline__ uint64_t make_composite(uint32_t key, int idx) {
  return (static_cast<uint64_t>(key) << kIdxBits) |
         static_cast<uint64_t>(kIdxMask - static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int composite_index(uint64_t c) {
  return static_cast<int>(kIdxMask - static_cast<uint32_t>(c & kIdxMask));
}

// The block whose chunk range [floor(b*C/grid), floor((b+1)*C/grid)) holds chunk x.
__host__ __device__ __forceinline__ int block_of_chunk(long long x, long long C, int grid) {
  int b = static_cast<int>(x * grid / C);
  while (b + 1 < grid && (static_cast<long long>(b + 1) * C) / grid <= x) ++b;
  while (b > 0 && (static_cast<long long>(b) * C) / grid > x) --b;
  return b;
}

// Group-wide (all nthreads threads, uniform call): in a histogram over
// [0, nbins) bins, the bin holding rank krem counted from the top, and the
// count above it, into res[0], res[1]. Each thread sums a run of bins, one
// exclusive scan over the threads finds the run holding the rank, and its
// thread walks it. wsum holds one entry per warp. Ends with a barrier.
template <typename Sync>
__device__ void find_bin_from_top(const unsigned* hist, int nbins, int krem, int* wsum, int* res,
                                  int tid, int nthreads, Sync sync) {
  const int per = (nbins + nthreads - 1) / nthreads;
  const int hi = nbins - tid * per;  // this thread's bins: hi - 1 down to hi - per
  int mine = 0;
  for (int e = 0; e < per; ++e) {
    const int bb = hi - 1 - e;
    if (bb >= 0) mine += static_cast<int>(hist[bb]);
  }
  const int lane = tid & 31, warp = tid >> 5;
  int incl = mine;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  if (tid == 0) {
    res[0] = 0;
    res[1] = 0;
  }
  sync();
  const int before = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? wsum[lane] : 0);
  const int ex = before + incl - mine;
  if (mine > 0 && ex < krem && ex + mine >= krem) {
    int above = ex;
    for (int e = 0; e < per && hi - 1 - e >= 0; ++e) {
      const int bb = hi - 1 - e;
      const int c = static_cast<int>(hist[bb]);
      if (above + c >= krem) {
        res[0] = bb;
        res[1] = above;
        break;
      }
      above += c;
    }
  }
  sync();
}

__device__ __forceinline__ void hist_add(unsigned* hist, int bin) {
  const int lane = threadIdx.x & 31;
  const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
  if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

struct SelectState {
  unsigned long long prefix, mask;
  int krem, done;
  uint32_t tau;
  int wsum[32], res[2];
};

// Group-wide: the kk-th largest of the n distinct 53-bit composites in src
// (kk >= 1, n >= kk); radix passes of 11/11/11/10/10 bits, stopping early once
// the bin holding the rank is taken whole (its lower edge then selects exactly
// kk: usually after the third pass, which resolves the full score key).
template <typename Sync>
__device__ uint64_t select_kth_composite(const uint64_t* src, int n, int kk, unsigned* hist,
                                         SelectState* st, int tid, int nthreads, Sync sync) {
  if (tid == 0) {
    st->prefix = 0ull;
    st->mask = 0ull;
    st->krem = kk;
    st->done = 0;
  }
  for (int pass = 0; pass < 5; ++pass) {
    const int shift = pass < 3 ? 42 - 11 * pass : (pass == 3 ? 10 : 0);
    const unsigned dmask = pass < 3 ? 2047u : 1023u;
    for (int b = tid; b < 2048; b += nthreads) hist[b] = 0;
    sync();
    const unsigned long long prefix = st->prefix, mask = st->mask;
    for (int base = 0; base < n; base += 4 * nthreads) {
      uint64_t c[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = base + e * nthreads + tid;
        c[e] = i < n ? src[i] : ~0ull;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = base + e * nthreads + tid;
        const int bin = (i < n && (c[e] & mask) == prefix) ? static_cast<int>((c[e] >> shift) & dmask) : -1;
        hist_add(hist, bin);
      }
    }
    sync();
    find_bin_from_top(hist, static_cast<int>(dmask) + 1, st->krem, st->wsum, st->res, tid,
                      nthreads, sync);
    if (tid == 0) {
      const int bin = st->res[0];
      st->prefix = prefix | (static_cast<unsigned long long>(bin) << shift);
      st->mask = mask | (static_cast<unsigned long long>(dmask) << shift);
      st->krem -= st->res[1];
      st->done = st->krem == static_cast<int>(hist[bin]) ? 1 : 0;
    }
    sync();
    if (st->done) break;
  }
  return st->prefix;
}

struct SegState {
  int cnt, cnt2, tau_set;
  float tau_f;
  SelectState sel;
};

// Candidate store of one block: keys in shared memory (SK) or in global
// memory, indices in global memory; one buffer, compacted in place.
template <int G, int b, int W, bool SK>
__global__ void KVS_SCAN_BOUNDS(G, b, W) fathom_scan_topk_kernel(ScanParams p) {
  using Core = ScanCore<G, b, W>;
  constexpr int NT = 32 * W;
  Core core(p);
  unsigned* hist = reinterpret_cast<unsigned*>(core.extra());
  SegState* st = reinterpret_cast<SegState*>(hist + 2048);
  auto sync = [] { consumer_sync<W>(); };
  uint32_t* kb = SK ? reinterpret_cast<uint32_t*>(st + 1)
                    : p.cbuf_key + static_cast<size_t>(blockIdx.x) * p.cand_cap;
  int32_t* ib = p.cbuf_idx + static_cast<size_t>(blockIdx.x) * p.cand_cap;
  const long long C = static_cast<long long>(p.RG) * p.chunks_per_row;
  if (threadIdx.x == 0) {
    st->cnt = 0;
    st->tau_set = 0;
  }
  // (visible to the consumers through the barrier at the first row change)

  // Lower edge of the 22-bit key cell holding the kk-th largest held key
  // (two histogram passes; at least kk held keys are >= it).
  auto cell_threshold = [&](int n, int kk) -> uint32_t {
    const int t = threadIdx.x;
    for (int bb = t; bb < 2048; bb += NT) hist[bb] = 0;
    sync();
    for (int base = 0; base < n; base += 4 * NT) {
      uint32_t kv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = base + e * NT + t;
        kv[e] = i < n ? kb[i] : 0u;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        hist_add(hist, base + e * NT + t < n ? static_cast<int>(kv[e] >> 21) : -1);
    }
    sync();
    find_bin_from_top(hist, 2048, kk, st->sel.wsum, st->sel.res, t, NT, sync);
    const uint32_t b1 = static_cast<uint32_t>(st->sel.res[0]);
    const int krem = kk - st->sel.res[1];
    for (int bb = t; bb < 2048; bb += NT) hist[bb] = 0;
    sync();
    for (int base = 0; base < n; base += 4 * NT) {
      uint32_t kv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = base + e * NT + t;
        kv[e] = i < n ? kb[i] : 0u;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool in = base + e * NT + t < n && (kv[e] >> 21) == b1;
        hist_add(hist, in ? static_cast<int>((kv[e] >> 10) & 2047u) : -1);
      }
    }
    sync();
    find_bin_from_top(hist, 2048, krem, st->sel.wsum, st->sel.res, t, NT, sync);
    return (b1 << 21) | (static_cast<uint32_t>(st->sel.res[0]) << 10);
  };

  // Keep the held entries with key >= tau, compacted in place: each round
  // reads kRound entries per thread (their index loads in flight together),
  // then (after a barrier) writes the kept ones below them, so no unread
  // entry is ever overwritten (uniform call).
  auto keep_at_least = [&](uint32_t tau, float tau_f) {
    constexpr int kRound = 8;
    const int t = threadIdx.x;
    const int n = st->cnt;
    if (t == 0) st->cnt2 = 0;
    sync();
    for (int base = 0; base < n; base += kRound * NT) {
      uint32_t key[kRound];
      int32_t ix[kRound];
#pragma unroll
      for (int e = 0; e < kRound; ++e) {
        const int i = base + e * NT + t;
        key[e] = i < n ? kb[i] : 0u;
      }
#pragma unroll
      for (int e = 0; e < kRound; ++e) {
        const int i = base + e * NT + t;
        ix[e] = (i < n && key[e] >= tau) ? ib[i] : 0;
      }
      sync();
      // one shared-memory atomic per warp and round
      const int lane = t & 31;
      const unsigned lt = (1u << lane) - 1u;
      unsigned m[kRound];
      int wtot = 0;
#pragma unroll
      for (int e = 0; e < kRound; ++e) {
        m[e] = __ballot_sync(0xFFFFFFFFu, base + e * NT + t < n && key[e] >= tau);
        wtot += __popc(m[e]);
      }
      if (wtot > 0) {
        int pos = 0;
        if (lane == 0) pos = atomicAdd(&st->cnt2, wtot);
        pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
#pragma unroll
        for (int e = 0; e < kRound; ++e) {
          if ((m[e] >> lane) & 1u) {
            kb[pos + __popc(m[e] & lt)] = key[e];
            ib[pos + __popc(m[e] & lt)] = ix[e];
          }
          pos += __popc(m[e]);
        }
      }
    }
    sync();
    if (t == 0) {
      st->cnt = st->cnt2;
      st->tau_set = 1;
      st->tau_f = tau_f;
    }
    sync();
  };

  // Exact cut to the best kk held entries by (key, index) composites; only
  // when a cell holds so many equal keys that the cell threshold cannot
  // shrink the set (uniform call).
  auto cut_exact = [&](int kk) {
    const int t = threadIdx.x;
    const int n = st->cnt;
    uint64_t* comp = p.cbuf_comp + static_cast<size_t>(blockIdx.x) * p.cand_cap;
    for (int i = t; i < n; i += NT) comp[i] = make_composite(kb[i], ib[i]);
    sync();
    const uint64_t tau = select_kth_composite(comp, n, min(kk, n), hist, &st->sel, t, NT, sync);
    if (t == 0) st->cnt2 = 0;
    sync();
    for (int base = 0; base < n; base += NT) {
      const int i = base + t;
      const uint64_t c = i < n ? comp[i] : 0ull;
      const bool take = i < n && c >= tau;
      const unsigned m = __ballot_sync(0xFFFFFFFFu, take);
      if (m == 0u) continue;
      const int lane = t & 31, leader = __ffs(m) - 1;
      int pos = 0;
      if (lane == leader) pos = atomicAdd(&st->cnt2, __popc(m));
      pos = __shfl_sync(0xFFFFFFFFu, pos, leader) + __popc(m & ((1u << lane) - 1u));
      if (take) {
        kb[pos] = static_cast<uint32_t>(c >> kIdxBits);
        ib[pos] = composite_index(c);
      }
    }
    sync();
    if (t == 0) {
      st->cnt = st->cnt2;
      st->tau_set = 1;
      st->tau_f = key_to_float(static_cast<uint32_t>(tau >> kIdxBits));
    }
    sync();
  };

  // Trim the held set to a superset of its top kk (uniform call).
  auto trim = [&](int kk) {
    if (st->cnt <= kk) return;
    const uint32_t tau = cell_threshold(st->cnt, kk);
    keep_at_least(tau, key_to_float(tau));
  };

  // A threshold for a segment's first chunk from the chunk's own scores (in
  // registers), when it holds at least k valid keys: the lower edge of the
  // 22-bit key cell holding its k-th largest key (uniform call).
  auto chunk_threshold = [&](int i0, int nr, const float (&acc)[kKeysPerThread]) {
    const int t = threadIdx.x;
    uint32_t key[kKeysPerThread];
#pragma unroll
    for (int j = 0; j < kKeysPerThread; ++j) key[j] = ordered_key(acc[j]);
    for (int bb = t; bb < 2048; bb += NT) hist[bb] = 0;
    sync();
#pragma unroll
    for (int j = 0; j < kKeysPerThread; ++j)
      hist_add(hist, i0 + j < nr ? static_cast<int>(key[j] >> 21) : -1);
    sync();
    find_bin_from_top(hist, 2048, p.k, st->sel.wsum, st->sel.res, t, NT, sync);
    const uint32_t b1 = static_cast<uint32_t>(st->sel.res[0]);
    const int krem = p.k - st->sel.res[1];
    for (int bb = t; bb < 2048; bb += NT) hist[bb] = 0;
    sync();
#pragma unroll
    for (int j = 0; j < kKeysPerThread; ++j)
      hist_add(hist, (i0 + j < nr && (key[j] >> 21) == b1) ? static_cast<int>((key[j] >> 10) & 2047u)
                                                            : -1);
    sync();
    find_bin_from_top(hist, 2048, krem, st->sel.wsum, st->sel.res, t, NT, sync);
    const uint32_t tau = (b1 << 21) | (static_cast<uint32_t>(st->sel.res[0]) << 10);
    if (t == 0) {
      st->tau_set = 1;
      st->tau_f = key_to_float(tau);
    }
    sync();
  };

  core.run([&](int u, int c, int nr, const float (&acc)[kKeysPerThread], int t) {
    // 1. keys at or above the running threshold join the segment's candidates
    const int i0 = 32 * (c * Core::CHUNK_WORDS + (t >> 1)) + kKeysPerThread * (t & 1);
    if (st->tau_set == 0 && nr - 32 * c * Core::CHUNK_WORDS >= p.k) chunk_threshold(i0, nr, acc);
    const bool has_tau = st->tau_set != 0;
    const float tau = st->tau_f;
    // one shared-memory atomic per warp and chunk: the warp's takes are
    // counted first, then written at ballot-ordered positions
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    unsigned m[kKeysPerThread];
    int wtotal = 0;
#pragma unroll
    for (int j = 0; j < kKeysPerThread; ++j) {
      m[j] = __ballot_sync(0xFFFFFFFFu, i0 + j < nr && (!has_tau || acc[j] >= tau));
      wtotal += __popc(m[j]);
    }
    if (wtotal > 0) {
      int base = 0;
      if (lane == 0) base = atomicAdd(&st->cnt, wtotal);
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
#pragma unroll
      for (int j = 0; j < kKeysPerThread; ++j) {
        if ((m[j] >> lane) & 1u) {
          const int pos = base + __popc(m[j] & lt);
          kb[pos] = ordered_key(acc[j]);
          ib[pos] = i0 + j;
        }
        base += __popc(m[j]);
      }
    }
    sync();
    // 2. the segment ends here, or there must be room for one more chunk
    const long long chunk_id = static_cast<long long>(u) * p.chunks_per_row + c;
    const long long last_chunk = static_cast<long long>(blockIdx.x + 1) * C / gridDim.x - 1;
    const bool seg_end = c == p.chunks_per_row - 1 || chunk_id == last_chunk;
    if (seg_end) {
      trim(p.k);
      if (st->cnt > p.seg_cap) cut_exact(p.k);
      const int kk = st->cnt;
      const int slot = static_cast<int>(blockIdx.x) -
                       block_of_chunk(static_cast<long long>(u) * p.chunks_per_row, C, gridDim.x);
      const size_t off = (static_cast<size_t>(u) * p.segs_per_row + slot) * p.seg_cap;
#pragma unroll 4
      for (int e = threadIdx.x; e < kk; e += NT) {
        p.cand_key[off + e] = kb[e];
        p.cand_idx[off + e] = ib[e];
      }
      if (threadIdx.x == 0) {
        p.cand_count[static_cast<size_t>(u) * p.segs_per_row + slot] = kk;
        st->cnt = 0;
        st->tau_set = 0;
      }
      sync();
    } else if (st->cnt > p.trim_at) {
      trim(p.k);
      if (st->cnt > p.cand_cap - 32 * Core::CHUNK_WORDS) cut_exact(p.k);
    }
  });
}

// One block per (r, g): gather the segments' candidates, select the k best,
// emit their indices in ascending order, look up their slots. 1024 threads.
// The ascending order comes from a bitmap over the row's key indices (in the
// workspace): the selected keys set their bits, each thread counts the bits
// of its run of words, one block-wide scan gives every thread its output
// position, and the threads write the set bits of their runs in order.
constexpr int kMergeThreads = 1024;
constexpr int kMergeMaxK = 4096;
constexpr int kMergeSmemEntries = 24576;
static_assert(kMergeThreads == 32 * 32, "the merge sums its per-warp counts with one warp");

__host__ __device__ __forceinline__ int bitmap_words(int n_max) {
  return (((n_max + 31) / 32) + 3) & ~3;
}

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(
    ScanParams p, int scan_grid, uint64_t* __restrict__ gscratch, uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ slot_map, int32_t* __restrict__ idx, int32_t* __restrict__ slots,
    int32_t* __restrict__ misses) {
  __shared__ unsigned hist[2048];
  __shared__ SelectState sel;
  __shared__ int seg_count[512], seg_off[513];
  __shared__ uint32_t seg_tau[512];
  __shared__ int kept_total;
  __shared__ int wsum[kMergeThreads / 32];
  __shared__ int miss_warp[kMergeThreads / 32];
  extern __shared__ __align__(16) uint64_t comp_smem[];
  const int u = blockIdx.x;
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int nr = p.n[u / p.Gheads];
  const int kk = min(p.k, nr);
  const long long C = static_cast<long long>(p.RG) * p.chunks_per_row;
  const int b0 = block_of_chunk(static_cast<long long>(u) * p.chunks_per_row, C, scan_grid);
  const int b1 = block_of_chunk(static_cast<long long>(u + 1) * p.chunks_per_row - 1, C, scan_grid);
  const int segs = (b1 - b0 + 1) * p.lists_per_seg;
  if (t < segs) {
    seg_count[t] = p.cand_count[static_cast<size_t>(u) * p.segs_per_row + t];
    seg_tau[t] = p.cand_tau ? p.cand_tau[static_cast<size_t>(u) * p.segs_per_row + t] : 0u;
  }
  if (t == 0) kept_total = 0;
  __syncthreads();
  if (t == 0) {
    int o = 0;
    for (int s = 0; s < segs; ++s) {
      seg_off[s] = o;
      o += seg_count[s];
    }
    seg_off[segs] = o;
  }
  // clear this row's bitmap meanwhile
  const int words = bitmap_words(p.n_max);
  uint32_t* bm = bitmap + static_cast<size_t>(u) * words;
  for (int w = 4 * t; w < words; w += 4 * kMergeThreads)
    *reinterpret_cast<uint4*>(bm + w) = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const int all = seg_off[segs];
  // entries below their segment's threshold are not needed; count the rest
  // first when all of them would not fit in shared memory
  bool in_smem = all <= kMergeSmemEntries;
  if (!in_smem) {
    int mine = 0;
    for (int f = t; f < all; f += kMergeThreads) {
      int s = 0;
      while (f >= seg_off[s + 1]) ++s;
      const size_t off = (static_cast<size_t>(u) * p.segs_per_row + s) * p.seg_cap + (f - seg_off[s]);
      mine += p.cand_key[off] >= seg_tau[s] ? 1 : 0;
    }
    mine = __reduce_add_sync(0xFFFFFFFFu, mine);
    if (lane == 0) atomicAdd(&kept_total, mine);
    __syncthreads();
    in_smem = kept_total <= kMergeSmemEntries;
    __syncthreads();
    if (t == 0) kept_total = 0;
    __syncthreads();
  }
  uint64_t* comp =
      in_smem ? comp_smem : gscratch + static_cast<size_t>(u) * p.segs_per_row * p.seg_cap;
  // gather the kept candidates as composites: keys and indices of eight
  // entries per thread in flight together
  for (int base = 0; base < all; base += 8 * kMergeThreads) {
    uint32_t key[8], kt[8];
    int32_t ix[8];
    bool keep[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int f = base + e * kMergeThreads + t;
      key[e] = 0u;
      ix[e] = 0;
      kt[e] = 0xFFFFFFFFu;
      if (f < all) {
        int s = 0;
        while (f >= seg_off[s + 1]) ++s;
        const size_t off = (static_cast<size_t>(u) * p.segs_per_row + s) * p.seg_cap + (f - seg_off[s]);
        key[e] = p.cand_key[off];
        ix[e] = p.cand_idx[off];
        kt[e] = seg_tau[s];
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) keep[e] = base + e * kMergeThreads + t < all && key[e] >= kt[e];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const unsigned m = __ballot_sync(0xFFFFFFFFu, keep[e]);
      if (m == 0u) continue;
      int pos = 0;
      if (lane == 0) pos = atomicAdd(&kept_total, __popc(m));
      pos = __shfl_sync(0xFFFFFFFFu, pos, 0) + __popc(m & ((1u << lane) - 1u));
      if (keep[e]) comp[pos] = make_composite(key[e], ix[e]);
    }
  }
  __syncthreads();
  const int total = kept_total;
  uint64_t tau = 0ull;
  if (kk > 0 && total > kk)
    tau = select_kth_composite(comp, total, kk, hist, &sel, t, kMergeThreads,
                               [] { __syncthreads(); });
  // the selected keys set their bits
  if (kk > 0) {
    for (int f = t; f < total; f += kMergeThreads) {
      const uint64_t c = comp[f];
      if (c >= tau) {
        const int i = composite_index(c);
        atomicOr(bm + (i >> 5), 1u << (i & 31));
      }
    }
  }
  __syncthreads();
  // ascending emission: thread t owns words [t * wpt, (t + 1) * wpt)
  const int wpt = ((words + kMergeThreads - 1) / kMergeThreads + 3) & ~3;
  const int w_beg = min(words, t * wpt), w_end = min(words, w_beg + wpt);
  int cnt = 0;
  for (int w = w_beg; w < w_end; w += 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(bm + w);
    cnt += __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
  }
  int incl = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  const int before = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? wsum[lane] : 0);
  int pos = before + incl - cnt;
  int32_t* irow = idx + static_cast<size_t>(u) * p.k;
  for (int w = w_beg; w < w_end && cnt > 0; ++w) {
    uint32_t bits = bm[w];
    while (bits) {
      const int bpos = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < p.k) irow[pos] = 32 * w + bpos;
      ++pos;
    }
  }
  __syncthreads();
  const int chosen_total =
      min(__reduce_add_sync(0xFFFFFFFFu, wsum[lane]), kk);  // 32 warps: one entry per lane
  // pad, slots and misses
  int my_miss = 0;
  for (int j = t; j < p.k; j += kMergeThreads) {
    int i = -1;
    if (j < chosen_total)
      i = irow[j];
    else
      irow[j] = -1;
    int s = -2;
    if (i >= 0) {
      s = slot_map ? slot_map[static_cast<size_t>(u) * p.n_max + i] : -1;
      my_miss += s < 0 ? 1 : 0;
    }
    if (slots) slots[static_cast<size_t>(u) * p.k + j] = s;
  }
  const int wm = __reduce_add_sync(0xFFFFFFFFu, my_miss);
  if (lane == 0) miss_warp[warp] = wm;
  __syncthreads();
  if (t == 0 && misses) {
    int m = 0;
    for (int e = 0; e < kMergeThreads / 32; ++e) m += miss_warp[e];
    misses[u] = m;
  }
}

// ---------------------------------------------------------------------------
// Top-k of one (request, KV head) row from its scores and 16-key group maxima
// (the byte-indexed scan writes both). One block of 1,024 threads per row.
//  A. T = (a lower bound of) the kk-th largest group maximum: each group
//     maximum is a distinct key, so at least kk keys are >= T and the row's
//     kk-th largest score is >= T. The maxima are kept as 16-bit key prefixes,
//     selected in 12-bit digits from the highest bit in which they differ
//     (one digit when they span less than 2^12 prefixes).
//     Groups whose maximum is below T hold no selected key and are never read
//     (about a quarter of the groups remain for Gaussian-like scores).
//  B. The remaining groups are listed in index order (8 per thread, one
//     block-wide scan per 8,192 groups).
//  C. Each warp takes a contiguous slice of that list, four lanes per group
//     (one 16-byte load each, so a warp's load touches 8 groups' lines), and
//     appends its keys >= T with their indices, in index order, to a list of
//     its own; the warps' lists in warp order are the row's candidates in
//     index order.
//  D. Radix select over the candidates in digits of up to 12 bits, from the
//     highest bit in which the smallest and the largest candidate differ:
//     either a whole key cell holds the last selected ranks (select every key
//     >= its lower edge: exactly kk keys), or the exact kk-th largest key K*
//     (select the keys > K*, and of the keys equal to K* the lowest indices).
//  E. Each warp emits its selected keys at their ranks in index order (one
//     block-wide exchange of the warps' counts), with the slot of each; the
//     row's miss count closes the kernel.
// Rows longer than 65,536 groups, or whose candidates overflow the on-chip
// lists, take the same selection over global memory with a bitmap.
constexpr int kTkThreads = 1024;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkBins = 4096;

struct TkState {
  int wsum[32], res[2];
  uint32_t prefix, mask;
  int krem, done, gt;
  int wcnt[32], ws[32], wt[32];
  uint32_t wmax[32];
  int miss_warp[32];
};

// Block-wide radix select of the kk-th largest key over the keys enumerated by
// each(visit) (every thread visits its own share; the same set each pass).
// Returns the cell or key; *whole is true when every key >= the returned value
// is selected (exactly kk of them), false when it is the exact kk-th key and
// *gt keys lie strictly above it.
template <typename Each>
__device__ uint32_t radix_kth_key(Each&& each, int kk, unsigned* hist, TkState* st, bool* whole, int* gt) {
  const int t = threadIdx.x;
  if (t == 0) {
    st->prefix = 0u;
    st->mask = 0u;
    st->krem = kk;
    st->done = 0;
    st->gt = 0;
  }
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass < 2 ? 2047u : 1023u;
    for (int b = t; b < 2048; b += kTkThreads) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = st->prefix, mask = st->mask;
    each([&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    });
    __syncthreads();
    find_bin_from_top(hist, static_cast<int>(dmask) + 1, st->krem, st->wsum, st->res, t, kTkThreads,
                      [] { __syncthreads(); });
    if (t == 0) {
      const int bin = st->res[0];
      st->prefix = prefix | (static_cast<uint32_t>(bin) << shift);
      st->mask = mask | (dmask << shift);
      st->krem -= st->res[1];
      st->gt += st->res[1];
      st->done = st->krem == static_cast<int>(hist[bin]) ? 1 : (pass == 2 ? 2 : 0);
    }
    __syncthreads();
    if (st->done) break;
  }
  *whole = st->done == 1;
  *gt = st->gt;
  return st->prefix;
}

// The same select when every key agrees with `prefix` on the bits above `top`:
// digits of up to 12 bits from bit `top` down. With first_ready, hist already
// holds the histogram of the first digit (built while the keys were produced).
template <typename Each>
__device__ uint32_t radix_select_from(Each&& each, int top, uint32_t prefix, int kk, bool first_ready,
                                      unsigned* hist, TkState* st, bool* whole, int* gt) {
  const int t = threadIdx.x;
  uint32_t mask = top >= 31 ? 0u : ~((2u << top) - 1u);
  int krem = kk, above = 0;
  for (;;) {
    const int width = min(12, top + 1);
    const int shift = top + 1 - width;
    const uint32_t dmask = (1u << width) - 1u;
    const int nb = 1 << width;
    if (!first_ready) {
      for (int b = t; b < nb; b += kTkThreads) hist[b] = 0;
      __syncthreads();
      each([&](uint32_t key) {
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
      });
      __syncthreads();
    }
    first_ready = false;
    find_bin_from_top(hist, nb, krem, st->wsum, st->res, t, kTkThreads, [] { __syncthreads(); });
    const int bin = st->res[0];
    const int ab = st->res[1];
    const int inbin = static_cast<int>(hist[bin]);
    prefix |= static_cast<uint32_t>(bin) << shift;
    mask |= dmask << shift;
    krem -= ab;
    above += ab;
    const int done = krem == inbin ? 1 : (shift == 0 ? 2 : 0);
    __syncthreads();  // hist[bin] and res are read before the next pass rewrites them
    if (done) {
      *whole = done == 1;
      *gt = above;
      return prefix;
    }
    top = shift - 1;
  }
}

constexpr int kTkMaxGroups = 65536;  // group maxima kept in shared memory (16-bit prefixes)
constexpr int kTkCandGroups = 8192;  // candidate groups on chip
// per-warp candidate lists (key, index), over the maxima once those are read
constexpr int kTkWarpKeys = static_cast<int>(kTkMaxGroups * sizeof(uint16_t) / (kTkWarps * sizeof(uint2)));
constexpr size_t kTkSmem = kTkMaxGroups * sizeof(uint16_t) + kTkCandGroups * sizeof(int);

// Block-wide exclusive prefix of c over the threads (in thread order); returns
// it and the block total.
__device__ __forceinline__ int block_excl_scan(int c, TkState* st, int* total) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int incl = c;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) st->wsum[warp] = incl;
  __syncthreads();
  const int before = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? st->wsum[lane] : 0);
  *total = __reduce_add_sync(0xFFFFFFFFu, st->wsum[lane]);
  __syncthreads();
  return before + incl - c;
}

__global__ void __launch_bounds__(kTkThreads, 1) topk_scores_kernel(
    const float* __restrict__ scores, const float* __restrict__ gmax, const int32_t* __restrict__ n,
    int Gheads, int n_max, int k, uint32_t* __restrict__ bitmap, const int32_t* __restrict__ slot_map,
    int32_t* __restrict__ idx, int32_t* __restrict__ slots, int32_t* __restrict__ misses) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned hist[kTkBins];
  __shared__ TkState st;
  extern __shared__ __align__(16) unsigned char tk_smem[];
  uint16_t* gk = reinterpret_cast<uint16_t*>(tk_smem);                          // [kTkMaxGroups]
  uint2* lists = reinterpret_cast<uint2*>(tk_smem);                              // [kTkWarps][kTkWarpKeys]
  int* cg = reinterpret_cast<int*>(tk_smem + kTkMaxGroups * sizeof(uint16_t));  // [kTkCandGroups]
  constexpr int NG = 16;  // keys per group
  constexpr unsigned FULL = 0xFFFFFFFFu;
  const float ninf = -__int_as_float(0x7f800000);
  const int u = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int nr = min(n[u / Gheads], n_max);
  const int kk = min(k, nr);
  const int ldg = (n_max + NG - 1) / NG;
  const int m = (nr + NG - 1) / NG;
  const float* sc = scores + static_cast<size_t>(u) * n_max;
  const float* gm = gmax + static_cast<size_t>(u) * ldg;
  const bool vec = (n_max & 3) == 0;
  int32_t* irow = idx + static_cast<size_t>(u) * k;
  int32_t* srow = slots ? slots + static_cast<size_t>(u) * k : nullptr;
  const int32_t* smap = slot_map ? slot_map + static_cast<size_t>(u) * n_max : nullptr;

  bool onchip = kk > 0 && m <= kTkMaxGroups;
  uint32_t T = 0u;
  int my_miss = 0;
  if (onchip) {
    // A. maxima as 16-bit prefixes (the histogram of their bits 15..4 built
    // as they load) and the largest of them; T
    for (int b = t; b < kTkBins; b += kTkThreads) hist[b] = 0;
    __syncthreads();
    uint32_t pmax = 0u;
#pragma unroll 8
    for (int g = t; g < m; g += kTkThreads) {
      const uint32_t pfx = ordered_key(__ldg(gm + g)) >> 16;
      gk[g] = static_cast<uint16_t>(pfx);
      atomicAdd(&hist[pfx >> 4], 1u);
      pmax = max(pmax, pfx);
    }
    pmax = __reduce_max_sync(FULL, pmax);
    if (lane == 0) st.wmax[warp] = pmax;
    __syncthreads();
    // every key of the row is <= hi (the prefix of its largest maximum, low bits set)
    const uint32_t hi = (__reduce_max_sync(FULL, st.wmax[lane]) << 16) | 0xFFFFu;
    if (kk <= m) {
      bool wh;
      int g0;
      T = radix_select_from([&](auto visit) {
            for (int g = t; g < m; g += kTkThreads) visit(static_cast<uint32_t>(gk[g]));
          }, 15, 0u, kk, true, hist, &st, &wh, &g0) << 16;
    }
    // the candidates lie in [T, hi]: the first digit of their select starts at
    // the highest bit in which T and hi differ
    const uint32_t xr = T ^ hi;
    const int top1 = xr ? 31 - __clz(xr) : 0;
    const int width1 = min(12, top1 + 1);
    const int shift1 = top1 + 1 - width1;
    const uint32_t dmask1 = (1u << width1) - 1u;
    for (int b = t; b < kTkBins; b += kTkThreads) hist[b] = 0;  // visible after B's barriers
    // B. candidate groups in index order
    const uint32_t Tp = T >> 16;
    int ncg = 0;
    for (int r0 = 0; r0 < m; r0 += 8 * kTkThreads) {
      const int g0 = r0 + 8 * t;
      uint32_t flags = 0u;
      if (g0 < m) {
        const uint4 w = *reinterpret_cast<const uint4*>(gk + g0);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t pfx = (ww[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
          if (g0 + j < m && pfx >= Tp) flags |= 1u << j;
        }
      }
      int tot;
      int q = ncg + block_excl_scan(__popc(flags), &st, &tot);
      if (q + __popc(flags) <= kTkCandGroups) {
        while (flags) {
          const int j = __ffs(flags) - 1;
          flags &= flags - 1u;
          cg[q++] = g0 + j;
        }
      }
      ncg += tot;
    }
    onchip = ncg <= kTkCandGroups;
    if (onchip) {
      __syncthreads();  // cg is complete; the maxima are no longer read
      // C. this warp's slice of the candidate groups, four lanes per group
      const int per_w = (ncg + kTkWarps - 1) / kTkWarps;
      const int e_beg = min(ncg, warp * per_w), e_end = min(ncg, e_beg + per_w);
      uint2* wl = lists + warp * kTkWarpKeys;
      const int sub = lane >> 2, qtr = lane & 3;
      int wc = 0;
      bool ovf = false;
      // four iterations' loads in flight per warp
      constexpr int kU = 4;
      const int niter = (e_end - e_beg + 7) >> 3;
      // key(v) >= T: for T >= key(+0) one signed compare of v's bits
      const bool tpos = (T & 0x80000000u) != 0u;
      const int tint = static_cast<int>(T & 0x7FFFFFFFu);
      for (int it0 = 0; it0 < niter && !ovf; it0 += kU) {
        float4 f[kU];
        int base[kU];
#pragma unroll
        for (int a = 0; a < kU; ++a) {
          const int e = e_beg + 8 * (it0 + a) + sub;
          base[a] = -1;
          f[a] = make_float4(ninf, ninf, ninf, ninf);
          if (it0 + a < niter && e < e_end) {
            base[a] = cg[e] * NG + 4 * qtr;
            if (vec && base[a] + 4 <= n_max) {
              f[a] = __ldg(reinterpret_cast<const float4*>(sc + base[a]));
            } else {
              const float* s0 = sc + base[a];
              f[a].x = base[a] < n_max ? __ldg(s0) : ninf;
              f[a].y = base[a] + 1 < n_max ? __ldg(s0 + 1) : ninf;
              f[a].z = base[a] + 2 < n_max ? __ldg(s0 + 2) : ninf;
              f[a].w = base[a] + 3 < n_max ? __ldg(s0 + 3) : ninf;
            }
          }
        }
#pragma unroll
        for (int a = 0; a < kU; ++a) {
          if (it0 + a >= niter) break;
          const float v[4] = {f[a].x, f[a].y, f[a].z, f[a].w};
          uint32_t pass = 0u;
          if (base[a] >= 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const bool ge = tpos ? __float_as_int(v[j]) >= tint : ordered_key(v[j]) >= T;
              if (ge && base[a] + j < nr) pass |= 1u << j;
            }
          }
          const int c = __popc(pass);
          const unsigned b0 = __ballot_sync(FULL, c & 1), b1 = __ballot_sync(FULL, c & 2),
                         b2 = __ballot_sync(FULL, c & 4);
          const int tot = __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
          if (wc + tot > kTkWarpKeys) {
            ovf = true;
            break;
          }
          int q = wc + __popc(b0 & lt) + 2 * __popc(b1 & lt) + 4 * __popc(b2 & lt);
          while (pass) {
            const int j = __ffs(pass) - 1;
            pass &= pass - 1u;
            const float x = j == 0 ? v[0] : (j == 1 ? v[1] : (j == 2 ? v[2] : v[3]));
            const uint32_t key = ordered_key(x);
            wl[q++] = make_uint2(key, static_cast<uint32_t>(base[a] + j));
            atomicAdd(&hist[(key >> shift1) & dmask1], 1u);
          }
          wc += tot;
        }
      }
      if (lane == 0) st.wcnt[warp] = ovf ? -1 : wc;
      __syncthreads();
      onchip = !__any_sync(FULL, st.wcnt[lane] < 0);
      if (onchip) {
        // D. the kk-th largest candidate key (first digit counted in C)
        const uint32_t upper = top1 >= 31 ? 0u : ~((2u << top1) - 1u);
        bool whole;
        int gt;
        const uint32_t cut = radix_select_from([&](auto visit) {
              for (int i = lane; i < wc; i += 32) visit(wl[i].x);
            }, top1, T & upper, kk, true, hist, &st, &whole, &gt);
        // E. ranks in index order: keys above the cut, then the first `need` ties
        const int need = whole ? 0 : kk - gt;
        int ns = 0, nt = 0;
        for (int i = lane; i < wc; i += 32) {
          const uint32_t key = wl[i].x;
          ns += (whole ? key >= cut : key > cut) ? 1 : 0;
          nt += (!whole && key == cut) ? 1 : 0;
        }
        ns = __reduce_add_sync(FULL, ns);
        nt = __reduce_add_sync(FULL, nt);
        if (lane == 0) {
          st.ws[warp] = ns;
          st.wt[warp] = nt;
        }
        __syncthreads();
        int s_run = __reduce_add_sync(FULL, lane < warp ? st.ws[lane] : 0);
        int t_run = __reduce_add_sync(FULL, lane < warp ? st.wt[lane] : 0);
        for (int i0 = 0; i0 < wc; i0 += 32) {
          const int i = i0 + lane;
          const uint2 c = i < wc ? wl[i] : make_uint2(0u, 0u);
          const bool strict = i < wc && (whole ? c.x >= cut : c.x > cut);
          const bool tie = i < wc && !whole && c.x == cut;
          const unsigned bs = __ballot_sync(FULL, strict), bt = __ballot_sync(FULL, tie);
          const int sb = s_run + __popc(bs & lt), tb = t_run + __popc(bt & lt);
          const int pos = sb + min(tb, need);
          if ((strict || (tie && tb < need)) && pos < kk) {
            const int ix = static_cast<int>(c.y);
            irow[pos] = ix;
            const int sl = smap ? smap[ix] : -1;
            my_miss += sl < 0 ? 1 : 0;
            if (srow) srow[pos] = sl;
          }
          s_run += __popc(bs);
          t_run += __popc(bt);
        }
        for (int j = kk + t; j < k; j += kTkThreads) {
          irow[j] = -1;
          if (srow) srow[j] = -2;
        }
      }
    }
  }
  if (!onchip) {
    // too many candidates for the chip (or no row at all): the same selection
    // over the rows' scores in global memory (groups whose maximum is below T
    // are skipped), emitted through a bitmap over the row
    const int words = bitmap_words(n_max);
    uint32_t* bm = bitmap + static_cast<size_t>(u) * words;
    for (int w = 4 * t; w < words; w += 4 * kTkThreads)
      *reinterpret_cast<uint4*>(bm + w) = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    auto load_group = [&](int g, float (&v)[NG]) {
      const float* src = sc + static_cast<size_t>(g) * NG;
      if (vec && g * NG + NG <= n_max) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 f = __ldg(reinterpret_cast<const float4*>(src) + q);
          v[4 * q] = f.x;
          v[4 * q + 1] = f.y;
          v[4 * q + 2] = f.z;
          v[4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < NG; ++j) v[j] = g * NG + j < n_max ? __ldg(src + j) : ninf;
      }
    };
    if (kk > 0) {
      bool whole;
      int gt;
      const uint32_t key_cut = radix_kth_key([&](auto visit) {
            for (int g = t; g < m; g += kTkThreads) {
              if (ordered_key(__ldg(gm + g)) < T) continue;
              float v[NG];
              load_group(g, v);
#pragma unroll
              for (int j = 0; j < NG; ++j)
                if (g * NG + j < nr) {
                  const uint32_t key = ordered_key(v[j]);
                  if (key >= T) visit(key);
                }
            }
          }, kk, hist, &st, &whole, &gt);
      const int need = whole ? 0 : kk - gt;
      int tie_base = 0;
      for (int r0 = 0; r0 < m; r0 += kTkThreads) {
        const int g = r0 + t;
        uint32_t sel = 0u, tie = 0u;
        if (g < m && ordered_key(__ldg(gm + g)) >= key_cut) {
          float v[NG];
          load_group(g, v);
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            if (g * NG + j >= nr) continue;
            const uint32_t key = ordered_key(v[j]);
            if (whole ? key >= key_cut : key > key_cut) sel |= 1u << j;
            else if (!whole && key == key_cut) tie |= 1u << j;
          }
        }
        if (!whole) {
          int tot;
          int rank = tie_base + block_excl_scan(__popc(tie), &st, &tot);
          while (tie) {
            const int j = __ffs(tie) - 1;
            tie &= tie - 1u;
            if (rank < need) sel |= 1u << j;
            ++rank;
          }
          tie_base += tot;
        }
        if (sel) atomicOr(bm + (g >> 1), (g & 1) ? (sel << 16) : sel);
      }
    }
    __syncthreads();
    // ascending emission: thread t owns words [t * wpt, (t + 1) * wpt)
    const int wpt = ((words + kTkThreads - 1) / kTkThreads + 3) & ~3;
    const int w_beg = min(words, t * wpt), w_end = min(words, w_beg + wpt);
    int cnt = 0;
    for (int w = w_beg; w < w_end; w += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(bm + w);
      cnt += __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
    }
    int incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(FULL, incl, d);
      if (lane >= d) incl += o;
    }
    if (lane == 31) st.wsum[warp] = incl;
    __syncthreads();
    const int before = __reduce_add_sync(FULL, lane < warp ? st.wsum[lane] : 0);
    int pos = before + incl - cnt;
    for (int w = w_beg; w < w_end && cnt > 0; ++w) {
      uint32_t bits = bm[w];
      while (bits) {
        const int bpos = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (pos < k) irow[pos] = 32 * w + bpos;
        ++pos;
      }
    }
    __syncthreads();
    const int chosen_total = min(__reduce_add_sync(FULL, st.wsum[lane]), kk);
    for (int j = t; j < k; j += kTkThreads) {
      int i = -1;
      if (j < chosen_total)
        i = irow[j];
      else
        irow[j] = -1;
      int sl = -2;
      if (i >= 0) {
        sl = smap ? smap[i] : -1;
        my_miss += sl < 0 ? 1 : 0;
      }
      if (srow) srow[j] = sl;
    }
  }
  const int wm = __reduce_add_sync(FULL, my_miss);
  if (lane == 0) st.miss_warp[warp] = wm;
  __syncthreads();
  if (t == 0 && misses) {
    int mm = 0;
    for (int e = 0; e < kTkWarps; ++e) mm += st.miss_warp[e];
    misses[u] = mm;
  }
}

int fused_grid(int RG, int cpr) {
  const long long C = static_cast<long long>(RG) * cpr;
  return static_cast<int>(C < sm_count() ? C : sm_count());
}

int fused_segs_per_row(int RG, int cpr, int grid) {
  const long long C = static_cast<long long>(RG) * cpr;
  int mx = 1;
  for (int u = 0; u < RG; ++u) {
    const int b0 = block_of_chunk(static_cast<long long>(u) * cpr, C, grid);
    const int b1 = block_of_chunk(static_cast<long long>(u + 1) * cpr - 1, C, grid);
    mx = max(mx, b1 - b0 + 1);
  }
  return mx;
}

struct Layout {
  int grid, cpr, segs, lists, list_cap;  // segments per row, candidate lists per segment
};

// Plans of more than 144 planes: the group-table core, one candidate list of
// 2k per (block, row) segment.
Layout fused_layout(int RG, int n_max, int k, int B) {
  Layout L{};
  int G, b, nsets;
  scan_schedule(B, G, b, nsets);
  L.cpr = scan_chunks_per_row(n_max, scan_warps(G, b));
  L.lists = 1;
  L.list_cap = 2 * k;
  L.grid = fused_grid(RG, L.cpr);
  L.segs = L.grid > 0 ? fused_segs_per_row(RG, L.cpr, L.grid) : 1;
  return L;
}


struct FusedLaunch {
  const ScanParams& p;
  int grid;
  cudaStream_t s;
  template <int G, int b, int W>
  kvs_status operator()() const {
    using Core = ScanCore<G, b, W>;
    const size_t base_extra = 2048 * sizeof(unsigned) + sizeof(SegState);
    const int chunk_keys = 32 * Core::CHUNK_WORDS;
    // keys in shared memory when 2k + one chunk of them fit beside two stages
    const int cap_s = 2 * p.k + chunk_keys;
    const size_t extra_s = base_extra + static_cast<size_t>(cap_s) * sizeof(uint32_t);
    ScanParams q = p;
    q.warps = W;
    if (Core::nstages(p.nsets, extra_s) >= 2) {
      q.cand_cap = cap_s;
      q.trim_at = 2 * p.k;
      q.nstage = Core::nstages(p.nsets, extra_s);
      const size_t smem = Core::smem_bytes(p.nsets, extra_s);
      auto kern = fathom_scan_topk_kernel<G, b, W, true>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      kern<<<grid, Core::THREADS, smem, s>>>(q);
    } else {
      q.cand_cap = kCandCap;
      q.trim_at = kCandCap - chunk_keys;
      q.nstage = Core::nstages(p.nsets, base_extra);
      const size_t smem = Core::smem_bytes(p.nsets, base_extra);
      auto kern = fathom_scan_topk_kernel<G, b, W, false>;
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      kern<<<grid, Core::THREADS, smem, s>>>(q);
    }
    return check_launch("decode_step(scan+topk)");
  }
};

}  // namespace

bool fused_topk_supported(int n_max, int k, int B) {
  return B > 0 && k >= 1 && k <= kMergeMaxK && 2 * k <= kCandCap - 6144 &&
         n_max <= (1 << kIdxBits);
}

size_t fused_ws_bytes(int RG, int n_max, int k, int B, bool host_mapped) {
  if (B <= kPMaxB || host_mapped) {
    WsCarver c(nullptr);
    c.take<float>(static_cast<size_t>(RG) * n_max);
    c.take<float>(static_cast<size_t>(RG) * ((n_max + kPKeys - 1) / kPKeys));
    c.take<uint32_t>(static_cast<size_t>(RG) * bitmap_words(n_max));
    return c.used;
  }
  const Layout L = fused_layout(RG, n_max, k, B);
  const size_t lists = static_cast<size_t>(RG) * L.segs * L.lists;
  const size_t comp = static_cast<size_t>(kCandCap > L.lists * L.list_cap ? kCandCap : L.lists * L.list_cap);
  WsCarver c(nullptr);
  c.take<uint32_t>(static_cast<size_t>(L.grid) * kCandCap);
  c.take<int32_t>(static_cast<size_t>(L.grid) * kCandCap);
  c.take<uint64_t>(static_cast<size_t>(L.grid) * comp);
  c.take<uint32_t>(lists * L.list_cap);
  c.take<int32_t>(lists * L.list_cap);
  c.take<int32_t>(lists);
  c.take<uint32_t>(lists);
  c.take<uint64_t>(lists * L.list_cap);
  c.take<uint32_t>(static_cast<size_t>(RG) * bitmap_words(n_max));
  return c.used;
}

kvs_status fathom_scan_topk_launch(ScanParams p, void* ws, const int32_t* slot_map, int32_t* idx,
                                   int32_t* slots, int32_t* misses, cudaStream_t s,
                                   cudaEvent_t after_scan, bool host_mapped) {
  if (p.B <= kPMaxB || host_mapped) {
    // scores and 16-key group maxima from the byte-indexed scan, then the
    // per-row top-k over them
    WsCarver c(ws);
    ScanParams q = p;
    q.scores = c.take<float>(static_cast<size_t>(p.RG) * p.n_max);
    q.gmax = c.take<float>(static_cast<size_t>(p.RG) * ((p.n_max + kPKeys - 1) / kPKeys));
    uint32_t* bitmap = c.take<uint32_t>(static_cast<size_t>(p.RG) * bitmap_words(p.n_max));
    // the index in mapped host memory: the plain scan, reading over the host link
    kvs_status st = host_mapped
                        ? fathom_scan_simple_launch(p.planes, p.W, p.RG / p.Gheads, p.Gheads, p.plane_idx,
                                                    p.plane_w, p.C, p.B, p.n, p.n_max, q.scores, s, q.gmax)
                        : fathom_scan_lut_launch(q, s);
    if (st != KVS_OK) return st;
    if (after_scan) cudaEventRecord(after_scan, s);
    cudaFuncSetAttribute(topk_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kTkSmem));
    launch_chained(topk_scores_kernel, dim3(p.RG), dim3(kTkThreads), kTkSmem, s, q.scores, q.gmax, p.n, p.Gheads, p.n_max, p.k,
                                                         bitmap, slot_map, idx, slots, misses);
    return check_launch("decode_step(top-k over scores)");
  }
  const Layout L = fused_layout(p.RG, p.n_max, p.k, p.B);
  if (L.grid <= 0) return KVS_OK;
  if (L.segs * L.lists > 512) return fail(KVS_EUNSUPPORTED, "decode_step: %d segments per row", L.segs);
  p.chunks_per_row = L.cpr;
  p.segs_per_row = L.segs * L.lists;
  p.seg_cap = L.list_cap;
  p.lists_per_seg = L.lists;
  const size_t lists = static_cast<size_t>(p.RG) * p.segs_per_row;
  const size_t comp = static_cast<size_t>(kCandCap > L.lists * L.list_cap ? kCandCap : L.lists * L.list_cap);
  WsCarver c(ws);
  p.cbuf_key = c.take<uint32_t>(static_cast<size_t>(L.grid) * kCandCap);
  p.cbuf_idx = c.take<int32_t>(static_cast<size_t>(L.grid) * kCandCap);
  p.cbuf_comp = c.take<uint64_t>(static_cast<size_t>(L.grid) * comp);
  p.cand_key = c.take<uint32_t>(lists * L.list_cap);
  p.cand_idx = c.take<int32_t>(lists * L.list_cap);
  p.cand_count = c.take<int32_t>(lists);
  p.cand_tau = c.take<uint32_t>(lists);
  uint64_t* gscratch = c.take<uint64_t>(lists * L.list_cap);
  uint32_t* bitmap = c.take<uint32_t>(static_cast<size_t>(p.RG) * bitmap_words(p.n_max));
  p.cand_tau = nullptr;  // this kernel keeps no per-list threshold
  kvs_status st = dispatch_schedule(p, FusedLaunch{p, L.grid, s});
  if (after_scan) cudaEventRecord(after_scan, s);
  const size_t msmem = static_cast<size_t>(kMergeSmemEntries) * sizeof(uint64_t);
  cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(msmem));
  topk_merge_kernel<<<p.RG, kMergeThreads, msmem, s>>>(p, L.grid, gscratch, bitmap, slot_map, idx,
                                                        slots, misses);
  return check_launch("decode_step(top-k merge)");
}

}  // namespace kvs
