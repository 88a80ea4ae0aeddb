// scan_topk.cu -- a2 + a3 fused for decode_step: the Fathom scan keeps each
// row's top-k candidates on chip instead of writing every score to HBM.
//
// Selection order is (score desc, index asc) ("XM-Sparse: Pushing the
// Throughput Frontier of Sparse Attention with Netpreme X-Mem", modelled
// study: 2,048 entries are picked per layer and step).
//
// Scan kernel (scan_core.cuh's pipeline, this epilogue): each block walks a
// contiguous range of chunks; the part of one (request, KV head) row inside a
// block is a "segment". Per segment the block appends to a buffer in L2 every
// key whose score is at least a running threshold tau (all keys, until a
// threshold exists), as (order-preserving score key, index). When the buffer
// may not hold another chunk, two histogram passes over the held keys (bits
// 31..21, then 20..10) find the cell holding the k-th largest key; tau becomes
// that cell's lower edge and every held key below it is dropped. The held set
// always contains the segment's top-k (at least k keys are >= tau), so nothing
// of the answer is ever lost; it is a superset, trimmed again at the segment's
// end (and cut exactly to k only if it would still be too large).
//
// Merge kernel: one block per row gathers its segments' candidates as
// distinct 53-bit composites (score key << 21 | (2^21 - 1 - index)), selects
// exactly the k largest (radix passes), emits their indices in ascending order
// through a bitmap over the row, and looks every selected key up in the
// hot-buffer slot map (slots; misses = the number absent from the hot buffer).
#include "internal.cuh"
#include "scan_core.cuh"
#include "scan_prmt.cuh"

namespace kvs {

namespace {

constexpr int kIdxBits = 21;
constexpr uint32_t kIdxMask = (1u << kIdxBits) - 1u;
constexpr int kCandCap = 16384;  // per-block candidate buffer entries in global memory
constexpr int kPCandCap = 24576; // per-segment candidates of the byte-indexed fused scan

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

// ---------------------------------------------------------------------------
// Fused scan + top-k on the byte-indexed lookup core (plans of <= 144 planes).
//
// The eight scoring warps only write each chunk's 4,096 scores into the
// consumed stage slot (scan_prmt.cuh, staged mode); four selector warps, one
// per scheduler, read them there (two scoring warps' bands each) and keep the
// segment's candidates, so the latency of the selection never stalls the
// scoring warps. A segment's candidates are appended straight into its output
// region (capacity kPCandCap) as (order-preserving score key, index): a lane
// marks which of its 32 scores are at or above the running threshold tau, the
// warp takes its positions with one shuffle scan and one shared atomic, and
// only the marked scores are read again and written.
//
// tau: the segment's first chunk (when it holds >= k valid keys) is binned
// linearly over [min, max] of its scores into 2048 bins; tau becomes the
// smallest score in the bin holding the k-th largest, so exactly the keys of
// that bin and above are held. Every later appended key is counted in its
// bin. Whenever the held count has grown by k/4 since the last raise, the one
// selector warp that moves the raise mark (a compare-and-swap) finds the bin b
// holding the k-th largest held key and raises tau to the lower edge of bin
// b - 1 (one bin of margin against rounding). The counts it reads may lag
// appends still in flight, so they are lower bounds: at least k held keys are
// >= tau at all times and the held set is a superset of the segment's top-k.
// A segment of n keys appends about k (1 + ln(n / 4096)) keys (~9,000 for
// 113K keys, ~10,500 for 230K). Every second chunk the selectors check the
// fill; near capacity (ties, degenerate ranges) the held set is cut to exactly
// the k best by (score, index) and, since later keys have larger indices, only
// keys strictly above the k-th score are appended afterwards. The segment's
// final tau is stored beside its count; the merge drops entries below it.
struct SelStateP {
  int cnt, tau_set, strict, hist_on, next_raise;
  float tau_f, lo, w, inv_w;
  float red_min[kPSel], red_max[kPSel];
  SelectState sel;
};

__device__ __forceinline__ int score_bin(float s, float lo, float inv_w) {
  return min(2047, max(0, static_cast<int>((s - lo) * inv_w)));
}

// One warp: the bin holding the k-th largest count of hist (from the top), or
// -1 when the histogram holds fewer than k. Lane l first sums bins
// [2048 - 64 (l + 1), 2048 - 64 l) (16-byte reads in a lane-rotated order),
// then the lane holding the rank is resolved two bins per lane.
__device__ __forceinline__ int warp_kth_bin(const unsigned* hist, int k, int lane) {
  const uint4* h4 = reinterpret_cast<const uint4*>(hist);
  const int q0 = 512 - 16 * (lane + 1);
  unsigned sum = 0;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint4 v = h4[q0 + ((e + lane) & 15)];
    sum += v.x + v.y + v.z + v.w;
  }
  unsigned incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const unsigned o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += o;
  }
  const unsigned hit = __ballot_sync(0xFFFFFFFFu, incl >= static_cast<unsigned>(k));
  if (hit == 0u) return -1;
  const int L = __ffs(hit) - 1;
  const unsigned krem = static_cast<unsigned>(k) - __shfl_sync(0xFFFFFFFFu, incl - sum, L);
  const int b_hi = 2048 - 64 * L - 1 - 2 * lane;
  const unsigned c_hi = hist[b_hi], c_lo = hist[b_hi - 1];
  const unsigned c2 = c_hi + c_lo;
  unsigned incl2 = c2;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const unsigned o = __shfl_up_sync(0xFFFFFFFFu, incl2, d);
    if (lane >= d) incl2 += o;
  }
  const unsigned hit2 = __ballot_sync(0xFFFFFFFFu, incl2 >= krem);
  const int l2 = hit2 ? __ffs(hit2) - 1 : 31;
  const unsigned before = __shfl_sync(0xFFFFFFFFu, incl2 - c2, l2);
  const unsigned top_cnt = __shfl_sync(0xFFFFFFFFu, c_hi, l2);
  const int bb = 2048 - 64 * L - 1 - 2 * l2;
  return before + top_cnt >= krem ? bb : bb - 1;
}

// Barrier of the selector warps only; and the same returning the OR of a predicate.
__device__ __forceinline__ void sel_sync() {
  asm volatile("bar.sync 2, %0;\n" ::"n"(32 * kPSel) : "memory");
}
__device__ __forceinline__ bool sel_sync_or(bool pred) {
  int r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.s32 p, %1, 0;\n bar.red.or.pred q, 2, %2, p;\n"
      " selp.s32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(pred ? 1 : 0), "n"(32 * kPSel)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kPThreadsStaged, 1) fathom_scan_topk_prmt_kernel(ScanParams p) {
  using Core = ScanCoreP<true>;
  Core core(p);
  unsigned* hist = reinterpret_cast<unsigned*>(core.extra());
  SelStateP* st = reinterpret_cast<SelStateP*>(hist + 2048);
  volatile SelStateP* vst = st;
  core.run([](int, int, int, const float (&)[kPKeys], int, unsigned char*) {}, [&](int beg, int end) {
    constexpr int NS = 32 * kPSel;
    constexpr int CK = 32 * kPChunkWords;  // keys per chunk
    const int lane = threadIdx.x & 31;
    const int sw = (threadIdx.x >> 5) - (kPWarps + kPProd);
    const int tid = 32 * sw + lane;
    const long long C = static_cast<long long>(p.RG) * p.chunks_per_row;
    const int last_chunk = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * C / gridDim.x) - 1;
    const int raise_step = max(256, p.k / 4);
    const float pinf = __int_as_float(0x7f800000), ninf = -pinf;
    // lane's place in a chunk: iteration e reads row 4e + (lane >> 3), 16 bytes
    // q4 = lane & 7 of this warp's 128-byte part (scoring warps 2 sw, 2 sw + 1)
    const int q4 = lane & 7;
    const int cw = 2 * sw + (q4 >> 2);  // scoring warp whose scores these are
    int u = beg / p.chunks_per_row, c = beg % p.chunks_per_row, stg = 0;
    uint32_t phase = 0u;
    int chunk_i = 0, seg_u = -1;
    size_t seg = 0;
    bool fresh = false, dead = false;
    for (int it = beg; it < end; ++it) {
      const int nr = p.n[u / p.Gheads];
      if (u != seg_u) {
        seg = static_cast<size_t>(u) * p.segs_per_row +
              (static_cast<int>(blockIdx.x) -
               block_of_chunk(static_cast<long long>(u) * p.chunks_per_row, C, gridDim.x));
        seg_u = u;
        fresh = true;
        if (tid == 0) {
          st->cnt = 0;
          st->tau_set = 0;
          st->strict = 0;
          st->hist_on = 0;
        }
        sel_sync();
      }
      if (!dead && !mbar_wait(&core.scored[stg], phase)) {
        core.fail_timeout();
        dead = true;
      }
      unsigned char* slot = g_scan_smem + core.stage0 + stg * core.slot_bytes;
      uint32_t* kb = p.cand_key + seg * p.seg_cap;
      int32_t* ib = p.cand_idx + seg * p.seg_cap;
      // this lane's 32 scores and their validity; score j is key
      // kbase0 + 64 (j >> 2) + (j & 3)
      const int kbase0 = 32 * (c * kPChunkWords + 16 * cw + (lane >> 4)) + 16 * ((lane >> 3) & 1) + 4 * (q4 & 3);
      float4 v[8];
      uint32_t valid = 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = 4 * e + (lane >> 3);
        v[e] = *reinterpret_cast<const float4*>(slot + r * kPRowBytes + 128 * sw + 16 * q4);
        const int nv = nr - (kbase0 + 64 * e);
        valid |= (nv >= 4 ? 15u : (nv <= 0 ? 0u : ((1u << nv) - 1u))) << (4 * e);
      }
      auto score = [&](int j) -> float {
        const float4 f = v[j >> 2];
        const int cc = j & 3;
        return cc == 0 ? f.x : (cc == 1 ? f.y : (cc == 2 ? f.z : f.w));
      };
      // 0. the segment's first chunk: tau from its own scores (its held keys are
      // then already counted in the histogram)
      bool binned_now = false;
      if (fresh) {
        fresh = false;
        if (nr - 32 * c * kPChunkWords >= p.k) {
          float mn = pinf, mx = ninf;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if ((valid >> j) & 1u) {
              mn = fminf(mn, score(j));
              mx = fmaxf(mx, score(j));
            }
          for (int d = 16; d > 0; d >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, d));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
          }
          if (lane == 0) {
            st->red_min[sw] = mn;
            st->red_max[sw] = mx;
          }
          for (int b = tid; b < 2048; b += NS) hist[b] = 0;
          sel_sync();
          float lo = st->red_min[0], hi = st->red_max[0];
#pragma unroll
          for (int q = 1; q < kPSel; ++q) {
            lo = fminf(lo, st->red_min[q]);
            hi = fmaxf(hi, st->red_max[q]);
          }
          const float w = (hi - lo) * (1.0f / 2048.0f);
          const float mag = fmaxf(fabsf(lo), fabsf(hi));
          // bins are usable when one bin is well above the rounding of scores
          if (hi > lo && w > 16.0f * mag * 5.96e-8f) {  // the same in every selector thread
            const float inv_w = 2048.0f / (hi - lo);
            binned_now = true;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if ((valid >> j) & 1u) atomicAdd(&hist[score_bin(score(j), lo, inv_w)], 1u);
            sel_sync();
            const int bstar = warp_kth_bin(hist, p.k, lane);  // the same in every warp
            // tau = the smallest score in bin bstar (exact: bins are monotone in the score)
            float bmin = pinf;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (((valid >> j) & 1u) && score_bin(score(j), lo, inv_w) == bstar) bmin = fminf(bmin, score(j));
            for (int d = 16; d > 0; d >>= 1) bmin = fminf(bmin, __shfl_xor_sync(0xFFFFFFFFu, bmin, d));
            sel_sync();  // every warp has read the histogram
            // the held keys are exactly bins >= bstar: clear the rest of the histogram
            for (int b = tid; b < bstar; b += NS) hist[b] = 0;
            if (lane == 0) st->red_min[sw] = bmin;
            sel_sync();
            if (tid == 0) {
              float tm = st->red_min[0];
              for (int q = 1; q < kPSel; ++q) tm = fminf(tm, st->red_min[q]);
              st->tau_f = tm;
              st->tau_set = 1;
              st->hist_on = 1;
              st->lo = lo;
              st->w = w;
              st->inv_w = inv_w;
              st->next_raise = p.k + raise_step;
            }
            sel_sync();
          }
        }
      }

      // 1. keys at or above tau join the segment's candidates
      const bool count_bins = vst->hist_on != 0 && !binned_now;
      float tau = ninf;
      if (vst->tau_set) {
        tau = vst->tau_f;
        if (vst->strict) tau = nextafterf(tau, pinf);  // strictly above the cut's k-th score
      }
      uint32_t mask = 0u;
#pragma unroll
      for (int j = 0; j < 32; ++j) mask |= score(j) >= tau ? (1u << j) : 0u;
      mask &= valid;
      // appends, in two halves of 16 keys per lane: lane L first writes its
      // passing (score, key) pairs densely into row L of this warp's part of
      // the slot (128 bytes: 16 pairs; its scores are in registers now), then
      // the warp writes them out one pair per lane (each lane finds the pair's
      // source lane by binary search over the lanes' offsets), with one shared
      // atomic per half for their positions
      __syncwarp();
      int new_cnt = -1;
      unsigned char* mine = slot + lane * kPRowBytes + 128 * sw;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t hm = (mask >> (16 * half)) & 0xFFFFu;
        const int cnt = __popc(hm);
        int incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
          if (lane >= d) incl += o;
        }
        const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        if (total == 0) continue;
        uint32_t woff = 0u;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int j = 16 * half + jj;
          if ((hm >> jj) & 1u) {
            *reinterpret_cast<uint2*>(mine + woff) = make_uint2(
                __float_as_uint(score(j)), static_cast<uint32_t>(kbase0 + 64 * (j >> 2) + (j & 3)));
            woff += 8u;
          }
        }
        int base = 0;
        if (lane == 0) base = atomicAdd(&st->cnt, total);
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        new_cnt = base + total;
        const int excl = incl - cnt;
        __syncwarp();
        const float lo = st->lo, inv_w = st->inv_w;
        for (int f0 = 0; f0 < total; f0 += 32) {
          const int f = f0 + lane;
          // source lane: the last lane whose exclusive offset is <= f
          int src = 0;
#pragma unroll
          for (int step = 16; step > 0; step >>= 1) {
            const int probe = src + step;
            if (__shfl_sync(0xFFFFFFFFu, excl, probe) <= f) src = probe;
          }
          const int rank = f - __shfl_sync(0xFFFFFFFFu, excl, src);
          if (f < total) {
            const uint2 e = *reinterpret_cast<const uint2*>(slot + src * kPRowBytes + 128 * sw + 8 * rank);
            const float sc = __uint_as_float(e.x);
            if (base + f < p.seg_cap) {
              kb[base + f] = ordered_key(sc);
              ib[base + f] = static_cast<int32_t>(e.y);
            }
            if (count_bins) atomicAdd(&hist[score_bin(sc, lo, inv_w)], 1u);
          }
        }
        __syncwarp();
      }
      // the warp that moves the raise mark raises tau from the histogram
      if (count_bins && new_cnt >= 0) {
        int won = 0;
        if (lane == 0) {
          const int mark = vst->next_raise;
          won = new_cnt >= mark && atomicCAS(&st->next_raise, mark, new_cnt + raise_step) == mark;
        }
        if (__shfl_sync(0xFFFFFFFFu, won, 0)) {
          const int b = warp_kth_bin(hist, p.k, lane);
          if (lane == 0 && b >= 1) {
            const float edge = st->lo + static_cast<float>(b - 1) * st->w;
            if (edge > vst->tau_f) vst->tau_f = edge;
          }
        }
      }

      // the slot goes back to the producers; rows that are padding planes
      // (B < 32) must be zero again
      if (p.B < 32) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (4 * e + (lane >> 3) >= p.B)
            *reinterpret_cast<float4*>(slot + (4 * e + (lane >> 3)) * kPRowBytes + 128 * sw + 16 * q4) =
                make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncwarp();
      if (!dead && lane == 0) mbar_arrive(&core.empty[stg]);

      // 3. at the segment's end (publish), and every second chunk (the buffer
      // may take two more chunks of appends before it must be cut)
      const bool seg_end = c == p.chunks_per_row - 1 || u * p.chunks_per_row + c == last_chunk;
      if (seg_end || (chunk_i & 1)) {
        sel_sync();  // every warp's appends of this chunk are done
        // one decision for all: the count is read after the barrier, and no warp
        // appends again before every thread has read it
        if (sel_sync_or(!seg_end && st->cnt > p.seg_cap - 2 * CK)) {
          // exact cut to the k best by (score key, index)
          const int n = st->cnt;
          uint64_t* comp = p.cbuf_comp + static_cast<size_t>(blockIdx.x) * p.seg_cap;
          for (int i = tid; i < n; i += NS) comp[i] = make_composite(kb[i], ib[i]);
          sel_sync();
          const int kk = min(p.k, n);
          const uint64_t thr = select_kth_composite(comp, n, kk, hist, &st->sel, tid, NS, sel_sync);
          if (tid == 0) st->cnt = 0;
          sel_sync();
          for (int b0 = 0; b0 < n; b0 += NS) {
            const int i = b0 + tid;
            const uint64_t cv = i < n ? comp[i] : 0ull;
            const bool take = i < n && cv >= thr;
            const unsigned m = __ballot_sync(0xFFFFFFFFu, take);
            if (m == 0u) continue;
            const int leader = __ffs(m) - 1;
            int pos = 0;
            if (lane == leader) pos = atomicAdd(&st->cnt, __popc(m));
            pos = __shfl_sync(0xFFFFFFFFu, pos, leader) + __popc(m & ((1u << lane) - 1u));
            if (take) {
              kb[pos] = static_cast<uint32_t>(cv >> kIdxBits);
              ib[pos] = composite_index(cv);
            }
          }
          sel_sync();
          if (tid == 0) {
            st->tau_f = key_to_float(static_cast<uint32_t>(thr >> kIdxBits));
            st->tau_set = 1;
            st->strict = 1;
            st->hist_on = 0;
          }
          sel_sync();
        }
        if (seg_end) {
          if (tid == 0) {
            p.cand_count[seg] = min(st->cnt, p.seg_cap);
            p.cand_tau[seg] = st->tau_set ? ordered_key(st->tau_f) : 0u;
          }
          sel_sync();
        }
      }
      ++chunk_i;
      if (++c == p.chunks_per_row) {
        c = 0;
        ++u;
      }
      if (++stg == core.nstage) {
        stg = 0;
        phase ^= 1u;
      }
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
  __shared__ int seg_count[64], seg_off[65];
  __shared__ uint32_t seg_tau[64];
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
  const int segs = b1 - b0 + 1;
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
  int grid, cpr, segs, seg_cap;
};

// Plans of <= 144 planes run the byte-indexed core, whose segments hold up to
// kPCandCap candidates each; longer plans the group-table core (2k each).
Layout fused_layout(int RG, int n_max, int k, int B) {
  Layout L{};
  if (B <= kPMaxB) {
    L.cpr = prmt_chunks_per_row(n_max);
    L.seg_cap = kPCandCap;
  } else {
    int G, b, nsets;
    scan_schedule(B, G, b, nsets);
    L.cpr = scan_chunks_per_row(n_max, scan_warps(G, b));
    L.seg_cap = 2 * k;
  }
  L.grid = fused_grid(RG, L.cpr);
  L.segs = L.grid > 0 ? fused_segs_per_row(RG, L.cpr, L.grid) : 1;
  return L;
}

constexpr size_t kPFusedExtra = 2048 * sizeof(unsigned) + sizeof(SelStateP);

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

size_t fused_ws_bytes(int RG, int n_max, int k, int B) {
  const Layout L = fused_layout(RG, n_max, k, B);
  WsCarver c(nullptr);
  const size_t cap = static_cast<size_t>(kCandCap > L.seg_cap ? kCandCap : L.seg_cap);
  c.take<uint32_t>(static_cast<size_t>(L.grid) * kCandCap);
  c.take<int32_t>(static_cast<size_t>(L.grid) * kCandCap);
  c.take<uint64_t>(static_cast<size_t>(L.grid) * cap);
  c.take<uint32_t>(static_cast<size_t>(RG) * L.segs * L.seg_cap);
  c.take<int32_t>(static_cast<size_t>(RG) * L.segs * L.seg_cap);
  c.take<int32_t>(static_cast<size_t>(RG) * L.segs);
  c.take<uint32_t>(static_cast<size_t>(RG) * L.segs);
  c.take<uint64_t>(static_cast<size_t>(RG) * L.segs * L.seg_cap);
  c.take<uint32_t>(static_cast<size_t>(RG) * bitmap_words(n_max));
  return c.used;
}

kvs_status fathom_scan_topk_launch(ScanParams p, void* ws, const int32_t* slot_map, int32_t* idx,
                                   int32_t* slots, int32_t* misses, cudaStream_t s,
                                   cudaEvent_t after_scan) {
  const Layout L = fused_layout(p.RG, p.n_max, p.k, p.B);
  if (L.grid <= 0) return KVS_OK;
  if (L.segs > 64) return fail(KVS_EUNSUPPORTED, "decode_step: %d segments per row", L.segs);
  p.chunks_per_row = L.cpr;
  p.segs_per_row = L.segs;
  p.seg_cap = L.seg_cap;
  WsCarver c(ws);
  const size_t cap = static_cast<size_t>(kCandCap > L.seg_cap ? kCandCap : L.seg_cap);
  p.cbuf_key = c.take<uint32_t>(static_cast<size_t>(L.grid) * kCandCap);
  p.cbuf_idx = c.take<int32_t>(static_cast<size_t>(L.grid) * kCandCap);
  p.cbuf_comp = c.take<uint64_t>(static_cast<size_t>(L.grid) * cap);
  p.cand_key = c.take<uint32_t>(static_cast<size_t>(p.RG) * L.segs * L.seg_cap);
  p.cand_idx = c.take<int32_t>(static_cast<size_t>(p.RG) * L.segs * L.seg_cap);
  p.cand_count = c.take<int32_t>(static_cast<size_t>(p.RG) * L.segs);
  p.cand_tau = c.take<uint32_t>(static_cast<size_t>(p.RG) * L.segs);
  uint64_t* gscratch = c.take<uint64_t>(static_cast<size_t>(p.RG) * L.segs * L.seg_cap);
  uint32_t* bitmap = c.take<uint32_t>(static_cast<size_t>(p.RG) * bitmap_words(p.n_max));
  kvs_status st;
  if (p.B <= kPMaxB) {
    p.nstage = prmt_nstages(p.B, kPFusedExtra);
    if (p.nstage < 2) return fail(KVS_EUNSUPPORTED, "decode_step: no room for two stages at B=%d", p.B);
    const size_t smem = prmt_smem_bytes(p.B, p.nstage, kPFusedExtra);
    cudaFuncSetAttribute(fathom_scan_topk_prmt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    fathom_scan_topk_prmt_kernel<<<L.grid, kPThreadsStaged, smem, s>>>(p);
    st = check_launch("decode_step(scan+topk, prmt)");
  } else {
    p.cand_tau = nullptr;
    st = dispatch_schedule(p, FusedLaunch{p, L.grid, s});
  }
  if (st != KVS_OK) return st;
  if (after_scan) cudaEventRecord(after_scan, s);
  const size_t msmem = static_cast<size_t>(kMergeSmemEntries) * sizeof(uint64_t);
  cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(msmem));
  topk_merge_kernel<<<p.RG, kMergeThreads, msmem, s>>>(p, L.grid, gscratch, bitmap, slot_map, idx,
                                                        slots, misses);
  return check_launch("decode_step(top-k merge)");
}

}  // namespace kvs
