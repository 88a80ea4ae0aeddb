// scan_core.cuh -- the warp-specialised core of the HBM Fathom scan (see
// scan_lut.cu for the method): TMA bulk staging of plane segments, in-register
// bit transposes, and bank-rotated group lookup tables. The epilogue (write
// scores, or keep top-k candidates) is supplied by the kernel.
#pragma once

#include "internal.cuh"

namespace kvs {

constexpr int kKeysPerThread = 16;              // half of a 32-key word per consumer thread
constexpr int kMaxScanWarps = 12;               // consumer warps per block, at most
constexpr long long kWaitCycles = 2000000000ll;  // ~1 s bound on every wait

struct ScanParams {
  const uint32_t* planes;  // [RG][D][4][W]
  int W;
  int RG, Gheads;  // rows (r, g), and KV heads per request (row u belongs to request u / Gheads)
  const uint16_t* plane_idx;  // [RG][B]
  const float* plane_w;       // [RG][B]
  const float* C;             // [RG]
  int B;
  const int32_t* n;
  int n_max;
  int G, b, nsets;  // lookup schedule: G groups of b planes per set
  int warps;        // consumer warps per block (8 or 12); a chunk is 16 * warps words
  int chunks_per_row;
  float* scores;  // unfused output [RG][n_max]
  float* gmax;    // optional: max score of each 16-key group [RG][ceil(n_max / 16)] (-inf if none valid)
  int32_t* dev_status;
  int nstage;  // pipeline depth (set by the launcher from the shared memory budget)
  // fused top-k candidates (scan_topk.cu)
  int k;
  int segs_per_row, seg_cap;  // candidate lists per row, and entries per list
  int lists_per_seg;          // lists of one (block, row) segment: 1, or one per scoring warp
  int cand_cap, trim_at;  // per-block candidate capacity, and the count that triggers a trim
  uint32_t* cbuf_key;   // [grid][2][cap] per-block candidate buffers: score keys
  int32_t* cbuf_idx;    //                                             indices
  uint64_t* cbuf_comp;  // [grid][cap] scratch for an exact cut
  uint32_t* cand_key;   // [RG][segs][seg_cap] per-segment candidates
  int32_t* cand_idx;
  int32_t* cand_count;  // [RG][segs]
  uint32_t* cand_tau;   // [RG][segs] score key below which a segment's entries are not needed
  // the bound of every wait in cycles (0: kWaitCycles), and a self-test switch:
  // producer warp 0 of every block withholds its arrival on its first chunk,
  // so that the consumers' wait for that chunk runs out (kvs_selftest_scan_timeout)
  long long wait_cycles;
  int withhold_arrive;
};

// Picks the lookup schedule for a budget of B planes: the fewest groups per
// set with tables of at most 2^9 entries.
inline void scan_schedule(int B, int& G, int& b, int& nsets) {
  if (B <= 72) {
    G = 8;
    b = B <= 0 ? 1 : (B + 7) / 8;
    nsets = 1;
  } else if (B <= 144) {
    G = 16;
    b = (B + 15) / 16;
    nsets = 1;
  } else {
    G = 16;
    b = 6;
    nsets = (B + 95) / 96;
  }
}

// Consumer warps for a schedule: 12 when two pipeline stages of 12 warps'
// chunks still fit next to the tables (every schedule but 16 groups of 8 or 9
// planes), else 8. More warps hide more of the scan's latency.
__host__ __device__ constexpr int scan_warps(int G, int b) { return (G == 16 && b >= 8) ? 8 : 12; }

inline int scan_chunks_per_row(int n_max, int warps) {
  const int words = (n_max + 31) / 32;
  const int cw = 16 * warps;
  return (words + cw - 1) / cw;
}

// Register budget of the scan kernels: one block per SM. 128 registers a
// thread hold every schedule without spills and timed no slower than the
// whole file the block size leaves (B = 92 and 136 at 128K keys a row).
#ifndef KVS_SCAN_MAXNREG
#define KVS_SCAN_MAXNREG 128
#endif
#define KVS_SCAN_BOUNDS(G, b, W) __maxnreg__(KVS_SCAN_MAXNREG)

// A zero plane segment in global memory: the source of padding slots.
__device__ __align__(16) uint32_t kZeroRow[16 * kMaxScanWarps];

// Dynamic shared memory of the scan kernels: [tables | stages | barriers |
// epilogue scratch]. Indexing this symbol directly keeps every table lookup a
// shared-memory load with the base folded into the address.
extern __shared__ __align__(1024) unsigned char g_scan_smem[];

// ----------------------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a phase: false when `limit` cycles (about one second by
// default) pass without it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
// Barrier of the consumer warps only (the producer warp does not take part).
template <int W>
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(32 * W) : "memory");
}

// Half of a 32x32 bit transpose, in registers. On entry x[k] holds, for one
// 16-key half of a word, the 16 bits of plane k in its low half and those of
// plane k + 16 in its high half (the first, 16-bit stage of the full
// transpose, done by the loads). On exit bit c of x[r] is plane c's bit for
// key r of the half. One byte-permute stage and three shift/select stages.
__device__ __forceinline__ void transpose16(uint32_t (&x)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (k & 8) continue;
    const uint32_t a = x[k], c = x[k + 8];
    x[k] = __byte_perm(a, c, 0x6240);
    x[k + 8] = __byte_perm(a, c, 0x7351);
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (k & 4) continue;
    const uint32_t t = ((x[k] >> 4) ^ x[k + 4]) & 0x0F0F0F0Fu;
    x[k + 4] ^= t;
    x[k] ^= t << 4;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (k & 2) continue;
    const uint32_t t = ((x[k] >> 2) ^ x[k + 2]) & 0x33333333u;
    x[k + 2] ^= t;
    x[k] ^= t << 2;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (k & 1) continue;
    const uint32_t t = ((x[k] >> 1) ^ x[k + 1]) & 0x55555555u;
    x[k + 1] ^= t;
    x[k] ^= t << 1;
  }
}

template <int G, int b, int W>
struct ScanCore {
  static constexpr int THREADS = 32 * (W + 1);   // W consumer warps + one producer warp
  static constexpr int CHUNK_WORDS = 16 * W;     // two consumer threads per 32-key word
  static constexpr int ROW_BYTES = 4 * CHUNK_WORDS;
  static constexpr int NPOS = G * b;             // plane slots per set
  static constexpr int NBLK = (NPOS + 31) / 32;  // 32-plane transposes per set
  static constexpr int TBL_BYTES = (1 << b) * 128;
  static constexpr int STAGE_BYTES = NPOS * ROW_BYTES;

  // layout: [tables | nstage stages | 256 bytes of barriers | extra], within
  // the 227 KB of dynamic shared memory a block may opt in to on sm_100
  static int nstages(int nsets, size_t extra = 0) {
    const int budget = 227 * 1024 - nsets * TBL_BYTES - 256 - static_cast<int>(extra);
    const int s = budget / STAGE_BYTES;
    return s > 4 ? 4 : s;
  }
  static size_t smem_bytes(int nsets, size_t extra = 0) {
    return static_cast<size_t>(nsets) * TBL_BYTES +
           static_cast<size_t>(nstages(nsets, extra)) * STAGE_BYTES + 256 + extra;
  }

  const ScanParams& p;
  int nstage;
  unsigned char* stages;
  uint64_t* full;
  uint64_t* empty;
  int* abort_flag;

  __device__ explicit ScanCore(const ScanParams& params) : p(params) {
    nstage = p.nstage;
    stages = g_scan_smem + p.nsets * TBL_BYTES;
    full = reinterpret_cast<uint64_t*>(stages + nstage * STAGE_BYTES);
    empty = full + nstage;
    abort_flag = reinterpret_cast<int*>(empty + nstage);
  }

  __device__ unsigned char* extra() const {
    return g_scan_smem + p.nsets * TBL_BYTES + nstage * STAGE_BYTES + 256;
  }

  __device__ void fail_timeout() {
    set_status(p.dev_status, KVS_ETIMEOUT);
    atomicExch(abort_flag, 1);
  }

  // item -> (row u, chunk c, set s)
  __device__ void decode_item(int it, int& u, int& c, int& s) const {
    s = it % p.nsets;
    const int rc = it / p.nsets;
    c = rc % p.chunks_per_row;
    u = rc / p.chunks_per_row;
  }

  __device__ void produce(int beg, int end) {
    const int lane = threadIdx.x & 31;
    int issued = 0;
    for (int it = beg; it < end; ++it) {
      const int k = it - beg, st = k % nstage;
      if (k >= nstage && !mbar_wait(&empty[st], ((k / nstage) - 1) & 1)) {
        if (lane == 0) fail_timeout();
        break;
      }
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      int u, c, s;
      decode_item(it, u, c, s);
      const int w0 = c * CHUNK_WORDS;
      const int nr = p.n[u / p.Gheads];
      const bool live = 32 * w0 < nr;
      const int words = min(CHUNK_WORDS, p.W - w0);
      const uint32_t bytes = live ? static_cast<uint32_t>(words) * 4u : 0u;
      if (lane == 0) mbar_expect_tx(&full[st], bytes * NPOS);
      __syncwarp();
      if (live) {
        unsigned char* dst0 = stages + st * STAGE_BYTES;
        const uint32_t* rowp = p.planes + static_cast<size_t>(u) * kD * 4 * p.W + w0;
        const uint16_t* pidx = p.plane_idx + static_cast<size_t>(u) * p.B;
        for (int q = lane; q < NPOS; q += 32) {
          const int slot = s * NPOS + q;
          const uint32_t* src =
              slot < p.B ? rowp + static_cast<size_t>(pidx[slot]) * p.W : kZeroRow;
          bulk_g2s(dst0 + q * ROW_BYTES, src, bytes, &full[st]);
        }
      }
      ++issued;
    }
    // drain: never leave copies in flight into this block's shared memory
    for (int k = max(0, issued - nstage); k < issued; ++k)
      mbar_wait(&full[k % nstage], (k / nstage) & 1);
  }

  __device__ void build_tables(int u) {
    const int t = threadIdx.x;
    const float* w = p.plane_w + static_cast<size_t>(u) * p.B;
    const int entries = p.nsets * (1 << b) * 32;
    for (int e = t; e < entries; e += 32 * W) {
      const int slot = e & 31;
      const int idx = (e >> 5) & ((1 << b) - 1);
      const int s = e >> (5 + b);
      const int base = s * NPOS + (slot % G) * b;
      float v = 0.f;
#pragma unroll
      for (int bi = 0; bi < b; ++bi)
        if (((idx >> bi) & 1) && base + bi < p.B) v += w[base + bi];
      *reinterpret_cast<float*>(g_scan_smem + s * TBL_BYTES + idx * 128 + slot * 4) = v;
    }
  }

  // Offset of stream position o (a static plane slot of the set) for a lane
  // whose planes are rotated by lp groups.
  __device__ __forceinline__ static int slot_offset(int o, int lp) {
    const int g = o / b, bi = o % b;
    return (((g + lp) & (G - 1)) * b + bi) * ROW_BYTES;
  }

  // The set's contribution for this thread's 16 keys, added into acc. Thread
  // t handles half (t & 1) of word (t >> 1) of the chunk: it reads that 16-bit
  // half of each plane word and transposes a 32-plane x 16-key block.
  __device__ __forceinline__ void compute_set(int stage_off, int s, float (&acc)[kKeysPerThread]) const {
    constexpr int NK = kKeysPerThread;
    const int t = threadIdx.x;
    const int lane = t & 31;
    // The two threads of a word share one rotation (so their plane loads hit
    // the same word of a bank) and use different replicas of the tables: pair
    // i = lane / 2 rotates by i mod G, and the 32 (rotation, replica)
    // combinations of a warp are 32 distinct banks.
    const int pair = lane >> 1;
    const int lp = pair % G;
    const int repl = (lane & 1) + 2 * (pair / G);
    const unsigned char* mine = g_scan_smem + stage_off + 4 * (t >> 1) + 2 * (t & 1);
    uint32_t prev[NK];
#pragma unroll
    for (int j = 0; j < NK; ++j) prev[j] = 0u;
#pragma unroll
    for (int m = 0; m < NBLK; ++m) {
      uint32_t x[NK];
#pragma unroll
      for (int q = 0; q < NK; ++q) {
        const int o1 = 32 * m + q, o2 = o1 + 16;
        const uint32_t lo =
            o1 < NPOS ? *reinterpret_cast<const uint16_t*>(mine + slot_offset(o1, lp)) : 0u;
        const uint32_t hi =
            o2 < NPOS ? *reinterpret_cast<const uint16_t*>(mine + slot_offset(o2, lp)) : 0u;
        x[q] = __byte_perm(lo, hi, 0x5410);
      }
      transpose16(x);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int st = g * b, en = st + b - 1;
        if ((en >> 5) != m) continue;
        const int sh = st & 31;
        const bool straddle = (st >> 5) != m;
        const uint32_t rs = static_cast<uint32_t>((((g + lp) & (G - 1)) + G * repl) * 4 +
                                                  s * TBL_BYTES);
        constexpr uint32_t mask7 = ((1u << b) - 1u) << 7;
#pragma unroll
        for (int j = 0; j < NK; ++j) {
          uint32_t v;
          if (straddle)
            v = __funnelshift_r(prev[j], x[j], sh - 7);
          else if (sh >= 7)
            v = x[j] >> (sh - 7);
          else
            v = x[j] << (7 - sh);
          const uint32_t addr = (v & mask7) | rs;
          acc[j] += *reinterpret_cast<const float*>(g_scan_smem + addr);
        }
      }
#pragma unroll
      for (int j = 0; j < NK; ++j) prev[j] = x[j];
    }
  }

  // Runs the pipeline over this block's chunks; epi(u, c, nr, acc, t) is
  // called by every consumer thread at the end of each chunk c of row u.
  template <typename Epi>
  __device__ void run(Epi&& epi) {
    // whole chunks per block: the sets of a chunk accumulate in one thread
    const int chunks = p.RG * p.chunks_per_row;
    const int cbeg = static_cast<int>(static_cast<long long>(blockIdx.x) * chunks / gridDim.x);
    const int cend = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * chunks / gridDim.x);
    const int beg = cbeg * p.nsets, end = cend * p.nsets;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
      for (int i = 0; i < nstage; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], W);
      }
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (warp == W) {
      produce(beg, end);
      return;
    }
    // Consumers never leave early: after a timed-out wait they stop working
    // but keep stepping through the same items, so that every named barrier
    // (here and in the epilogue) is still met by all of them.
    int cur_u = -1, row_n = 0;
    float row_C = 0.f;
    bool dead = false;
    float acc[kKeysPerThread];
    for (int it = beg; it < end; ++it) {
      const int k = it - beg, st = k % nstage;
      int u, c, s;
      decode_item(it, u, c, s);
      if (u != cur_u) {
        consumer_sync<W>();
        if (!dead) build_tables(u);
        row_n = p.n[u / p.Gheads];
        row_C = p.C[u];
        consumer_sync<W>();
        cur_u = u;
      }
      const int nr = row_n;
      const int w0 = c * CHUNK_WORDS;
      if (s == 0) {
#pragma unroll
        for (int j = 0; j < kKeysPerThread; ++j) acc[j] = row_C;
      }
      if (!dead && !mbar_wait(&full[st], (k / nstage) & 1)) {
        fail_timeout();
        dead = true;
      }
      if (!dead) {
        if (32 * w0 < nr) compute_set(p.nsets * TBL_BYTES + st * STAGE_BYTES, s, acc);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[st]);
      }
      if (s == p.nsets - 1) epi(u, c, nr, acc, static_cast<int>(threadIdx.x));
    }
  }
};

// Calls f.template operator()<G, b, W>() for the schedule of p (G, b, warps).
template <typename F>
kvs_status dispatch_schedule(const ScanParams& p, F&& f) {
#define KVS_SCHED(GG, BB) \
  if (p.G == GG && p.b == BB) return f.template operator()<GG, BB, scan_warps(GG, BB)>();
  KVS_SCHED(8, 1) KVS_SCHED(8, 2) KVS_SCHED(8, 3) KVS_SCHED(8, 4) KVS_SCHED(8, 5)
  KVS_SCHED(8, 6) KVS_SCHED(8, 7) KVS_SCHED(8, 8) KVS_SCHED(8, 9)
  KVS_SCHED(16, 5) KVS_SCHED(16, 6) KVS_SCHED(16, 7) KVS_SCHED(16, 8) KVS_SCHED(16, 9)
#undef KVS_SCHED
  return fail(KVS_EUNSUPPORTED, "index_scan: no lookup schedule for G=%d b=%d", p.G, p.b);
}

}  // namespace kvs
