// scan_prmt.cuh -- the byte-indexed lookup core of the HBM Fathom scan, for
// plans of at most 144 planes ("Fathom: Per-Query Read Depth for Sparse
// Decoding over Offloaded KV Caches", abstract: every key is scored from the
// B plane bits its query's allocation chose).
//
//   score_i = C + sum over the plan's planes q of W_q * bit_q(i)
//
// The planes are taken in groups of 8 (plan order); group g has a 256-entry
// table of the sums of its weights, so a key's score is C plus one table entry
// per group. What bounds this on B200 is the integer pipe and shared-memory
// bandwidth, not the plane bytes, so each step is shaped for instruction count:
//
//  * Staging. Four producer warps (one per scheduler) copy, for a chunk of 128
//    plane words (4,096 keys) of one (request, KV head) row, every plan
//    plane's 512-byte segment into one slot of a shared-memory ring: one
//    16-byte cp.async per lane and plane, completing on the slot's mbarrier
//    (cp.async.mbarrier.arrive). Measured on B200, 512-byte 1-D TMA bulk
//    copies cap this pattern near 2.4 TB/s even with nothing else running, the
//    warp-wide 16-byte copies near 5.7 TB/s. Rows past B in a slot stay zero.
//  * Partial transpose. Two consumer threads share a plane word, 16 keys each
//    (eight consumer warps, two per scheduler, to hide load latency). For a
//    block of 4 groups (32 planes) a thread loads its 16-bit halves of the 32
//    words, pairs plane p with plane p + 16 in one register, and runs three
//    shift/select stages that exchange the three low bits of the register
//    index with the three low bits of the key (4 integer operations per
//    register pair and stage). Afterwards byte 2 * (g >> 1) + (key >> 3) of
//    register 8 * (g & 1) + (key & 7) holds group g's 8 plane bits of the key:
//    exactly the table index. The byte-granular stages of a full transpose are
//    never needed.
//  * Lookup. One byte permute (prmt) builds the shared address
//    256 * index + 4 * bank + 128 * row directly from the transposed byte and
//    a per-lane bank byte; then one shared load and one add. Tables are stored
//    with a 256-byte entry stride, so the bank of a lookup depends only on its
//    bank byte, never on the data: each of two rows of 32 banks holds one
//    "set" of G groups (G = 1, 2, 4, 8 or 16), banks 2j and 2j + 1 serving
//    group j mod G. A thread pair reads its groups in a rotated order (blocks
//    rotated by pair / 4, groups within a block by pair % 4), takes at every
//    step the bank pair that holds the group it needs, and its two threads
//    take the two banks of that pair, so the 32 lanes of a warp always hit 32
//    distinct banks. Tables: 256 entries x 64 banks x 4 bytes = 64 KB.
//
// Per key at B = 92 (12 groups): ~21 integer operations for the transposes,
// 12 permutes, 12 shared loads for lookups plus 6 for plane halves, 12 adds.
#pragma once

#include "scan_core.cuh"

namespace kvs {

constexpr int kPWarps = 8;                      // consumer warps
constexpr int kPProd = 4;                       // producer warps
constexpr int kPThreads = 32 * (kPWarps + kPProd);
constexpr int kPKeys = 16;                      // keys per consumer thread (half a word)
constexpr int kPChunkWords = 16 * kPWarps;      // plane words per chunk (4,096 keys)
constexpr int kPRowBytes = 4 * kPChunkWords;    // one staged plane segment
constexpr int kPTableBytes = 256 * 256;         // 256 entries x 64 banks x 4 bytes
constexpr int kPZeroBytes = 8 * kPRowBytes;     // zero rows for empty group positions
constexpr int kPMaxB = 144;                     // 18 groups: two sets of <= 16
constexpr int kPSmemLimit = 227 * 1024;

// Groups of the two table sets for a plan of B planes (GA >= 4; GB may be 0).
__host__ __device__ inline void prmt_sets(int B, int& GA, int& GB) {
  const int ng = (B + 7) / 8;
  if (ng <= 4) {
    GA = 4;
    GB = 0;
  } else if (ng <= 8) {
    GA = 8;
    GB = 0;
  } else if (ng <= 12) {
    GA = 8;
    GB = ng == 9 ? 1 : (ng == 10 ? 2 : 4);
  } else if (ng <= 16) {
    GA = 16;
    GB = 0;
  } else {
    GA = 16;
    GB = ng == 17 ? 1 : 2;
  }
}

inline int prmt_slot_bytes(int B) {
  int GA, GB;
  prmt_sets(B, GA, GB);
  return 8 * (GA + GB) * kPRowBytes;
}

// Ring depth for B with `extra` bytes of epilogue scratch (0 when it does not fit).
inline int prmt_nstages(int B, size_t extra) {
  const long long budget =
      static_cast<long long>(kPSmemLimit) - kPTableBytes - kPZeroBytes - 256 - static_cast<long long>(extra);
  const long long s = budget / prmt_slot_bytes(B);
  return static_cast<int>(s > 4 ? 4 : (s < 0 ? 0 : s));
}

inline size_t prmt_smem_bytes(int B, int nstage, size_t extra) {
  return static_cast<size_t>(kPTableBytes) + kPZeroBytes +
         static_cast<size_t>(nstage) * prmt_slot_bytes(B) + 256 + extra;
}

inline int prmt_chunks_per_row(int n_max) {
  const int words = (n_max + 31) / 32;
  return (words + kPChunkWords - 1) / kPChunkWords;
}

// Exchanges bits 0..2 of the register index with bits 0..2 of the bit
// position, in both 16-bit halves: on entry bit j of x[q] is key j of plane
// position q and bit 16 + j key j of position q + 16; on exit byte
// 2 * (g >> 1) + (key >> 3) of x[8 * (g & 1) + (key & 7)] holds the 8 plane bits
// of group g (positions 8g .. 8g + 7) for key `key`.
// (a & m) | (b & ~m) in one 3-input logic operation
__device__ __forceinline__ uint32_t bit_select(uint32_t a, uint32_t b, uint32_t m) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;\n" : "=r"(d) : "r"(a), "r"(b), "r"(m));
  return d;
}

__device__ __forceinline__ void partial_transpose16(uint32_t (&x)[16]) {
#pragma unroll
  for (int st = 0; st < 3; ++st) {
    const int s = 1 << st;
    const uint32_t m = st == 0 ? 0x55555555u : (st == 1 ? 0x33333333u : 0x0F0F0F0Fu);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      if (q & s) continue;
      const uint32_t a = x[q], b = x[q + s];
      x[q] = bit_select(a, b << s, m);
      x[q + s] = bit_select(a >> s, b, m);
    }
  }
}

struct ScanCoreP {
  static constexpr int KEYS = kPKeys;
  static constexpr int CHUNK_WORDS = kPChunkWords;
  static constexpr int NCONS = 32 * kPWarps;

  // first key index of consumer thread t's 16 keys in chunk c
  __host__ __device__ static int key0(int c, int t) {
    return 32 * (c * kPChunkWords + (t >> 1)) + kPKeys * (t & 1);
  }

  const ScanParams& p;
  int nstage, GA, GB, slot_bytes;
  uint32_t stage0;  // shared offset of slot 0 (relative to g_scan_smem)
  uint64_t* full;
  uint64_t* empty;
  int* abort_flag;

  __device__ explicit ScanCoreP(const ScanParams& params) : p(params) {
    nstage = p.nstage;
    prmt_sets(p.B, GA, GB);
    slot_bytes = 8 * (GA + GB) * kPRowBytes;
    stage0 = kPTableBytes + kPZeroBytes;
    full = reinterpret_cast<uint64_t*>(g_scan_smem + stage0 + nstage * slot_bytes);
    empty = full + nstage;
    abort_flag = reinterpret_cast<int*>(empty + nstage);
  }

  __device__ unsigned char* extra() const {
    return g_scan_smem + stage0 + nstage * slot_bytes + 256;
  }

  __device__ void fail_timeout() {
    set_status(p.dev_status, KVS_ETIMEOUT);
    atomicExch(abort_flag, 1);
  }

  __device__ long long wait_limit() const { return p.wait_cycles > 0 ? p.wait_cycles : kWaitCycles; }

  __device__ static void sync() { consumer_sync<kPWarps>(); }

  // Producer warp j (0..3) stages planes j, j + 4, j + 8, ... of every chunk.
  __device__ void produce(int beg, int end) {
    const int lane = threadIdx.x & 31, j = (threadIdx.x >> 5) - kPWarps;
    int cur_u = -1;
    uint32_t off_lo = 0u, off_hi = 0u;  // plane indices of this warp's planes lane and lane + 32
    int u = beg / p.chunks_per_row, c = beg % p.chunks_per_row, st = 0;
    uint32_t phase = 0u;  // parity of the slot's next empty phase to wait for
    for (int it = beg; it < end; ++it) {
      if (it - beg >= nstage && !mbar_wait(&empty[st], phase, wait_limit())) {
        if (lane == 0) fail_timeout();
        break;
      }
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      if (u != cur_u) {
        const uint16_t* pidx = p.plane_idx + static_cast<size_t>(u) * p.B;
        const int q0 = j + 4 * lane, q1 = j + 4 * (lane + 32);
        off_lo = q0 < p.B ? pidx[q0] : 0u;
        off_hi = q1 < p.B ? pidx[q1] : 0u;
        cur_u = u;
      }
      const int w0 = c * kPChunkWords;
      const int nr = p.n[u / p.Gheads];
      if (32 * w0 < nr) {  // uniform over the warp
        const bool mine = 4 * lane < p.W - w0;  // this lane's 16 bytes lie inside the row
        const uint32_t* src0 = p.planes + static_cast<size_t>(u) * kD * 4 * p.W + w0 + 4 * lane;
        const uint32_t dst0 = smem_addr(g_scan_smem + stage0 + st * slot_bytes) + 16u * lane;
        const int nq = (p.B - j + 3) >> 2;  // this warp's planes
        for (int s = 0; s < nq; ++s) {
          const uint32_t pi = __shfl_sync(0xFFFFFFFFu, s < 32 ? off_lo : off_hi, s & 31);
          if (mine)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                             dst0 + static_cast<uint32_t>((j + 4 * s) * kPRowBytes)),
                         "l"(src0 + static_cast<size_t>(pi) * p.W)
                         : "memory");
        }
      }
      if (!(p.withhold_arrive && j == 0 && it == beg))
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_addr(&full[st]))
                     : "memory");
      if (++c == p.chunks_per_row) {
        c = 0;
        ++u;
      }
      if (++st == nstage) {
        st = 0;
        if (it - beg + 1 > nstage) phase ^= 1u;
      }
    }
    // never leave copies in flight into this block's shared memory
    asm volatile("cp.async.wait_all;\n" ::: "memory");
  }

  // The 64 KB of tables for row u (consumer threads only). Bank b of row
  // sigma serves group g0 + ((b >> 1) mod G) of that set; thread t fills
  // quarter t / 64 of the 256 entries of bank t % 64.
  __device__ void build_tables(int u) {
    const int t = threadIdx.x;
    const int slot = t & 63, quarter = t >> 6;
    const int sigma = slot >> 5, b = slot & 31;
    const int G = sigma ? GB : GA;
    if (G == 0) return;
    const int T = (sigma ? GA : 0) + ((b >> 1) & (G - 1));
    const float* w = p.plane_w + static_cast<size_t>(u) * p.B;
    float wv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wv[e] = 8 * T + e < p.B ? w[8 * T + e] : 0.f;
    float lo[16];
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((v >> e) & 1) s += wv[e];
      lo[v] = s;
    }
    float* tab = reinterpret_cast<float*>(g_scan_smem) + b + 32 * sigma;
#pragma unroll 1
    for (int hv = 0; hv < 4; ++hv) {
      const int h = quarter * 4 + hv;
      float hs = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((h >> e) & 1) hs += wv[4 + e];
#pragma unroll
      for (int lv = 0; lv < 16; ++lv) tab[(h * 16 + lv) * 64] = lo[lv] + hs;
    }
  }

  // Zero the padding rows of every slot and the zero region (consumer threads).
  __device__ void zero_fill() {
    const int t = threadIdx.x;
    const int rows = 8 * (GA + GB);
    uint4* z = reinterpret_cast<uint4*>(g_scan_smem + kPTableBytes);
    for (int i = t; i < kPZeroBytes / 16; i += NCONS) z[i] = make_uint4(0u, 0u, 0u, 0u);
    const int pad_rows = rows - p.B;
    if (pad_rows > 0) {
      const int per_slot = pad_rows * kPRowBytes / 16;
      for (int i = t; i < nstage * per_slot; i += NCONS) {
        const int st = i / per_slot, e = i % per_slot;
        reinterpret_cast<uint4*>(g_scan_smem + stage0 + st * slot_bytes + p.B * kPRowBytes)[e] =
            make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }

  // Per-lane constants of a set's block schedule. A set of G >= 4 groups
  // visits its G / 4 blocks in an order rotated by pair / 4 and, inside a
  // block, its groups in an order rotated by pair % 4; a set of 1 or 2 groups
  // has one block whose group positions rotate by the pair index.
  struct SetLane {
    uint32_t goff[4];  // byte offset of group position gi's first row in the slot (+ lane)
    uint32_t ya, yb;   // bank bytes of positions 0..2 and 3 (block-step term added per block)
  };

  __device__ __forceinline__ SetLane set_lane(int sigma, int g0, int G) const {
    const int t = threadIdx.x;
    const int lane = t & 31, i = lane >> 1, h = lane & 1, i0 = i & 3;
    const uint32_t lane_off = 4u * static_cast<uint32_t>(t >> 1) + 2u * static_cast<uint32_t>(h);
    const uint32_t rowb = 4u * static_cast<uint32_t>(h) + 128u * static_cast<uint32_t>(sigma);
    constexpr uint32_t GROUP = 8u * kPRowBytes;
    SetLane L;
    uint32_t bank[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      if (G >= 4) {
        L.goff[gi] = static_cast<uint32_t>(g0 + ((gi + i0) & 3)) * GROUP + lane_off;
        bank[gi] = rowb + 8u * static_cast<uint32_t>((i0 + gi) & 3);
      } else {
        L.goff[gi] = gi < G ? static_cast<uint32_t>(g0 + ((gi + i) & (G - 1))) * GROUP + lane_off
                            : 0x80000000u + lane_off;  // marks the zero region
        bank[gi] = rowb + 8u * static_cast<uint32_t>((i + gi) & 15);
      }
    }
    L.ya = bank[0] | (bank[1] << 8) | (bank[2] << 16);
    L.yb = bank[3];
    return L;
  }

  // One set's contribution (row sigma of the tables, groups g0 .. g0 + G - 1)
  // to this thread's 16 keys.
  __device__ __forceinline__ void set_pass(uint32_t slot_off, int G, const SetLane& L,
                                           float (&acc)[kPKeys]) const {
    const int i2 = (threadIdx.x & 31) >> 3;
    const int NB = (G + 3) >> 2;
    constexpr uint32_t GROUP = 8u * kPRowBytes;
#pragma unroll 1
    for (int m = 0; m < NB; ++m) {
      uint32_t gb[4];
      uint32_t y_a = L.ya, y_b = L.yb;
      if (G >= 4) {
        const uint32_t bb = slot_off + static_cast<uint32_t>(4 * ((m + i2) & (NB - 1))) * GROUP;
        const uint32_t step = 32u * static_cast<uint32_t>((i2 + m) & 3);
        y_a += step * 0x00010101u;
        y_b += step;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) gb[gi] = bb + L.goff[gi];
      } else {
#pragma unroll
        for (int gi = 0; gi < 4; ++gi)
          gb[gi] = (L.goff[gi] & 0x80000000u) ? static_cast<uint32_t>(kPTableBytes) + (L.goff[gi] & 0x7FFFFFFFu)
                                             : slot_off + L.goff[gi];
      }
      uint32_t x[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const uint32_t lo = *reinterpret_cast<const uint16_t*>(g_scan_smem + gb[q >> 3] + (q & 7) * kPRowBytes);
        const uint32_t hi = *reinterpret_cast<const uint16_t*>(g_scan_smem + gb[2 + (q >> 3)] + (q & 7) * kPRowBytes);
        x[q] = __byte_perm(lo, hi, 0x5410);
      }
      partial_transpose16(x);
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if (gi >= G) break;
        const uint32_t y = gi < 3 ? y_a : y_b;
        const uint32_t yb = gi < 3 ? static_cast<uint32_t>(gi) : 0u;
#pragma unroll
        for (int kk = 0; kk < kPKeys; ++kk) {
          // address = 256 * (group gi's byte of key kk) + bank byte; bytes 2, 3 = 0
          const uint32_t byte = static_cast<uint32_t>(2 * (gi >> 1) + (kk >> 3));
          const uint32_t a = __byte_perm(x[8 * (gi & 1) + (kk & 7)], y,
                                         (7u << 12) | (7u << 8) | (byte << 4) | (4u + yb));
          acc[kk] += *reinterpret_cast<const float*>(g_scan_smem + a);
        }
      }
    }
  }

  // epi(u, c, nr, acc, t) runs in every consumer thread after each chunk c of
  // row u (acc: its 16 scores; nr: the row's length).
  template <typename Epi>
  __device__ void run(Epi&& epi) {
    const int chunks = p.RG * p.chunks_per_row;
    const int beg = static_cast<int>(static_cast<long long>(blockIdx.x) * chunks / gridDim.x);
    const int end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * chunks / gridDim.x);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
      for (int i = 0; i < nstage; ++i) {
        mbar_init(&full[i], 32 * kPProd);
        mbar_init(&empty[i], kPWarps);
      }
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (warp >= kPWarps) {
      produce(beg, end);
      return;
    }
    zero_fill();
    const int lane = threadIdx.x & 31;
    const SetLane la = set_lane(0, 0, GA);
    const SetLane lb = set_lane(1, GA, GB);
    int cur_u = -1, row_n = 0;
    float row_C = 0.f;
    bool dead = false;
    float acc[kPKeys];
    int u = beg / p.chunks_per_row, c = beg % p.chunks_per_row, st = 0;
    uint32_t phase = 0u;
    for (int it = beg; it < end; ++it) {
      if (u != cur_u) {
        sync();
        if (!dead) build_tables(u);
        row_n = p.n[u / p.Gheads];
        row_C = p.C[u];
        sync();
        cur_u = u;
      }
      const int nr = row_n;
#pragma unroll
      for (int j = 0; j < kPKeys; ++j) acc[j] = row_C;
      if (!dead && !mbar_wait(&full[st], phase, wait_limit())) {
        fail_timeout();
        dead = true;
      }
      const uint32_t soff = stage0 + static_cast<uint32_t>(st * slot_bytes);
      if (!dead && 32 * c * kPChunkWords < nr) {
        set_pass(soff, GA, la, acc);
        if (GB > 0) set_pass(soff, GB, lb, acc);
      }
      __syncwarp();
      if (!dead && lane == 0) mbar_arrive(&empty[st]);
      epi(u, c, nr, acc, static_cast<int>(threadIdx.x));
      if (++c == p.chunks_per_row) {
        c = 0;
        ++u;
      }
      if (++st == nstage) {
        st = 0;
        phase ^= 1u;
      }
    }
  }
};

}  // namespace kvs
