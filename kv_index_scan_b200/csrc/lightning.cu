// lightning.cu -- a2-L, the lightning-indexer variant of the index scan
// ("MiniMax-M3: share the sparse index top-k across layers and reuse the
// decode top-k buffer", description: every sparse layer runs a lightning
// indexer whose output picks the top-k KV blocks).
//
// Reading (the page gives no formula): for request r and token i,
//   S_i = sum_{h < Hi} w_h * max(0, q_h . k_i),
// with e4m3 keys k_i [n][128], bf16 index queries q_h and f32 head weights;
// the block score is the max of S over the block's valid tokens.
//
// The q.K products are a dense GEMM per request (tokens x heads x 128), run on
// the 5th-generation tensor cores straight on the e4m3 keys:
//  * a producer thread loads 128-token tiles (16 KB) with a 2-D TMA tensor map
//    over the keys [R * n_max][128 bytes], 128-byte swizzled: each tile lands
//    in the canonical K-major layout of the MMA's A operand, no conversion;
//  * the queries of a request become one e4m3 B operand of 2 Hi rows after
//    scaling by a power of two (exact) that brings max|q| to [2^7, 2^8):
//    row h holds hi = e4m3(q_h 2^e) and row Hi + h lo = e4m3(q_h 2^e - hi).
//    A bf16 value has 8 significant bits, so hi + lo is q 2^e exactly unless
//    lo falls below the e4m3 subnormal range (elements 2^10 below the
//    largest: an absolute error under 2^-10 there);
//  * one elected thread issues tcgen05.mma kind::f8f6f4 (M = 128 tokens,
//    N = 2 Hi, K = 32 per instruction, four per tile) into one of up to eight
//    f32 accumulators in tensor memory;
//  * sixteen worker warps in four groups of four read the accumulators back,
//    group g the tiles i = g (mod 4), so that four tiles drain at once: one
//    token row per thread (warp w reads the TMEM lanes of tokens
//    32 (w mod 4) .. + 31), each head's hi and lo columns added, ReLU and the
//    head weights (with the scale undone), then 32/64/128-token block maxima
//    by warp shuffles and across the group's warps. The workers also write
//    each request's query operand up to four tiles ahead of its first tile
//    (two buffers, by request parity).
// Every wait is bounded; a wait that runs out sets KVS_ETIMEOUT in the status
// word and the block winds down without leaving copies in flight or TMEM
// allocated.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kTileTok = 128;                 // tokens per tile (MMA M)
constexpr int kTileBytes = kTileTok * 128;     // e4m3 tile: one 128-byte swizzle row per token
constexpr int kNStage = 8;                     // key tiles in flight
static_assert((kNStage & (kNStage - 1)) == 0, "the stage index is a mask");
constexpr int kNAccMax = 8;                    // accumulators in tensor memory (8 for Hi <= 64, else 4)
constexpr int kLWork = 16;                     // warps 0-15: query operands + read-back
constexpr int kLWorkThreads = 32 * kLWork;
constexpr int kLoadWarp = kLWork, kMmaWarp = kLWork + 1;
constexpr int kLThreads = kLWorkThreads + 64;
constexpr long long kLWaitCycles = 2000000000ll;

struct LSmem {
  alignas(1024) unsigned char a[kNStage][kTileBytes];  // key tiles (SW128 K-major, by TMA)
  alignas(1024) unsigned char bq[2][2][128 * 128];     // queries: [request parity][2 Hi rows]: hi, then lo
  float w[4][128];                                     // weights (scale undone), request sequence mod 4
  float blockpart[kNAccMax][4];                        // per-warp block maxima
  float qmax[kLWork];
  uint64_t a_full[kNStage], a_empty[kNStage], acc_full[kNAccMax], acc_empty[kNAccMax], q_full[2], q_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(LSmem) + 1024 <= 227 * 1024, "lightning shared memory over the per-block limit");

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint64_t* b, uint32_t c) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(saddr(b)), "r"(c) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ void bar_expect(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(saddr(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool bar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool bar_wait(uint64_t* b, uint32_t parity) {
  if (bar_try(b, parity)) return true;
  const long long t0 = clock64();
  while (!bar_try(b, parity))
    if (clock64() - t0 > kLWaitCycles) return false;
  return true;
}
// A 2-D tile of the tensor map at (x, y) into shared memory, completing on bar.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          saddr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(saddr(bar))
      : "memory");
}
__device__ __forceinline__ void group_sync() {  // the worker warps
  asm volatile("bar.sync 2, %0;\n" ::"n"(kLWorkThreads) : "memory");
}
__device__ __forceinline__ void tile_sync(int grp) {  // the four warps of one tile's 128 tokens
  asm volatile("bar.sync %0, 128;\n" ::"r"(3 + grp) : "memory");
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle
// layout: 8-row groups 1024 bytes apart, version 1, swizzle mode 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(16 >> 4) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Byte offset of 16-byte chunk j (0..7) of row r in one 128-byte-wide
// K block of the swizzled layout.
__device__ __forceinline__ uint32_t sw128_off(int r, int j) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

__device__ __forceinline__ void mma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   saddr(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
// 16 consecutive f32 columns of this warp's 32 TMEM lanes (one row per
// thread); the registers are valid after tmem_ld_wait()
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// Two f32 lanes in one 64-bit register, and the packed fused multiply-add.
__device__ __forceinline__ unsigned long long f2_pack(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long x) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(r.x), "=f"(r.y) : "l"(x));
  return r;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

struct LParams {
  const uint8_t* kidx;   // [R][n_max][128] e4m3
  const uint16_t* qidx;  // [R][Hi][128] bf16
  const float* w;        // [R][Hi]
  const int32_t* n;
  int R, n_max, Hi, block, tiles_per_req;
  float* out;  // [R][ceil(n_max/block)]
  int nb_max;
  int32_t* dev_status;
};

// NC = Hi / 16 head-column chunks of 16 (1..8).
template <int NC>
__global__ void __launch_bounds__(kLThreads, 1) lightning_scan_kernel(LParams p,
                                                                      const __grid_constant__ CUtensorMap kmap) {
  extern __shared__ __align__(1024) unsigned char lsm_raw[];
  LSmem& sm = *reinterpret_cast<LSmem*>(
      lsm_raw + ((1024 - (saddr(lsm_raw) & 1023u)) & 1023u));  // 1024-byte aligned base
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.R * p.tiles_per_req;
  const int beg = static_cast<int>(static_cast<long long>(blockIdx.x) * T / gridDim.x);
  const int end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * T / gridDim.x);
  const int ntile = end - beg;
  constexpr int Hi = 16 * NC;
  // nacc accumulators of 2 Hi columns (the hi and the lo query parts), as many
  // as fit in 512 columns up to kNAccMax, in a power of two >= 32 columns
  int nacc = kNAccMax;
  while (nacc * 2 * Hi > 512) nacc >>= 1;
  uint32_t tmem_cols = 32u;
  while (tmem_cols < static_cast<uint32_t>(nacc * 2 * Hi)) tmem_cols <<= 1;
  auto req_of = [&](int i) { return (beg + i) / p.tiles_per_req; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNStage; ++i) {
      bar_init(&sm.a_full[i], 1);
      bar_init(&sm.a_empty[i], 1);
    }
    for (int i = 0; i < kNAccMax; ++i) {
      bar_init(&sm.acc_full[i], 1);
      bar_init(&sm.acc_empty[i], 4);  // the four warps of the tile's group
    }
    for (int i = 0; i < 2; ++i) {
      bar_init(&sm.q_full[i], 1);
      bar_init(&sm.q_empty[i], 1);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     saddr(&sm.tmem_base)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  auto fail = [&] {
    set_status(p.dev_status, KVS_ETIMEOUT);
    atomicExch(&sm.abort_flag, 1);
  };
  auto aborted = [&] { return *reinterpret_cast<volatile int*>(&sm.abort_flag) != 0; };

  if (warp == kLoadWarp) {
    // ---------------- producer: key tiles by TMA ----------------
    // (one thread: every per-tile step is on its dependency chain, so the
    // request, its length and the stage are tracked incrementally)
    if (lane == 0) {
      int issued = 0;
      int r = beg / p.tiles_per_req, tin = beg % p.tiles_per_req;
      int nr = ntile > 0 ? p.n[r] : 0;
      for (int i = 0; i < ntile; ++i) {
        const int st = i & (kNStage - 1);
        if (i >= kNStage && !bar_wait(&sm.a_empty[st], ((i / kNStage) - 1) & 1)) {
          fail();
          break;
        }
        if (aborted()) break;
        const int t0 = tin * kTileTok;
        if (t0 < nr) {
          // rows past the request's end belong to the next request or lie
          // outside the map (zero fill); the read-back masks them
          bar_expect(&sm.a_full[st], kTileBytes);
          tma_load_2d(sm.a[st], &kmap, 0, r * p.n_max + t0, &sm.a_full[st]);
        } else {
          bar_arrive(&sm.a_full[st]);  // no valid token: nothing to load
        }
        ++issued;
        if (++tin == p.tiles_per_req) {
          tin = 0;
          ++r;
          if (i + 1 < ntile) nr = p.n[r];
        }
      }
      // no copy may still be in flight when the block ends
      for (int i = max(0, issued - kNStage); i < issued; ++i)
        bar_wait(&sm.a_full[i & (kNStage - 1)], (i / kNStage) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (static_cast<uint32_t>((2 * Hi) >> 3) << 17) | (8u << 24);
      // descriptors of stage 0 / query buffer 0; stage st, parity par and K
      // step ks add (st * 16384 + 32 ks) or (par * 32768 + 32 ks) bytes, i.e.
      // that >> 4, to the start-address field (which cannot overflow: shared
      // memory ends below 2^18 bytes)
      const uint64_t adesc0 = sw128_desc(saddr(sm.a[0]));
      const uint64_t bdesc0 = sw128_desc(saddr(sm.bq[0][0]));
      static_assert(kTileBytes == 16384 && sizeof(sm.bq[0][0]) == 16384, "descriptor steps assume 16 KB operands");
      int seq = -1;
      int tin = beg % p.tiles_per_req;
      for (int i = 0; i < ntile; ++i) {
        if (i == 0 || tin == 0) {
          // the previous request's MMAs are all issued: its query buffers are
          // free once they complete
          if (seq >= 0) mma_commit(&sm.q_empty[seq & 1]);
          ++seq;
          if (!bar_wait(&sm.q_full[seq & 1], (seq >> 1) & 1)) {
            fail();
            break;
          }
        }
        if (++tin == p.tiles_per_req) tin = 0;
        const int st = i & (kNStage - 1), x = i & (nacc - 1);
        if (!bar_wait(&sm.a_full[st], (i / kNStage) & 1)) {
          fail();
          break;
        }
        if (i >= nacc && !bar_wait(&sm.acc_empty[x], ((i / nacc) - 1) & 1)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint64_t ad = adesc0 + static_cast<uint64_t>(st * (16384 >> 4));
        const uint64_t bd = bdesc0 + static_cast<uint64_t>((seq & 1) * (32768 >> 4));
        const uint32_t dcol = tmem + static_cast<uint32_t>(x * 2 * Hi);
        // N = 2 Hi: query rows 0..Hi-1 hold the hi parts, Hi..2Hi-1 the lo parts
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_f8(dcol, ad + 2 * ks, bd + 2 * ks, idesc, ks > 0 ? 1u : 0u);
        mma_commit(&sm.a_empty[st]);
        mma_commit(&sm.acc_full[x]);
      }
    }
  } else {
    // ---------------- workers: query operands + read-back (warps 0-15) ----------------
    const int t = threadIdx.x;
    bool dead = false;
    int seq_prep = -1;
    // the query operands of the request whose first tile is tile i
    auto prep = [&](int i) {
      const int r = req_of(i);
      const int s = ++seq_prep, par = s & 1;
      if (s >= 2 && t == 0 && !dead && !aborted() && !bar_wait(&sm.q_empty[par], ((s >> 1) - 1) & 1))
        fail();
      const uint16_t* q = p.qidx + static_cast<size_t>(r) * Hi * 128;
      float mx = 0.f;
      for (int e = t; e < Hi * 128; e += kLWorkThreads) mx = fmaxf(mx, fabsf(bf16_bits_to_float(q[e])));
      for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
      if (lane == 0) sm.qmax[warp] = mx;
      group_sync();  // also: the buffers of this parity are free (thread 0 waited)
      dead = dead || aborted();
      mx = 0.f;
      for (int e = 0; e < kLWork; ++e) mx = fmaxf(mx, sm.qmax[e]);
      int ex = 0;
      if (mx > 0.f) {
        int e2;
        frexpf(mx, &e2);  // mx in [2^(e2-1), 2^e2)
        ex = 8 - e2;      // scaled max in [2^7, 2^8)
      }
      const float sc = ldexpf(1.f, ex), inv = ldexpf(1.f, -ex);
      for (int c = t; c < Hi * 8; c += kLWorkThreads) {  // 16 channels of head h: chunk j
        const int h = c >> 3, j = c & 7;
        const uint16_t* src = q + h * 128 + j * 16;
        uint32_t hi4[4], lo4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t hw = 0u, lw = 0u;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float x = bf16_bits_to_float(src[4 * e + b]) * sc;
            const __nv_fp8_storage_t h8 = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
            const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(h8, __NV_E4M3)));
            const __nv_fp8_storage_t l8 = __nv_cvt_float_to_fp8(x - hv, __NV_SATFINITE, __NV_E4M3);
            hw |= static_cast<uint32_t>(h8) << (8 * b);
            lw |= static_cast<uint32_t>(l8) << (8 * b);
          }
          hi4[e] = hw;
          lo4[e] = lw;
        }
        unsigned char* qb = &sm.bq[par][0][0];  // [2 Hi rows][128 bytes]: hi rows, then lo rows
        *reinterpret_cast<uint4*>(qb + sw128_off(h, j)) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
        *reinterpret_cast<uint4*>(qb + sw128_off(Hi + h, j)) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
      }
      for (int h = t; h < Hi; h += kLWorkThreads) sm.w[s & 3][h] = p.w[static_cast<size_t>(r) * Hi + h] * inv;
      // generic-proxy writes of the operands must be visible to the tensor core
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      group_sync();
      if (t == 0) bar_arrive(&sm.q_full[par]);
    };
    const int grp = warp >> 2, quarter = warp & 3;
    const int tin = quarter * 32 + lane;  // this thread's token (TMEM lane) in a tile
    auto epilogue = [&](int i) {
      const int tile = beg + i;
      const int r = tile / p.tiles_per_req, t0 = (tile % p.tiles_per_req) * kTileTok;
      const int nr = p.n[r];
      const int x = i % nacc;
      // request sequence of tile i (consecutive requests in a contiguous tile range)
      const int seq = r - beg / p.tiles_per_req;
      const float* wv = sm.w[seq & 3];
      // head chunks c = cg, cg + 4, ... summed into part[cg] (even and odd heads
      // in the two lanes of a packed pair), then (part0 + part1) + (part2 + part3)
      unsigned long long part[4] = {0ull, 0ull, 0ull, 0ull};
      // one lane per warp polls the barrier (32 pollers per CTA instead of 512
      // keep the shared-memory pipe free for the TMA writes); the warp then
      // synchronises and fences before reading tensor memory
      int ok = 0;
      if (lane == 0) ok = !dead && !aborted() && bar_wait(&sm.acc_full[x], (i / nacc) & 1);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      __syncwarp();
      if (ok) {
        tc_fence_after();
        const uint32_t taddr =
            tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(x * 2 * Hi);
#pragma unroll 1
        for (int c0 = 0; c0 < NC; c0 += 4) {
#pragma unroll
          for (int cg = 0; cg < 4; ++cg) {
            const int c = c0 + cg;
            if (c < NC) {
              // q.k of heads 16c..16c+15 = the hi column plus the lo column
              uint32_t vh[16], vl[16];
              tmem_ld16(taddr + static_cast<uint32_t>(16 * c), vh);
              tmem_ld16(taddr + static_cast<uint32_t>(Hi + 16 * c), vl);
              tmem_ld_wait();
              unsigned long long S = part[cg];
#pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                const ulonglong2 w4 = *reinterpret_cast<const ulonglong2*>(wv + 16 * c + 4 * e4);
                float d[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  d[e] = fmaxf(__uint_as_float(vh[4 * e4 + e]) + __uint_as_float(vl[4 * e4 + e]), 0.f);
                S = f2_fma(w4.x, f2_pack(d[0], d[1]), S);
                S = f2_fma(w4.y, f2_pack(d[2], d[3]), S);
              }
              part[cg] = S;
            }
          }
        }
        tc_fence_before();
      } else if (!dead) {
        fail();
        dead = true;
      }
      __syncwarp();
      if (lane == 0 && !dead) bar_arrive(&sm.acc_empty[x]);
      float ps[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 pp = f2_unpack(part[e]);
        ps[e] = pp.x + pp.y;
      }
      const float S = (ps[0] + ps[1]) + (ps[2] + ps[3]);
      const int tok = t0 + tin;
      const float ninf = -__int_as_float(0x7f800000);
      float v = tok < nr ? S : ninf;
      float* out = p.out + static_cast<size_t>(r) * p.nb_max;
      if (p.block == 1) {
        if (tok < p.n_max) out[tok] = v;
        return;
      }
      const int wblk = min(p.block, 32);
      for (int d = 1; d < wblk; d <<= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, d));
      if (p.block <= 32) {
        if ((lane & (p.block - 1)) == 0 && tok < p.n_max) out[tok / p.block] = v;
        return;
      }
      // 64- or 128-token blocks span 2 or 4 warps of the group
      if (lane == 0) sm.blockpart[x][quarter] = v;
      tile_sync(grp);
      if (lane == 0) {
        const int per = p.block / 32;
        if (quarter % per == 0) {
          float m = v;
          for (int q = 1; q < per; ++q) m = fmaxf(m, sm.blockpart[x][quarter + q]);
          if (tok < p.n_max) out[tok / p.block] = m;
        }
      }
      tile_sync(grp);
    };
    // every group prepares every request's operands in the same order (the
    // preparation is block-wide), each before its first tile at or past
    // (first tile of the request) - 4
    int prepared = -1;  // first tile of the last prepared request
    auto next_first = [&](int b) {  // first tile of the request after tile b's
      return (req_of(b) + 1) * p.tiles_per_req - beg;
    };
    for (int i = grp;; i += 4) {
      while (true) {
        const int b = prepared < 0 ? 0 : next_first(prepared);
        if (b >= ntile || b > i + 4) break;
        prep(b);
        prepared = b;
      }
      if (i >= ntile) break;
      epilogue(i);
    }
  }
  // wind down: TMEM is released by the warp that allocated it
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(tmem_cols)
                 : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library links no driver library), looked up once per process.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

}  // namespace

kvs_status lightning_scan_dispatch(const kvs_scan_args* a, float* scores, int32_t* dev_status,
                                   cudaStream_t s) {
  KVS_REQUIRE(a->kidx && a->qidx && a->widx, KVS_EINVAL, "index_scan(lightning): null pointer");
  KVS_REQUIRE(a->Dl == 128, KVS_EUNSUPPORTED, "index_scan(lightning): Dl=%d (only 128 is built)",
              a->Dl);
  KVS_REQUIRE(a->Hi >= 16 && a->Hi <= 128 && a->Hi % 16 == 0, KVS_EUNSUPPORTED,
              "index_scan(lightning): Hi=%d (a multiple of 16 up to 128)", a->Hi);
  KVS_REQUIRE(a->block == 1 || a->block == 32 || a->block == 64 || a->block == 128, KVS_EUNSUPPORTED,
              "index_scan(lightning): block=%d (1, 32, 64 or 128)", a->block);
  KVS_REQUIRE(aligned16(a->kidx), KVS_EINVAL, "index_scan(lightning): kidx must be 16-byte aligned");
  if (a->n_max == 0) return KVS_OK;
  LParams p{};
  p.kidx = a->kidx;
  p.qidx = a->qidx;
  p.w = a->widx;
  p.n = a->n;
  p.R = a->R;
  p.n_max = a->n_max;
  p.Hi = a->Hi;
  p.block = a->block;
  p.tiles_per_req = (a->n_max + kTileTok - 1) / kTileTok;
  p.out = scores;
  p.nb_max = (a->n_max + a->block - 1) / a->block;
  p.dev_status = dev_status;
  KVS_REQUIRE(static_cast<long long>(a->R) * a->n_max < (1ll << 31), KVS_EUNSUPPORTED,
              "index_scan(lightning): R*n_max=%lld rows (below 2^31 supported)",
              static_cast<long long>(a->R) * a->n_max);
  // the keys as a 2-D tensor [R * n_max][128 bytes], read in 128 x 128 boxes
  // with the 128-byte swizzle of the MMA operand layout
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  KVS_REQUIRE(encode != nullptr, KVS_ECUDA, "index_scan(lightning): cuTensorMapEncodeTiled unavailable");
  CUtensorMap kmap;
  const cuuint64_t gdim[2] = {128, static_cast<cuuint64_t>(a->R) * a->n_max};
  const cuuint64_t gstride[1] = {128};
  const cuuint32_t box[2] = {128, kTileTok};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult enc = encode(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a->kidx), gdim,
                              gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  KVS_REQUIRE(enc == CUDA_SUCCESS, KVS_ECUDA, "index_scan(lightning): tensor map encoding failed (%d)",
              static_cast<int>(enc));
  const int T = p.R * p.tiles_per_req;
  const int grid = min(T, sm_count());
  const size_t smem = sizeof(LSmem) + 1024;
  auto go = [&](auto kernel) {
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    kernel<<<grid, kLThreads, smem, s>>>(p, kmap);
  };
  switch (a->Hi / 16) {
    case 1: go(lightning_scan_kernel<1>); break;
    case 2: go(lightning_scan_kernel<2>); break;
    case 3: go(lightning_scan_kernel<3>); break;
    case 4: go(lightning_scan_kernel<4>); break;
    case 5: go(lightning_scan_kernel<5>); break;
    case 6: go(lightning_scan_kernel<6>); break;
    case 7: go(lightning_scan_kernel<7>); break;
    default: go(lightning_scan_kernel<8>); break;
  }
  return check_launch("index_scan(lightning)");
}

}  // namespace kvs
