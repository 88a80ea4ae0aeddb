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
// the 5th-generation tensor cores:
//  * a producer warp streams 128-token e4m3 tiles (16 KB, one 1-D TMA bulk
//    copy each) into a shared-memory ring;
//  * sixteen converter warps turn each tile into f16 (exact for e4m3) in the
//    canonical 128-byte-swizzled K-major layout of the MMA's A operand; the
//    queries become the B operand once per request, in f16 after scaling by a
//    power of two (exact) that brings max|q| to [2^13, 2^14);
//  * one elected thread issues tcgen05.mma kind::f16 (M = 128 tokens,
//    N = Hi heads, K = 16 per instruction, 8 instructions) into one of three
//    f32 accumulators in tensor memory, and commits to mbarriers;
//  * the converter warps then read the accumulators back (tcgen05.ld: one
//    token row per thread; warp w reads the TMEM lanes of tokens
//    32 (w mod 4) .. + 31 and the 16-head column chunks c = w / 4, w / 4 + 4),
//    apply ReLU and the head weights (with the scale undone); the four partial
//    head sums of a token meet in shared memory, and warps 0-3 reduce
//    32/64/128-token blocks with warp shuffles. (Four warps, one per
//    scheduler, left the conversion and read-back latency-bound.)
// Every wait is bounded; a wait that runs out sets KVS_ETIMEOUT in the status
// word and the block winds down without leaving copies in flight or TMEM
// allocated.
#include <cuda_fp8.h>

#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kTileTok = 128;                 // tokens per tile (MMA M)
constexpr int kRawBytes = kTileTok * 128;      // e4m3 tile: 128 tokens x 128 channels
constexpr int kATileBytes = kTileTok * 256;    // f16 tile, two 128-byte-wide K blocks
constexpr int kNRaw = 3;                       // raw tile ring depth
constexpr int kNAcc = 3;                       // A tiles and accumulators in flight
constexpr int kLConvWarps = 16;                // warps 0-15 convert + epilogue
constexpr int kLConv = 32 * kLConvWarps;
constexpr int kLoadWarp = kLConvWarps, kMmaWarp = kLConvWarps + 1;
constexpr int kLThreads = kLConv + 64;
constexpr long long kLWaitCycles = 2000000000ll;

struct LSmem {
  alignas(1024) unsigned char a[kNAcc][kATileBytes];  // converted A tiles (SW128 K-major)
  alignas(1024) unsigned char bq[2][128 * 256];     // query B operand per request parity
  alignas(1024) unsigned char raw[kNRaw][kRawBytes];
  float w[4][128];                                  // weights (scale undone), request sequence mod 4
  float spart[kNAcc][4][kTileTok];                  // partial head sums per column group
  float blockpart[kNAcc][4];                        // per-warp block maxima
  float qmax[kLConvWarps];
  uint64_t raw_full[kNRaw], raw_empty[kNRaw], a_full[kNAcc], a_empty[kNAcc], acc_full[kNAcc],
      acc_empty[kNAcc];
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
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          saddr(dst)),
      "l"(src), "r"(bytes), "r"(saddr(bar))
      : "memory");
}
__device__ __forceinline__ void group_sync() {  // the converter / epilogue warps
  asm volatile("bar.sync 2, %0;\n" ::"n"(kLConv) : "memory");
}
__device__ __forceinline__ void tile_sync() {  // warps 0-3: one tile's 128 tokens
  asm volatile("bar.sync 3, 128;\n" ::: "memory");
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

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
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
// 16 consecutive f32 columns of this warp's 32 TMEM lanes (one row per thread)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
}

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

__global__ void __launch_bounds__(kLThreads, 1) lightning_scan_kernel(LParams p) {
  extern __shared__ __align__(1024) unsigned char lsm_raw[];
  LSmem& sm = *reinterpret_cast<LSmem*>(
      lsm_raw + ((1024 - (saddr(lsm_raw) & 1023u)) & 1023u));  // 1024-byte aligned base
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.R * p.tiles_per_req;
  const int beg = static_cast<int>(static_cast<long long>(blockIdx.x) * T / gridDim.x);
  const int end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * T / gridDim.x);
  const int Hi = p.Hi;
  // kNAcc accumulators of Hi columns (a power of two >= 32 columns)
  const uint32_t tmem_cols = Hi <= 32 ? 128u : (Hi <= 64 ? 256u : 512u);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNRaw; ++i) {
      bar_init(&sm.raw_full[i], 1);
      bar_init(&sm.raw_empty[i], kLConvWarps);
    }
    for (int i = 0; i < kNAcc; ++i) {
      bar_init(&sm.a_full[i], kLConvWarps);
      bar_init(&sm.a_empty[i], 1);
      bar_init(&sm.acc_full[i], 1);
      bar_init(&sm.acc_empty[i], kLConvWarps);
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
    // ---------------- producer: raw e4m3 tiles ----------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < end - beg; ++i) {
        const int st = i % kNRaw;
        if (i >= kNRaw && !bar_wait(&sm.raw_empty[st], ((i / kNRaw) - 1) & 1)) {
          fail();
          break;
        }
        if (aborted()) break;
        const int tile = beg + i;
        const int r = tile / p.tiles_per_req, t0 = (tile % p.tiles_per_req) * kTileTok;
        const int nr = p.n[r];
        const int toks = t0 < nr ? min(kTileTok, p.n_max - t0) : 0;
        const uint32_t bytes = static_cast<uint32_t>(toks) * 128u;
        bar_expect(&sm.raw_full[st], bytes);
        if (bytes)
          bulk_load(sm.raw[st], p.kidx + (static_cast<size_t>(r) * p.n_max + t0) * 128, bytes,
                    &sm.raw_full[st]);
        ++issued;
      }
      for (int i = max(0, issued - kNRaw); i < issued; ++i)
        bar_wait(&sm.raw_full[i % kNRaw], (i / kNRaw) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (static_cast<uint32_t>(Hi >> 3) << 17) | (8u << 24);
      int req_seq = -1, prev_r = -1;
      for (int i = 0; i < end - beg; ++i) {
        const int tile = beg + i;
        const int r = tile / p.tiles_per_req;
        if (r != prev_r) {
          ++req_seq;
          prev_r = r;
        }
        const int x = i % kNAcc;
        if (!bar_wait(&sm.a_full[x], (i / kNAcc) & 1)) {
          fail();
          break;
        }
        if (i >= kNAcc && !bar_wait(&sm.acc_empty[x], ((i / kNAcc) - 1) & 1)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t abase = saddr(sm.a[x]);
        const uint32_t bbase = saddr(sm.bq[req_seq & 1]);
        const uint32_t dcol = tmem + static_cast<uint32_t>(x * Hi);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t koff = static_cast<uint32_t>((ks >> 2) * (kTileTok * 128) + (ks & 3) * 32);
          const uint32_t kboff = static_cast<uint32_t>((ks >> 2) * (Hi * 128) + (ks & 3) * 32);
          mma_f16(dcol, sw128_desc(abase + koff), sw128_desc(bbase + kboff), idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&sm.a_empty[x]);
        mma_commit(&sm.acc_full[x]);
      }
    }
  } else {
    // ---------------- converters + epilogue (warps 0-15) ----------------
    const int t = threadIdx.x;
    int req_seq = -1, prev_r = -1;
    bool dead = false;
    auto epilogue = [&](int i) {
      const int tile = beg + i;
      const int r = tile / p.tiles_per_req, t0 = (tile % p.tiles_per_req) * kTileTok;
      const int nr = p.n[r];
      const int x = i % kNAcc;
      // request sequence of tile i (consecutive requests in a contiguous tile range)
      const int seq = r - beg / p.tiles_per_req;
      const float* wv = sm.w[seq & 3];
      const int quarter = warp & 3, cgrp = warp >> 2;
      const int tin = quarter * 32 + lane;  // this thread's token (TMEM lane) in the tile
      float S = 0.f;
      if (!dead && bar_wait(&sm.acc_full[x], (i / kNAcc) & 1)) {
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(x * Hi);
        for (int c = cgrp; c < Hi / 16; c += 4) {
          float v[16];
          tmem_ld16(taddr + static_cast<uint32_t>(16 * c), v);
#pragma unroll
          for (int e = 0; e < 16; ++e) S = fmaf(wv[16 * c + e], fmaxf(v[e], 0.f), S);
        }
        tc_fence_before();
      } else if (!dead) {
        fail();
        dead = true;
      }
      __syncwarp();
      if (lane == 0 && !dead) bar_arrive(&sm.acc_empty[x]);
      sm.spart[x][cgrp][tin] = S;
      group_sync();
      if (cgrp != 0) return;
      S = (sm.spart[x][0][tin] + sm.spart[x][1][tin]) + (sm.spart[x][2][tin] + sm.spart[x][3][tin]);
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
      // 64- or 128-token blocks span 2 or 4 warps
      if (lane == 0) sm.blockpart[x][warp] = v;
      tile_sync();
      if (lane == 0) {
        const int per = p.block / 32;
        if (warp % per == 0) {
          float m = v;
          for (int q = 1; q < per; ++q) m = fmaxf(m, sm.blockpart[x][warp + q]);
          if (tok < p.n_max) out[tok / p.block] = m;
        }
      }
      tile_sync();
    };
    for (int i = 0; i < end - beg; ++i) {
      const int tile = beg + i;
      const int r = tile / p.tiles_per_req;
      const int x = i % kNAcc;
      const int st = i % kNRaw;
      if (i >= kNAcc && !dead && !bar_wait(&sm.a_empty[x], ((i / kNAcc) - 1) & 1)) {
        fail();
        dead = true;
      }
      if (r != prev_r) {
        ++req_seq;
        prev_r = r;
        // the MMAs of the two previous tiles may still read the query buffer
        // of this parity: wait for them (a request has one tile at least)
        for (int j = max(0, i - 2); j < i && !dead; ++j)
          if (!bar_wait(&sm.a_empty[j % kNAcc], (j / kNAcc) & 1)) {
            fail();
            dead = true;
          }
        // the request's queries as the B operand, scaled by 2^e into f16
        const int par = req_seq & 1;
        const uint16_t* q = p.qidx + static_cast<size_t>(r) * Hi * 128;
        float mx = 0.f;
        for (int e = t; e < Hi * 128; e += kLConv) mx = fmaxf(mx, fabsf(bf16_bits_to_float(q[e])));
        for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
        if (lane == 0) sm.qmax[warp] = mx;
        group_sync();
        mx = 0.f;
        for (int e = 0; e < kLConvWarps; ++e) mx = fmaxf(mx, sm.qmax[e]);
        int ex = 0;
        if (mx > 0.f) {
          int e2;
          frexpf(mx, &e2);  // mx in [2^(e2-1), 2^e2)
          ex = 14 - e2;     // scaled max in [2^13, 2^14)
        }
        const float sc = ldexpf(1.f, ex), inv = ldexpf(1.f, -ex);
        for (int c = t; c < Hi * 16; c += kLConv) {  // 16-byte output chunks: row h, chunk cc
          const int h = c >> 4, cc = c & 15;
          const uint16_t* src = q + h * 128 + cc * 8;
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half lo = __float2half_rn(bf16_bits_to_float(src[2 * e]) * sc);
            const __half hi = __float2half_rn(bf16_bits_to_float(src[2 * e + 1]) * sc);
            packed[e] = static_cast<uint32_t>(__half_as_ushort(lo)) |
                        (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
          }
          const int kb = cc >> 3, j = cc & 7;
          *reinterpret_cast<uint4*>(sm.bq[par] + kb * (Hi * 128) + sw128_off(h, j)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        for (int h = t; h < Hi; h += kLConv) sm.w[req_seq & 3][h] = p.w[static_cast<size_t>(r) * Hi + h] * inv;
      }
      // convert the raw tile into the swizzled f16 A tile
      if (!dead && !bar_wait(&sm.raw_full[st], (i / kNRaw) & 1)) {
        fail();
        dead = true;
      }
      if (!dead) {
        for (int c = t; c < kTileTok * 8; c += kLConv) {  // 16-byte raw chunk: row, part
          const int row = c >> 3, part = c & 7;
          const uint4 raw = *reinterpret_cast<const uint4*>(sm.raw[st] + row * 128 + part * 16);
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t h8[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(w4[e] & 0xFFFFu), __NV_E4M3);
            const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(w4[e] >> 16), __NV_E4M3);
            h8[2 * e] = static_cast<uint32_t>(lo.x) | (static_cast<uint32_t>(lo.y) << 16);
            h8[2 * e + 1] = static_cast<uint32_t>(hi.x) | (static_cast<uint32_t>(hi.y) << 16);
          }
          const int kb = part >> 2, j0 = (part & 3) * 2;
          unsigned char* abase = sm.a[x] + kb * (kTileTok * 128);
          *reinterpret_cast<uint4*>(abase + sw128_off(row, j0)) = make_uint4(h8[0], h8[1], h8[2], h8[3]);
          *reinterpret_cast<uint4*>(abase + sw128_off(row, j0 + 1)) =
              make_uint4(h8[4], h8[5], h8[6], h8[7]);
        }
        // generic-proxy writes of A (and B) must be visible to the tensor core
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          bar_arrive(&sm.raw_empty[st]);
          bar_arrive(&sm.a_full[x]);
        }
      }
      // the read-back runs two tiles behind the conversion, so that a tile's
      // MMAs have a whole conversion period to complete
      if (i >= 2) epilogue(i - 2);
    }
    for (int j = max(0, end - beg - 2); j < end - beg; ++j) epilogue(j);
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
  const int T = p.R * p.tiles_per_req;
  const int grid = min(T, sm_count());
  const size_t smem = sizeof(LSmem) + 1024;
  cudaFuncSetAttribute(lightning_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  lightning_scan_kernel<<<grid, kLThreads, smem, s>>>(p);
  return check_launch("index_scan(lightning)");
}

}  // namespace kvs
