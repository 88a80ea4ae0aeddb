// attn.cu -- a5: GQA decode attention over the selected rows only
// ("XM-Sparse: Pushing the Throughput Frontier of Sparse Attention with
// Netpreme X-Mem", opening paragraph: each decode step attends to the chosen
// KV entries alone).
//
// For each (r, g) and query head h: l_j = scale * q_h . K_j over the selected
// rows, o = sum_j softmax(l)_j V_j, with an online softmax in f32 (base-2
// exponent, scale folded with log2 e into q).
//
// The rows are read straight from where they live: a staged [k][D] buffer, the
// hot buffer / full store through the slot of each selected key, or the full
// store by index. The bound is the gather of 512 bytes of K/V per row; the
// arithmetic runs on the tensor cores so that it stays well below it:
//
//  * Each warp streams its own 16-row tiles through a three-stage ring in
//    shared memory with cp.async (16-byte copies, zero fill for padding rows,
//    chunk c of row r stored at c ^ (r & 7) so that ldmatrix reads are
//    conflict-free). The row locations of a tile are fetched four tiles ahead
//    of its copies, and its copies two tiles ahead of its arithmetic.
//  * Logits: S^T[heads][rows] = Q K^T with mma.m16n8k16 (bf16 inputs, f32
//    accumulation). The 16 MMA rows hold q split in two bf16 parts, q_hi in
//    rows 0..7 and q - q_hi in rows 8..15, so one MMA carries q to ~16 bits
//    and the two halves are added in f32.
//  * P.V: the logit accumulators are, element for element, the A operand of
//    the next MMA (O[heads][dims] += P[heads][rows] V[rows][dims]); P is split
//    into hi/lo bf16 parts the same way, V comes from ldmatrix.trans.
//  * With H <= 4 the 16 MMA rows are the tile's tokens instead and the 8
//    columns the heads' hi and lo query parts (4 + 4): S[rows][cols] = K Q^T
//    takes 8 MMAs per tile instead of 16, and O^T[dims][cols] += V^T P^T
//    8 instead of 16, with V^T from ldmatrix.trans and P^T from the logit
//    accumulators by movmatrix.trans (hi parts in the columns of lanes
//    c < 2, lo parts in those of c >= 2). A head's logit is the sum of its hi
//    and lo columns; O's two halves are added at the end.
//  * Online softmax per head: inside the four lanes that hold the head (H > 4),
//    or across the eight lane groups that hold the tile's tokens, with the
//    row sums kept per lane until the end (H <= 4). The block's warps merge
//    by log-sum-exp in shared memory, and the blocks (splits) of one (r, g)
//    in a second small kernel. (Merging the splits inside a
//    thread-block cluster instead made the kernel faster alone but the decode
//    step slower: a clustered launch lost the overlap with its neighbours that
//    programmatic dependent launch gives the step's kernels.)
#include <cuda_bf16.h>

#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kAttnBlocksPerSM = 2;
constexpr int kAttnStages = 3;
constexpr int kTileRows = 16;
constexpr int kSplitUnit = 64;                           // rows: the granularity of a split
constexpr int kStageBytes = 2 * kTileRows * kD * 2;      // K and V of one tile, bf16
constexpr int kAttnSmem = kAttnWarps * kAttnStages * kStageBytes;  // 96 KB

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t s, const void* gmem, bool valid) {
  const int bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D = A B + D, m16n8k16, bf16 inputs, f32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// The 8x8 b16 matrix held one row pair per lane (lane 4r + c: row r, columns
// 2c, 2c + 1), transposed in the same layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}
// Two floats as bf16 (round to nearest even), x in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), for a pair.
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(x, y);
  const float hx = __uint_as_float(hi << 16), hy = __uint_as_float(hi & 0xFFFF0000u);
  lo = pack_bf16(x - hx, y - hy);
}

// Where row j of (r, g) = u lives, as one code: -1 padding, c >= 0 row c of
// the staged / full store, c <= -2 hot slot -2 - c.
__device__ __forceinline__ int row_code(const RowSrc& src, int u, int j) {
  if (j >= src.k) return -1;
  if (src.mode == kRowsSlotStaged) {  // misses were fetched to staging row j
    const int32_t* irow =
        src.idx + (src.idx_shared ? static_cast<size_t>(u / src.G) : static_cast<size_t>(u)) * src.k;
    const int i = __ldg(irow + j);
    const int sl = __ldg(src.slots + static_cast<size_t>(u) * src.k + j);
    return i < 0 ? -1 : (sl >= 0 ? -2 - sl : j);
  }
  if (src.mode == kRowsStaged) {
    const int ke = src.k_eff ? src.k_eff[u] : src.k;
    return j < ke ? j : -1;
  }
  const int32_t* irow =
      src.idx + (src.idx_shared ? static_cast<size_t>(u / src.G) : static_cast<size_t>(u)) * src.k;
  if (src.mode == kRowsSlot && src.slots) {
    // both loads issued together (the slot of a padding entry is not used)
    const int i = __ldg(irow + j);
    const int sl = __ldg(src.slots + static_cast<size_t>(u) * src.k + j);
    return i < 0 ? -1 : (sl >= 0 ? -2 - sl : i);
  }
  const int i = irow[j];
  if (i < 0) return -1;
  if (src.mode == kRowsSlot) {
    const int sl = src.slots ? src.slots[static_cast<size_t>(u) * src.k + j]
                             : src.slot_map[static_cast<size_t>(u) * src.n_max + i];
    if (sl >= 0) return -2 - sl;
  }
  return i;
}

// q_early: q is read before the wait on the preceding kernel (allowed when no
// kernel of the chain writes q, as in the decode step, where q is its input).
template <int H>
__global__ void __launch_bounds__(kAttnThreads, kAttnBlocksPerSM) sparse_attn_kernel(
    const void* __restrict__ q, int q_bf16, RowSrc src, int nsplit, int rows_per_split,
    float scale_log2, float* __restrict__ out, float* __restrict__ lse,
    float* __restrict__ part, int q_early) {
  if (!q_early) pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) unsigned char attn_smem[];
  const float ninf = -__int_as_float(0x7f800000);
  const int u = blockIdx.x / nsplit;
  const int split = blockIdx.x % nsplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;  // MMA fragment row group / thread in group
  const int j_begin = split * rows_per_split;
  const int j_end = min(src.k, j_begin + rows_per_split);
  const uint32_t ring = smem_u32(attn_smem) + warp * kAttnStages * kStageBytes;

  constexpr bool kTok = H <= 4;  // tokens as the MMA's M dimension
  // kTok: B operand of the logits MMA, column g = head g & 3, its hi part for
  // g < 4 and its lo part for g >= 4, over dims 16 ks + 2 tq (+1, +8, +9).
  // Otherwise: A operand, row g = q_hi of head g, row g + 8 = q_lo.
  uint32_t qa[8][kTok ? 2 : 4];
  auto q_pair = [&](int head, int d0, float& x, float& y) {
    x = 0.f;
    y = 0.f;
    if (head < H) {
      const size_t off = (static_cast<size_t>(u) * H + head) * kD + d0;
      if (q_bf16) {
        const uint16_t* qq = reinterpret_cast<const uint16_t*>(q) + off;
        x = bf16_bits_to_float(qq[0]);
        y = bf16_bits_to_float(qq[1]);
      } else {
        const float* qq = reinterpret_cast<const float*>(q) + off;
        x = qq[0];
        y = qq[1];
      }
      x *= scale_log2;
      y *= scale_log2;
    }
  };
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int d0 = 16 * ks + 8 * half + 2 * tq;
      float x, y;
      q_pair(kTok ? (g & 3) : g, d0, x, y);
      uint32_t hi, lo;
      split_bf16(x, y, hi, lo);
      if constexpr (kTok) {
        qa[ks][half] = g < 4 ? hi : lo;
      } else {
        qa[ks][2 * half] = hi;
        qa[ks][2 * half + 1] = lo;
      }
    }
  }
  if (q_early) pdl_wait();

  // row bases of this (r, g): staged rows are [u][k], full-store rows [u][n_max]
  const size_t full_rows = (src.mode == kRowsStaged || src.mode == kRowsSlotStaged)
                               ? static_cast<size_t>(src.k) : static_cast<size_t>(src.n_max);
  const uint16_t* fK = src.K + static_cast<size_t>(u) * full_rows * kD;
  const uint16_t* fV = src.V + static_cast<size_t>(u) * full_rows * kD;
  const uint16_t* hK = src.hotK ? src.hotK + static_cast<size_t>(u) * src.S * kD : fK;
  const uint16_t* hV = src.hotV ? src.hotV + static_cast<size_t>(u) * src.S * kD : fV;

  // this warp's tiles: rows j_begin + 16 * (warp + kAttnWarps * i)
  const int ntile_all = j_end > j_begin ? (j_end - j_begin + kTileRows - 1) / kTileRows : 0;
  const int ntiles = ntile_all > warp ? (ntile_all - warp + kAttnWarps - 1) / kAttnWarps : 0;
  auto tile_row0 = [&](int i) { return j_begin + kTileRows * (warp + kAttnWarps * i); };
  // lane r < 16 fetches the code of row r of tile i
  auto fetch_code = [&](int i) -> int {
    if (i >= ntiles || lane >= kTileRows) return -1;
    const int j = tile_row0(i) + lane;
    return j < j_end ? row_code(src, u, j) : -1;
  };
  // copies of tile i (codes in lanes 0..15) into stage st; returns its valid-row mask
  auto issue = [&](int i, int code, int st) -> unsigned {
    const unsigned vm = __ballot_sync(0xFFFFFFFFu, lane < kTileRows && code != -1) & 0xFFFFu;
    if (i < ntiles) {
      const uint32_t sbase = ring + st * kStageBytes;
      const int ch = lane & 15;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int rc = 2 * e + (lane >> 4);  // row copy: K rows 0..15, then V rows 0..15
        const int r = rc & 15;
        const bool isv = rc >= 16;
        const int c = __shfl_sync(0xFFFFFFFFu, code, r);
        const uint16_t* base = c >= 0 ? (isv ? fV : fK) : (isv ? hV : hK);
        const size_t row = static_cast<size_t>(c >= 0 ? c : (c == -1 ? 0 : -2 - c));
        const uint32_t dst = sbase + (isv ? kTileRows * kD * 2 : 0) + r * (kD * 2) +
                             ((ch ^ (r & 7)) << 4);
        cp_async16(dst, base + row * kD + ch * 8, c != -1);
      }
    }
    cp_async_commit();
    return vm;
  };

  float o[kTok ? 8 : 16][4];
#pragma unroll
  for (int d = 0; d < (kTok ? 8 : 16); ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[d][e] = 0.f;
  float m_run = ninf, l_run = 0.f;  // of head g, shared by the four lanes of group g
  // kTok: this lane's heads hA = 2 (tq & 1) and hA + 1; l is the lane's part
  // (tokens g and g + 8 of each tile), summed over the lanes at the end
  float mA = ninf, mB = ninf, lA = 0.f, lB = 0.f;

  // prologue: tiles 0 and 1 in flight, the codes of tiles 2..5 on their way
  // (row locations are fetched four tiles ahead of their copies)
  // The codes of tile t live in register c[t % 4] (the loop is unrolled by 4
  // so that each stays in place until used: moving a register whose load is
  // still in flight would wait for it).
  unsigned vm0 = issue(0, fetch_code(0), 0);
  unsigned vm1 = issue(1, fetch_code(1), 1);
  int c0 = fetch_code(4), c1 = fetch_code(5), c2 = fetch_code(2), c3 = fetch_code(3);

  for (int i0 = 0; i0 < ntiles; i0 += 4)
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + a;
    if (i >= ntiles) break;
    int& code_cur = a == 0 ? c2 : (a == 1 ? c3 : (a == 2 ? c0 : c1));  // tile i + 2's
    const int st = i % kAttnStages;
    const unsigned vm2 = issue(i + 2, code_cur, (i + 2) % kAttnStages);
    code_cur = fetch_code(i + 6);
    cp_async_wait<kAttnStages - 1>();
    __syncwarp();
    const uint32_t kst = ring + st * kStageBytes;
    const uint32_t vst = kst + kTileRows * kD * 2;

    if constexpr (kTok) {
      // ---- S[tokens][cols] = K Q^T: A = the K tile (ldmatrix), B = q ----
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        const int row = lane & 15;
        const int chunk = 2 * ks + (lane >> 4);
        ldsm_x4(kst + row * (kD * 2) + ((chunk ^ (row & 7)) << 4), a);
        mma_bf16(sc, a, qa[ks][0], qa[ks][1]);
      }
      // logits of heads hA, hA + 1 for tokens g and g + 8: hi column + lo column
      float s4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) s4[e] = sc[e] + __shfl_xor_sync(0xFFFFFFFFu, sc[e], 2);
      const bool vg = (vm0 >> g) & 1u, vg8 = (vm0 >> (g + 8)) & 1u;
      s4[0] = vg ? s4[0] : ninf;
      s4[1] = vg ? s4[1] : ninf;
      s4[2] = vg8 ? s4[2] : ninf;
      s4[3] = vg8 ? s4[3] : ninf;
      float mxA = fmaxf(s4[0], s4[2]), mxB = fmaxf(s4[1], s4[3]);
#pragma unroll
      for (int d = 4; d < 32; d <<= 1) {
        mxA = fmaxf(mxA, __shfl_xor_sync(0xFFFFFFFFu, mxA, d));
        mxB = fmaxf(mxB, __shfl_xor_sync(0xFFFFFFFFu, mxB, d));
      }
      const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
      const bool noneA = nA == ninf, noneB = nB == ninf;
      const float alA = noneA ? 1.f : exp2f(mA - nA), alB = noneB ? 1.f : exp2f(mB - nB);
      float p4[4];
      p4[0] = noneA ? 0.f : exp2f(s4[0] - nA);
      p4[2] = noneA ? 0.f : exp2f(s4[2] - nA);
      p4[1] = noneB ? 0.f : exp2f(s4[1] - nB);
      p4[3] = noneB ? 0.f : exp2f(s4[3] - nB);
      lA = lA * alA + (p4[0] + p4[2]);
      lB = lB * alB + (p4[1] + p4[3]);
      mA = nA;
      mB = nB;
      if (!__all_sync(0xFFFFFFFFu, alA == 1.f && alB == 1.f)) {
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          o[d][0] *= alA;
          o[d][2] *= alA;
          o[d][1] *= alB;
          o[d][3] *= alB;
        }
      }
      // ---- O^T[dims][cols] += V^T P^T: P^T by movmatrix, V^T by ldmatrix.trans ----
      uint32_t h01, l01, h23, l23;
      split_bf16(p4[0], p4[1], h01, l01);
      split_bf16(p4[2], p4[3], h23, l23);
      const uint32_t b0 = movmatrix_trans(tq < 2 ? h01 : l01);
      const uint32_t b1 = movmatrix_trans(tq < 2 ? h23 : l23);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a[4];
        const int mi = lane >> 3;
        const int tok = (lane & 7) + 8 * (mi >> 1);
        const int chunk = 2 * mt + (mi & 1);
        ldsm_x4_trans(vst + tok * (kD * 2) + ((chunk ^ (tok & 7)) << 4), a);
        mma_bf16(o[mt], a, b0, b1);
      }
    } else {
    // ---- logits of the tile's 16 rows (two n-tiles of 8) ----
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b[4];
        const int row = (lane & 7) + ((lane >> 4) << 3);
        const int chunk = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(kst + row * (kD * 2) + ((chunk ^ (row & 7)) << 4), b);
        mma_bf16(sc[0], qa[ks], b[0], b[1]);
        mma_bf16(sc[1], qa[ks], b[2], b[3]);
      }
      // ---- online softmax of head g over rows n = 8 nt + 2 tq + e ----
      float s[2][2];
      float mx = ninf;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int n = 8 * nt + 2 * tq + e;
          const float v = sc[nt][e] + sc[nt][e + 2];
          s[nt][e] = ((vm0 >> n) & 1u) ? v : ninf;
          mx = fmaxf(mx, s[nt][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const bool none = m_new == ninf;
      const float alpha = none ? 1.f : exp2f(m_run - m_new);
      float p[2][2];
      float ps = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          p[nt][e] = none ? 0.f : exp2f(s[nt][e] - m_new);
          ps += p[nt][e];
        }
      ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 1);
      ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 2);
      l_run = l_run * alpha + ps;
      m_run = m_new;
      if (!__all_sync(0xFFFFFFFFu, alpha == 1.f)) {
#pragma unroll
        for (int d = 0; d < 16; ++d)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[d][e] *= alpha;
      }
      // ---- P.V: P (hi/lo split) is the A operand, V from ldmatrix.trans ----
      uint32_t pa[4];
      split_bf16(p[0][0], p[0][1], pa[0], pa[1]);
      split_bf16(p[1][0], p[1][1], pa[2], pa[3]);
#pragma unroll
      for (int d2 = 0; d2 < 8; ++d2) {
        uint32_t b[4];
        const int mi = lane >> 3;
        const int row = (lane & 7) + 8 * (mi & 1);
        const int chunk = 2 * d2 + (mi >> 1);
        ldsm_x4_trans(vst + row * (kD * 2) + ((chunk ^ (row & 7)) << 4), b);
        mma_bf16(o[2 * d2], pa, b[0], b[1]);
        mma_bf16(o[2 * d2 + 1], pa, b[2], b[3]);
      }
    }
    __syncwarp();  // the stage is refilled by the next iteration's copies
    vm0 = vm1;
    vm1 = vm2;
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the block's warps by log-sum-exp (the ring is free now) ----
  float* sm_o = reinterpret_cast<float*>(attn_smem);  // [warps][H][kD]
  float* sm_ml = sm_o + kAttnWarps * H * kD;          // [warps][H][2]
  if constexpr (kTok) {
    // O = the hi columns + the lo columns (lanes tq and tq ^ 2); l over the
    // lanes' tokens
#pragma unroll
    for (int d = 0; d < 8; ++d)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[d][e] += __shfl_xor_sync(0xFFFFFFFFu, o[d][e], 2);
#pragma unroll
    for (int d = 4; d < 32; d <<= 1) {
      lA += __shfl_xor_sync(0xFFFFFFFFu, lA, d);
      lB += __shfl_xor_sync(0xFFFFFFFFu, lB, d);
    }
    const int hA = 2 * (tq & 1), hB = hA + 1;
    if (tq < 2) {
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        if (hA < H) {
          sm_o[(warp * H + hA) * kD + 16 * d + g] = o[d][0];
          sm_o[(warp * H + hA) * kD + 16 * d + g + 8] = o[d][2];
        }
        if (hB < H) {
          sm_o[(warp * H + hB) * kD + 16 * d + g] = o[d][1];
          sm_o[(warp * H + hB) * kD + 16 * d + g + 8] = o[d][3];
        }
      }
      if (g == 0) {
        if (hA < H) {
          sm_ml[(warp * H + hA) * 2] = mA;
          sm_ml[(warp * H + hA) * 2 + 1] = lA;
        }
        if (hB < H) {
          sm_ml[(warp * H + hB) * 2] = mB;
          sm_ml[(warp * H + hB) * 2 + 1] = lB;
        }
      }
    }
  } else if (g < H) {
    float* dst = sm_o + (warp * H + g) * kD + 2 * tq;
#pragma unroll
    for (int d = 0; d < 16; ++d)
      *reinterpret_cast<float2*>(dst + 8 * d) = make_float2(o[d][0] + o[d][2], o[d][1] + o[d][3]);
    if (tq == 0) {
      sm_ml[(warp * H + g) * 2] = m_run;
      sm_ml[(warp * H + g) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  for (int h = warp; h < H; h += kAttnWarps) {
    float M = ninf;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, sm_ml[(w * H + h) * 2]);
    float L = 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != ninf) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float sw = exp2f(sm_ml[(w * H + h) * 2] - M);
        L = fmaf(sm_ml[(w * H + h) * 2 + 1], sw, L);
        const float4 ow = *reinterpret_cast<const float4*>(sm_o + (w * H + h) * kD + 4 * lane);
        acc[0] = fmaf(ow.x, sw, acc[0]);
        acc[1] = fmaf(ow.y, sw, acc[1]);
        acc[2] = fmaf(ow.z, sw, acc[2]);
        acc[3] = fmaf(ow.w, sw, acc[3]);
      }
    }
    if (nsplit == 1) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      *reinterpret_cast<float4*>(out + (static_cast<size_t>(u) * H + h) * kD + 4 * lane) =
          make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      if (lse && lane == 0)
        lse[static_cast<size_t>(u) * H + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : ninf;
    } else {
      float* pp = part + ((static_cast<size_t>(u) * nsplit + split) * H + h) * (kD + 4);
      *reinterpret_cast<float4*>(pp + 4 + 4 * lane) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      if (lane == 0) {
        pp[0] = M;
        pp[1] = L;
      }
    }
  }
}

// Merge of the splits of one (r, g): warp h merges head h by log-sum-exp.
__global__ void attn_combine_kernel(const float* __restrict__ part, int nsplit, int H,
                                    float* __restrict__ out, float* __restrict__ lse) {
  pdl_wait();
  const int u = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (h >= H) return;
  const float* base = part + static_cast<size_t>(u) * nsplit * H * (kD + 4);
  float M = -__int_as_float(0x7f800000);
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, base[(static_cast<size_t>(s) * H + h) * (kD + 4)]);
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -__int_as_float(0x7f800000)) {
    for (int s = 0; s < nsplit; ++s) {
      const float* pp = base + (static_cast<size_t>(s) * H + h) * (kD + 4);
      const float w = exp2f(pp[0] - M);
      L += pp[1] * w;
      const float4 v = *reinterpret_cast<const float4*>(pp + 4 + 4 * lane);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  *reinterpret_cast<float4*>(out + (static_cast<size_t>(u) * H + h) * kD + 4 * lane) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lse && lane == 0)
    lse[static_cast<size_t>(u) * H + h] =
        L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -__int_as_float(0x7f800000);
}

template <int H>
kvs_status launch_h(const void* q, int q_bf16, const RowSrc& src, int RG, int nsplit, int rps,
                    float scale_log2, float* out, float* lse, float* part, int q_early, cudaStream_t s) {
  cudaFuncSetAttribute(sparse_attn_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kAttnSmem);
  launch_chained(sparse_attn_kernel<H>, dim3(RG * nsplit), dim3(kAttnThreads), kAttnSmem, s, q, q_bf16, src,
                 nsplit, rps, scale_log2, out, lse, part, q_early);
  if (nsplit > 1) launch_chained(attn_combine_kernel, dim3(RG), dim3(H * 32), 0, s, part, nsplit, H, out, lse);
  return check_launch("sparse_decode_attn");
}

}  // namespace

// Split of the k rows across blocks: the split count that minimises (waves of
// blocks) x (64-row units per block + one unit of per-block overhead), ties to
// fewer splits. With max_part_bytes > 0 only the splits whose partial results
// (RG * nsplit * H * (128 + 4) floats) fit in that many bytes are considered;
// one split needs none, so there is always one.
static void attn_split_impl(int RG, int H, int k, size_t max_part_bytes, int& nsplit,
                            int& rows_per_split) {
  const int units = max(1, (k + kSplitUnit - 1) / kSplitUnit);
  const long long slots = static_cast<long long>(kAttnBlocksPerSM) * sm_count();
  int best = 1;
  long long best_cost = -1;
  for (int ns = 1; ns <= min(units, 64); ++ns) {
    const int per = (units + ns - 1) / ns;
    const int used = (units + per - 1) / per;
    if (max_part_bytes > 0 && used > 1 &&
        static_cast<size_t>(RG) * used * H * (kD + 4) * sizeof(float) > max_part_bytes)
      continue;
    const long long waves = (static_cast<long long>(RG) * used + slots - 1) / slots;
    const long long cost = waves * (per + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = used;
    }
  }
  const int per = (units + best - 1) / best;
  rows_per_split = per * kSplitUnit;
  nsplit = (units + per - 1) / per;
}

void attn_split(int RG, int k, int& nsplit, int& rows_per_split) {
  attn_split_impl(RG, 1, k, 0, nsplit, rows_per_split);
}

size_t attn_ws_bytes(int RG, int H, int k) {
  int nsplit, rps;
  attn_split(RG, k, nsplit, rps);
  if (nsplit <= 1) return 0;
  return static_cast<size_t>(RG) * nsplit * H * (kD + 4) * sizeof(float);
}

static kvs_status attn_launch_split(const void* q, int q_bf16, const RowSrc& src, int RG, int H,
                                    float scale, float* out, float* lse, float* part, int nsplit,
                                    int rps, int q_early, cudaStream_t s) {
  const float sl2 = scale * 1.4426950408889634f;
  switch (H) {
    case 1: return launch_h<1>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 2: return launch_h<2>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 3: return launch_h<3>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 4: return launch_h<4>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 5: return launch_h<5>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 6: return launch_h<6>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 7: return launch_h<7>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    case 8: return launch_h<8>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, q_early, s);
    default: return fail(KVS_EUNSUPPORTED, "H=%d query heads per KV head (1..8 supported)", H);
  }
}

kvs_status attn_launch(const void* q, int q_bf16, const RowSrc& src, int RG, int H, float scale,
                       float* out, float* lse, void* ws, cudaStream_t s, bool q_early) {
  int nsplit, rps;
  attn_split(RG, src.k, nsplit, rps);
  return attn_launch_split(q, q_bf16, src, RG, H, scale, out, lse, static_cast<float*>(ws), nsplit,
                           rps, q_early ? 1 : 0, s);
}

// The attention with a split whose partial results fit in part_bytes (the
// cheapest such split; one split writes none). *need receives the bytes used.
kvs_status attn_launch_fit(const void* q, int q_bf16, const RowSrc& src, int RG, int H,
                           float scale, float* out, float* lse, float* part, size_t part_bytes,
                           size_t* need, cudaStream_t s) {
  int nsplit, rps;
  attn_split_impl(RG, H, src.k, part_bytes, nsplit, rps);
  *need = nsplit > 1 ? static_cast<size_t>(RG) * nsplit * H * (kD + 4) * sizeof(float) : 0;
  if (*need > part_bytes) return fail(KVS_EINVAL, "attention split needs %zu bytes, %zu available", *need, part_bytes);
  return attn_launch_split(q, q_bf16, src, RG, H, scale, out, lse, part, nsplit, rps, 0, s);
}

}  // namespace kvs

// ----------------------------------------------------------------------------
// sparse_decode_attn_noalloc: the same attention for callers that cannot
// allocate device memory. Its split-K partial results (the only scratch the
// attention needs) live in one fixed array of this library instead of a
// caller workspace.
#include <mutex>

namespace {

// 4 MiB of partial results: R*G*nsplit*H*(128+4) floats. Each call takes the
// cheapest split of the k rows whose partial results fit here; one split per
// (r, g) writes none, so every size runs (sizes whose workspace split would
// need more than 4 MiB run with fewer splits). Every GPU that loads this
// library holds the array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) float g_attn_scratch[kNoAllocScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
float* g_scratch_dev[64] = {nullptr};

// Device address of g_attn_scratch on the current device. The name of the
// array in host code is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached for the life of the
// process; the cache does not survive cudaDeviceReset (after a reset, reload
// the library before calling again).
kvs_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return kvs::fail(KVS_ECUDA, "sparse_decode_attn_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return kvs::fail(KVS_EUNSUPPORTED, "sparse_decode_attn_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess || p == nullptr)
      return kvs::fail(KVS_ECUDA, "sparse_decode_attn_noalloc: cudaGetSymbolAddress: %s",
                       cudaGetErrorString(e));
    g_scratch_dev[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_dev[dev];
  return KVS_OK;
}

}  // namespace

extern "C" kvs_status sparse_decode_attn_noalloc(const void* q, int32_t q_dtype, const uint16_t* K,
                                                 const uint16_t* V, const int32_t* k_eff, int32_t R,
                                                 int32_t G, int32_t H, int32_t D, int32_t k,
                                                 float scale, float* out, float* lse,
                                                 int32_t* dev_status, void* stream) {
  using namespace kvs;
  (void)dev_status;
  KVS_REQUIRE(q && K && V && out, KVS_EINVAL, "sparse_decode_attn_noalloc: null pointer argument");
  KVS_REQUIRE(q_dtype == KVS_F32 || q_dtype == KVS_BF16, KVS_EINVAL,
              "sparse_decode_attn_noalloc: q_dtype=%d", q_dtype);
  KVS_REQUIRE(R >= 1 && G >= 1 && k >= 1 && H >= 1 && H <= 8, KVS_EINVAL,
              "sparse_decode_attn_noalloc: R=%d G=%d H=%d k=%d", R, G, H, k);
  KVS_REQUIRE(D == kD, KVS_EUNSUPPORTED, "sparse_decode_attn_noalloc: D=%d (only 128 is built)", D);
  KVS_REQUIRE(aligned16(K) && aligned16(V) && aligned16(out), KVS_EINVAL,
              "sparse_decode_attn_noalloc: K, V and out must be 16-byte aligned");
  float* scratch = nullptr;
  kvs_status st = noalloc_scratch(&scratch);
  if (st != KVS_OK) return st;
  RowSrc src{};
  src.mode = kRowsStaged;
  src.K = K;
  src.V = V;
  src.k_eff = k_eff;
  src.G = G;
  src.k = k;
  size_t need = 0;
  st = attn_launch_fit(q, q_dtype == KVS_BF16, src, R * G, H, scale, out, lse, scratch,
                       kNoAllocScratchBytes, &need, static_cast<cudaStream_t>(stream));
  if (st == KVS_EINVAL)
    return fail(KVS_EINVAL,
                "sparse_decode_attn_noalloc: R=%d G=%d H=%d k=%d needs %zu bytes of scratch, more "
                "than the fixed %zu-byte array",
                R, G, H, k, need, kNoAllocScratchBytes);
  return st == KVS_OK ? ok() : st;
}
