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
// store by index. Each block takes a split of one (r, g)'s rows, double-buffers
// 64-row K/V tiles into shared memory with cp.async (16-byte copies, zero fill
// for padding rows), computes q.K with one thread per (row, head pair), then a
// warp per head rescales and accumulates P.V. Splits are merged by their
// log-sum-exp in a second small kernel. The bound is HBM: 512 bytes of K/V per
// selected row against ~2 flops per byte.
#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kTile = 64;
constexpr int kThreads = 128;
constexpr int kKStride = kD + 8;  // 272-byte K rows in shared memory: conflict-free 16-byte reads

struct AttnSmem {
  uint16_t K[2][kTile][kKStride];
  uint16_t V[2][kTile][kD];
  float q[8][kD];
  float lg[8][kTile];
  const uint16_t* kp[2][kTile];
  const uint16_t* vp[2][kTile];
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Pointers of row j of (r, g) = u; null when the row is padding.
__device__ __forceinline__ void resolve_row(const RowSrc& src, int u, int j,
                                            const uint16_t*& kp, const uint16_t*& vp) {
  kp = nullptr;
  vp = nullptr;
  if (j >= src.k) return;
  if (src.mode == kRowsStaged) {
    const int ke = src.k_eff ? src.k_eff[u] : src.k;
    if (j < ke) {
      kp = src.K + (static_cast<size_t>(u) * src.k + j) * kD;
      vp = src.V + (static_cast<size_t>(u) * src.k + j) * kD;
    }
    return;
  }
  const int32_t* irow =
      src.idx + (src.idx_shared ? static_cast<size_t>(u / src.G) : static_cast<size_t>(u)) * src.k;
  const int i = irow[j];
  if (i < 0) return;
  if (src.mode == kRowsSlot) {
    const int s = src.slots ? src.slots[static_cast<size_t>(u) * src.k + j]
                            : src.slot_map[static_cast<size_t>(u) * src.n_max + i];
    if (s >= 0) {
      kp = src.hotK + (static_cast<size_t>(u) * src.S + s) * kD;
      vp = src.hotV + (static_cast<size_t>(u) * src.S + s) * kD;
      return;
    }
  }
  kp = src.K + (static_cast<size_t>(u) * src.n_max + i) * kD;
  vp = src.V + (static_cast<size_t>(u) * src.n_max + i) * kD;
}

template <int H>
__global__ void __launch_bounds__(kThreads) sparse_attn_kernel(
    const void* __restrict__ q, int q_bf16, RowSrc src, int nsplit, int rows_per_split,
    float scale_log2, float* __restrict__ out, float* __restrict__ lse,
    float* __restrict__ part) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int u = blockIdx.x / nsplit;
  const int split = blockIdx.x % nsplit;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j_begin = split * rows_per_split;
  const int j_end = min(src.k, j_begin + rows_per_split);
  const int ntiles = j_end > j_begin ? (j_end - j_begin + kTile - 1) / kTile : 0;

  for (int e = tid; e < H * kD; e += kThreads) {
    const size_t off = static_cast<size_t>(u) * H * kD + e;
    const float v = q_bf16 ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(q)[off])
                           : reinterpret_cast<const float*>(q)[off];
    sm.q[e / kD][e % kD] = v * scale_log2;
  }

  auto load_tile = [&](int t, int buf) {
    const int j0 = j_begin + t * kTile;
    if (tid < kTile) {
      const uint16_t *kp, *vp;
      resolve_row(src, u, (j0 + tid < j_end) ? j0 + tid : src.k, kp, vp);
      sm.kp[buf][tid] = kp;
      sm.vp[buf][tid] = vp;
    }
    __syncthreads();
#pragma unroll 4
    for (int e = tid; e < 2 * kTile * 16; e += kThreads) {
      const int which = e >> 10, row = (e >> 4) & (kTile - 1), part16 = e & 15;
      const uint16_t* base = which ? sm.vp[buf][row] : sm.kp[buf][row];
      void* dst = which ? static_cast<void*>(&sm.V[buf][row][part16 * 8])
                        : static_cast<void*>(&sm.K[buf][row][part16 * 8]);
      const void* srcp = base ? static_cast<const void*>(base + part16 * 8) : q;
      cp_async16(dst, srcp, base != nullptr);
    }
    cp_async_commit();
  };

  float m_run[2] = {-__int_as_float(0x7f800000), -__int_as_float(0x7f800000)};
  float l_run[2] = {0.f, 0.f};
  float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};

  if (ntiles > 0) load_tile(0, 0);
  for (int t = 0; t < ntiles; ++t) {
    const int buf = t & 1;
    if (t + 1 < ntiles) {
      load_tile(t + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    // ---- logits: thread = (row, head parity) ----
    {
      const int row = tid & (kTile - 1), hpar = tid >> 6;
      constexpr int NH = (H + 1) / 2;
      float acc[NH];
#pragma unroll
      for (int a = 0; a < NH; ++a) acc[a] = 0.f;
#pragma unroll 4
      for (int d8 = 0; d8 < kD / 8; ++d8) {
        const uint4 kk = *reinterpret_cast<const uint4*>(&sm.K[buf][row][d8 * 8]);
        const float kf[8] = {__uint_as_float(kk.x << 16), __uint_as_float(kk.x & 0xFFFF0000u),
                             __uint_as_float(kk.y << 16), __uint_as_float(kk.y & 0xFFFF0000u),
                             __uint_as_float(kk.z << 16), __uint_as_float(kk.z & 0xFFFF0000u),
                             __uint_as_float(kk.w << 16), __uint_as_float(kk.w & 0xFFFF0000u)};
#pragma unroll
        for (int a = 0; a < NH; ++a) {
          const int h = hpar + 2 * a;
          if (h < H) {
            const float4 q0 = *reinterpret_cast<const float4*>(&sm.q[h][d8 * 8]);
            const float4 q1 = *reinterpret_cast<const float4*>(&sm.q[h][d8 * 8 + 4]);
            acc[a] = fmaf(q0.x, kf[0], acc[a]);
            acc[a] = fmaf(q0.y, kf[1], acc[a]);
            acc[a] = fmaf(q0.z, kf[2], acc[a]);
            acc[a] = fmaf(q0.w, kf[3], acc[a]);
            acc[a] = fmaf(q1.x, kf[4], acc[a]);
            acc[a] = fmaf(q1.y, kf[5], acc[a]);
            acc[a] = fmaf(q1.z, kf[6], acc[a]);
            acc[a] = fmaf(q1.w, kf[7], acc[a]);
          }
        }
      }
      const bool valid = sm.kp[buf][row] != nullptr;
#pragma unroll
      for (int a = 0; a < NH; ++a) {
        const int h = hpar + 2 * a;
        if (h < H) sm.lg[h][row] = valid ? acc[a] : -__int_as_float(0x7f800000);
      }
    }
    __syncthreads();
    // ---- online softmax and P.V: warp w owns heads w and w + 4 ----
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int h = warp + 4 * a;
      if (h < H) {
        const float l0 = sm.lg[h][lane], l1 = sm.lg[h][lane + 32];
        float mx = fmaxf(l0, l1);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
        const float m_new = fmaxf(m_run[a], mx);
        float alpha = 1.f, p0 = 0.f, p1 = 0.f;
        if (m_new != -__int_as_float(0x7f800000)) {
          alpha = exp2f(m_run[a] - m_new);
          p0 = exp2f(l0 - m_new);
          p1 = exp2f(l1 - m_new);
        }
        float ps = p0 + p1;
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, d);
        l_run[a] = l_run[a] * alpha + ps;
        m_run[a] = m_new;
        sm.lg[h][lane] = p0;
        sm.lg[h][lane + 32] = p1;
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 4; ++e) o[a][e] *= alpha;
#pragma unroll 8
        for (int j = 0; j < kTile; ++j) {
          const float p = sm.lg[h][j];
          const uint2 vv = *reinterpret_cast<const uint2*>(&sm.V[buf][j][4 * lane]);
          o[a][0] = fmaf(p, __uint_as_float(vv.x << 16), o[a][0]);
          o[a][1] = fmaf(p, __uint_as_float(vv.x & 0xFFFF0000u), o[a][1]);
          o[a][2] = fmaf(p, __uint_as_float(vv.y << 16), o[a][2]);
          o[a][3] = fmaf(p, __uint_as_float(vv.y & 0xFFFF0000u), o[a][3]);
        }
      }
    }
    __syncthreads();
  }

  // ---- write: final output (one split) or a partial (m, l, o) ----
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int h = warp + 4 * a;
    if (h >= H) continue;
    if (nsplit == 1) {
      const float inv = l_run[a] > 0.f ? 1.f / l_run[a] : 0.f;
      float4 r4 = make_float4(o[a][0] * inv, o[a][1] * inv, o[a][2] * inv, o[a][3] * inv);
      *reinterpret_cast<float4*>(out + (static_cast<size_t>(u) * H + h) * kD + 4 * lane) = r4;
      if (lse && lane == 0)
        lse[static_cast<size_t>(u) * H + h] =
            l_run[a] > 0.f ? (m_run[a] + log2f(l_run[a])) * 0.6931471805599453f
                           : -__int_as_float(0x7f800000);
    } else {
      float* pp = part + ((static_cast<size_t>(u) * nsplit + split) * H + h) * (kD + 4);
      *reinterpret_cast<float4*>(pp + 4 + 4 * lane) = make_float4(o[a][0], o[a][1], o[a][2], o[a][3]);
      if (lane == 0) {
        pp[0] = m_run[a];
        pp[1] = l_run[a];
      }
    }
  }
}

// Merge of the splits of one (r, g): warp h merges head h by log-sum-exp.
__global__ void attn_combine_kernel(const float* __restrict__ part, int nsplit, int H,
                                    float* __restrict__ out, float* __restrict__ lse) {
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
                    float scale_log2, float* out, float* lse, float* part, cudaStream_t s) {
  const size_t smem = sizeof(AttnSmem);
  cudaFuncSetAttribute(sparse_attn_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  sparse_attn_kernel<H><<<RG * nsplit, kThreads, smem, s>>>(q, q_bf16, src, nsplit, rps,
                                                            scale_log2, out, lse, part);
  if (nsplit > 1) attn_combine_kernel<<<RG, H * 32, 0, s>>>(part, nsplit, H, out, lse);
  return check_launch("sparse_decode_attn");
}

}  // namespace

// Split of the k rows across blocks: enough blocks to fill the GPU a few times.
void attn_split(int RG, int k, int& nsplit, int& rows_per_split) {
  const int tiles = max(1, (k + kTile - 1) / kTile);
  const int target = 4 * sm_count();
  nsplit = min(tiles, max(1, (target + RG - 1) / RG));
  const int tiles_per = (tiles + nsplit - 1) / nsplit;
  rows_per_split = tiles_per * kTile;
  nsplit = (tiles + tiles_per - 1) / tiles_per;
}

size_t attn_ws_bytes(int RG, int H, int k) {
  int nsplit, rps;
  attn_split(RG, k, nsplit, rps);
  if (nsplit <= 1) return 0;
  return static_cast<size_t>(RG) * nsplit * H * (kD + 4) * sizeof(float);
}

kvs_status attn_launch(const void* q, int q_bf16, const RowSrc& src, int RG, int H, float scale,
                       float* out, float* lse, void* ws, cudaStream_t s) {
  int nsplit, rps;
  attn_split(RG, src.k, nsplit, rps);
  float* part = static_cast<float*>(ws);
  const float sl2 = scale * 1.4426950408889634f;
  switch (H) {
    case 1: return launch_h<1>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 2: return launch_h<2>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 3: return launch_h<3>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 4: return launch_h<4>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 5: return launch_h<5>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 6: return launch_h<6>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 7: return launch_h<7>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    case 8: return launch_h<8>(q, q_bf16, src, RG, nsplit, rps, sl2, out, lse, part, s);
    default: return fail(KVS_EUNSUPPORTED, "H=%d query heads per KV head (1..8 supported)", H);
  }
}

}  // namespace kvs

// ----------------------------------------------------------------------------
// sparse_decode_attn_noalloc: the same attention for callers that cannot
// allocate device memory. Its split-K partial results (the only scratch the
// attention needs) live in one fixed array of this library instead of a
// caller workspace.
#include <mutex>

namespace {

// 4 MiB of partial results (R*G*nsplit*H*(128+4) floats). The split count
// falls as the batch grows (about 4 blocks per SM in all), so the need stays
// below 8 * SMs * H * 528 bytes: on a 148-SM B200 every size with H <= 4 fits,
// and only H >= 7 with a few hundred (request, KV head) rows exceeds it.
// Every GPU that loads this library holds the array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) float g_attn_scratch[kNoAllocScratchBytes / sizeof(float)];

std::mutex g_scratch_mu;
float* g_scratch_dev[64] = {nullptr};

// Device address of g_attn_scratch on the current device. The name of the
// array in host code is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
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
  const size_t need = attn_ws_bytes(R * G, H, k);
  KVS_REQUIRE(need <= kNoAllocScratchBytes, KVS_EINVAL,
              "sparse_decode_attn_noalloc: R=%d G=%d H=%d k=%d needs %zu bytes of scratch, more "
              "than the fixed %zu-byte array; use sparse_decode_attn with a workspace",
              R, G, H, k, need, kNoAllocScratchBytes);
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
  st = attn_launch(q, q_dtype == KVS_BF16, src, R * G, H, scale, out, lse, scratch,
                   static_cast<cudaStream_t>(stream));
  return st == KVS_OK ? ok() : st;
}
