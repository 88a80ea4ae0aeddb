// build_index.cu -- a0: quantise a bf16 K cache into the 4-bit channel-major
// bit-plane index of "Fathom: Per-Query Read Depth for Sparse Decoding over
// Offloaded KV Caches" (abstract): per (request, KV head, channel) an
// asymmetric 4-bit quantiser over the request's keys, stored as 4 bit planes
// (plane 0 = most significant bit) so that a t-plane prefix is the channel's
// t-bit quantizer.
//
// Data preparation, not on the timed decode path. Three passes:
//   1. per-channel min / max over the valid keys (ordered-int atomics),
//   2. codes u = clamp(floor((k - m)/s + 1/2), 0, 15) in fp64 with the stored
//      f32 step s = f32((max - m)/15), packed 32 keys per word by warp ballots,
//      with exact integer sums of u and u^2 per channel,
//   3. kmin, kstep and the population variance of the dequantised values
//      f32((s*s) * ((n*S2 - S1^2) / (n*n))).
// Every rounding is a single IEEE fp64 operation in a fixed order, so the
// index is bit-reproducible.
#include "internal.cuh"

namespace kvs {

namespace {

constexpr int kMinMaxChunk = 512;  // tokens per block in pass 1
constexpr int kWordsPerBlock = 8;  // 32-key words per block in pass 2

__global__ void init_index_ws(uint32_t* mm, unsigned long long* sums, int total) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    mm[2 * i] = 0xFFFFFFFFu;
    mm[2 * i + 1] = 0u;
    sums[2 * i] = 0ull;
    sums[2 * i + 1] = 0ull;
  }
}

// Pass 1: grid (token chunks, R*G), 256 threads; lane l covers channels 4l..4l+3.
__global__ void __launch_bounds__(256) minmax_kernel(const uint16_t* __restrict__ K,
                                                     const int32_t* __restrict__ n, int G,
                                                     int n_max, uint32_t* __restrict__ mm) {
  const int u = blockIdx.y;
  const int nr = n[u / G];
  const int t0 = blockIdx.x * kMinMaxChunk;
  if (t0 >= nr) return;
  const int t1 = min(nr, t0 + kMinMaxChunk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float lo[4], hi[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    lo[e] = __int_as_float(0x7f800000);
    hi[e] = -__int_as_float(0x7f800000);
  }
  const uint16_t* row = K + (static_cast<size_t>(u) * n_max) * kD + 4 * lane;
  for (int t = t0 + warp; t < t1; t += 8) {
    uint2 v = *reinterpret_cast<const uint2*>(row + static_cast<size_t>(t) * kD);
    float f[4] = {bf16_bits_to_float(v.x & 0xFFFF), bf16_bits_to_float(v.x >> 16),
                  bf16_bits_to_float(v.y & 0xFFFF), bf16_bits_to_float(v.y >> 16)};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      lo[e] = fminf(lo[e], f[e]);
      hi[e] = fmaxf(hi[e], f[e]);
    }
  }
  __shared__ float slo[8][kD], shi[8][kD];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    slo[warp][4 * lane + e] = lo[e];
    shi[warp][4 * lane + e] = hi[e];
  }
  __syncthreads();
  if (threadIdx.x < kD) {
    const int c = threadIdx.x;
    float a = slo[0][c], b = shi[0][c];
    for (int w = 1; w < 8; ++w) {
      a = fminf(a, slo[w][c]);
      b = fmaxf(b, shi[w][c]);
    }
    atomicMin(&mm[2 * (static_cast<size_t>(u) * kD + c)], ordered_key(a));
    atomicMax(&mm[2 * (static_cast<size_t>(u) * kD + c) + 1], ordered_key(b));
  }
}

// The channel's (m, s) from the pass-1 extremes; s is the stored f32 step.
__device__ __forceinline__ void channel_range(const uint32_t* mm, int nr, double& m, float& s32) {
  if (nr <= 0) {
    m = 0.0;
    s32 = 0.f;
    return;
  }
  const double lo = static_cast<double>(key_to_float(mm[0]));
  const double hi = static_cast<double>(key_to_float(mm[1]));
  m = lo;
  s32 = __double2float_rn(__ddiv_rn(__dsub_rn(hi, lo), 15.0));
}

// Pass 2: grid (word chunks, R*G), 128 threads. A 32-key x 128-channel tile is
// staged in shared memory; warp w takes channels w, w+4, ...; lane j is key
// 32*word + j; the four plane words of a channel are ballots of the code bits.
__global__ void __launch_bounds__(128) pack_kernel(const uint16_t* __restrict__ K,
                                                   const int32_t* __restrict__ n, int G,
                                                   int n_max, int W, const uint32_t* __restrict__ mm,
                                                   uint32_t* __restrict__ planes,
                                                   unsigned long long* __restrict__ sums) {
  const int u = blockIdx.y;
  const int nr = n[u / G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ double sm_m[kD], sm_s[kD];
  __shared__ uint16_t tile[32][kD + 2];  // +2 elements: lanes of a warp hit distinct banks
  __shared__ long long s1[kD], s2[kD];
  {
    const int c = threadIdx.x;
    double m;
    float s32;
    channel_range(mm + 2 * (static_cast<size_t>(u) * kD + c), nr, m, s32);
    sm_m[c] = m;
    sm_s[c] = static_cast<double>(s32);
    s1[c] = 0;
    s2[c] = 0;
  }
  uint32_t* pl = planes + static_cast<size_t>(u) * kD * 4 * W;
  const uint16_t* Ku = K + static_cast<size_t>(u) * n_max * kD;
  const int w0 = blockIdx.x * kWordsPerBlock;
  for (int w = w0; w < min(W, w0 + kWordsPerBlock); ++w) {
    __syncthreads();
    const int key0 = 32 * w;
    if (key0 >= nr) {  // past the request: zero words
      for (int e = threadIdx.x; e < kD * 4; e += blockDim.x) pl[static_cast<size_t>(e) * W + w] = 0u;
      continue;
    }
    // stage 32 rows (8 KB) with 16-byte loads; rows past n_max are not read
    for (int e = threadIdx.x; e < 32 * 16; e += blockDim.x) {
      const int rrow = e >> 4, chunk = e & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (key0 + rrow < nr)
        v = *reinterpret_cast<const uint4*>(Ku + static_cast<size_t>(key0 + rrow) * kD + chunk * 8);
      uint32_t* dst = reinterpret_cast<uint32_t*>(&tile[rrow][chunk * 8]);
      dst[0] = v.x;
      dst[1] = v.y;
      dst[2] = v.z;
      dst[3] = v.w;
    }
    __syncthreads();
    const bool valid = key0 + lane < nr;
    for (int c = warp; c < kD; c += 4) {
      int code = 0;
      const double s = sm_s[c];
      if (valid && s != 0.0) {
        const double k = static_cast<double>(bf16_bits_to_float(tile[lane][c]));
        const double x = floor(__dadd_rn(__ddiv_rn(__dsub_rn(k, sm_m[c]), s), 0.5));
        code = x < 0.0 ? 0 : (x > 15.0 ? 15 : static_cast<int>(x));
      }
      const uint32_t b3 = __ballot_sync(0xFFFFFFFFu, code & 8);
      const uint32_t b2 = __ballot_sync(0xFFFFFFFFu, code & 4);
      const uint32_t b1 = __ballot_sync(0xFFFFFFFFu, code & 2);
      const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, code & 1);
      const unsigned a1 = __reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(code));
      const unsigned a2 = __reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(code * code));
      if (lane < 4) {
        const uint32_t word = lane == 0 ? b3 : lane == 1 ? b2 : lane == 2 ? b1 : b0;
        pl[(static_cast<size_t>(c) * 4 + lane) * W + w] = word;
      }
      if (lane == 0) {
        s1[c] += a1;
        s2[c] += a2;
      }
    }
  }
  __syncthreads();
  const int c = threadIdx.x;
  if (s1[c] | s2[c]) {
    atomicAdd(&sums[2 * (static_cast<size_t>(u) * kD + c)], static_cast<unsigned long long>(s1[c]));
    atomicAdd(&sums[2 * (static_cast<size_t>(u) * kD + c) + 1],
              static_cast<unsigned long long>(s2[c]));
  }
}

// Pass 3: one thread per (row, channel).
__global__ void finalize_kernel(const int32_t* __restrict__ n, int G, int RG,
                                const uint32_t* __restrict__ mm,
                                const unsigned long long* __restrict__ sums, float* kmin,
                                float* kstep, float* kvar) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= RG * kD) return;
  const int u = i / kD;
  const long long nr = n[u / G];
  double m;
  float s32;
  channel_range(mm + 2 * static_cast<size_t>(i), static_cast<int>(nr), m, s32);
  kmin[i] = static_cast<float>(m);
  kstep[i] = s32;
  double var = 0.0;
  if (nr > 0) {
    const long long S1 = static_cast<long long>(sums[2 * static_cast<size_t>(i)]);
    const long long S2 = static_cast<long long>(sums[2 * static_cast<size_t>(i) + 1]);
    const double num = static_cast<double>(nr * S2 - S1 * S1);
    const double den = __dmul_rn(static_cast<double>(nr), static_cast<double>(nr));
    const double s2 = __dmul_rn(static_cast<double>(s32), static_cast<double>(s32));
    var = __dmul_rn(s2, __ddiv_rn(num, den));
  }
  kvar[i] = __double2float_rn(var);
}

}  // namespace

size_t build_index_ws_bytes(int R, int G, int D) {
  WsCarver c(nullptr);
  c.take<uint32_t>(static_cast<size_t>(R) * G * D * 2);
  c.take<unsigned long long>(static_cast<size_t>(R) * G * D * 2);
  return c.used;
}

kvs_status build_index_launch(const uint16_t* K, const int32_t* n, int R, int G, int n_max, int W,
                              uint32_t* planes, float* kmin, float* kstep, float* kvar, void* ws,
                              cudaStream_t s) {
  WsCarver c(ws);
  uint32_t* mm = c.take<uint32_t>(static_cast<size_t>(R) * G * kD * 2);
  unsigned long long* sums = c.take<unsigned long long>(static_cast<size_t>(R) * G * kD * 2);
  const int total = R * G * kD;
  init_index_ws<<<(total + 255) / 256, 256, 0, s>>>(mm, sums, total);
  if (n_max > 0) {
    dim3 g1((n_max + kMinMaxChunk - 1) / kMinMaxChunk, R * G);
    minmax_kernel<<<g1, 256, 0, s>>>(K, n, G, n_max, mm);
  }
  dim3 g2((W + kWordsPerBlock - 1) / kWordsPerBlock, R * G);
  pack_kernel<<<g2, 128, 0, s>>>(K, n, G, n_max, W, mm, planes, sums);
  finalize_kernel<<<(total + 255) / 256, 256, 0, s>>>(n, G, R * G, mm, sums, kmin, kstep, kvar);
  return check_launch("build_fathom_index");
}

}  // namespace kvs
