// plan.cu -- a1: per-query bit allocation of "Fathom: Per-Query Read Depth for
// Sparse Decoding over Offloaded KV Caches" (abstract): each query spreads its
// per-key bit budget over the key channels by reverse water-filling on their
// variance-weighted importance.
//
// Reading: for (request r, KV head g) the H query heads sharing the KV head are
// summed, qbar = ((q0 + q1) + q2) + q3 (f32, in order), w_c = (qbar_c*qbar_c) *
// var_c (f32, two roundings), and B bits are given greedily, 0..4 per channel,
// each to argmax_c w_c 4^-t_c with ties to the lowest channel. That greedy takes
// the B largest "bit events" (c, j), value w_c 4^-j, in the order
// (value desc, c asc, j asc). Every event gets a distinct 64-bit key -- the bit
// pattern of the exact double w_c 4^-j (an f32 widened to fp64 has 29 zero low
// mantissa bits) with 511 - (4c + j) in the low bits -- and the events whose
// keys are among the B largest are taken: a bitonic sort of the 512 keys
// (descending; warp shuffles for partners closer than 32, shared memory
// beyond), the first B of it marked. One 512-thread block per (r, g).
#include "internal.cuh"

namespace kvs {

namespace {

__global__ void __launch_bounds__(512) plan_bits_kernel(
    const float* __restrict__ q, int H, const float* __restrict__ kmin,
    const float* __restrict__ kstep, const float* __restrict__ kvar, int B,
    uint8_t* __restrict__ t_out, uint16_t* __restrict__ plane_idx, float* __restrict__ plane_w,
    float* __restrict__ C_out) {
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  __shared__ float qb[kD], wv[kD];
  __shared__ unsigned long long kbuf[2][4 * kD];
  __shared__ int tcount[kD], start[kD];
  __shared__ unsigned char took[4 * kD];
  __shared__ float cterm[kD];
  if (tid < kD) {
    const float* qq = q + static_cast<size_t>(u) * H * kD;
    float acc = qq[tid];
    for (int h = 1; h < H; ++h) acc = __fadd_rn(acc, qq[h * kD + tid]);
    qb[tid] = acc;
    wv[tid] = __fmul_rn(__fmul_rn(acc, acc), kvar[static_cast<size_t>(u) * kD + tid]);
  }
  __syncthreads();
  const int c = tid >> 2, j = tid & 3;
  unsigned long long x;
  {
    const double scale = j == 0 ? 1.0 : j == 1 ? 0.25 : j == 2 ? 0.0625 : 0.015625;
    double v = __dmul_rn(static_cast<double>(wv[c]), scale);
    v = v > 0.0 ? v : 0.0;  // -0 -> +0 (weights are non-negative)
    x = static_cast<unsigned long long>(__double_as_longlong(v)) | static_cast<unsigned long long>(511 - tid);
  }
  took[tid] = 0;
  // bitonic sort, descending, one key per thread: the partner at distance
  // `stride` is read by warp shuffle below 32 and through shared memory (two
  // buffers in turn, one barrier per stage) above
  int buf = 0;
  for (int size = 2; size <= 4 * kD; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      unsigned long long y;
      if (stride >= 32) {
        kbuf[buf][tid] = x;
        __syncthreads();
        y = kbuf[buf][tid ^ stride];
        buf ^= 1;
      } else {
        y = __shfl_xor_sync(0xFFFFFFFFu, x, stride);
      }
      const bool keep_max = ((tid & size) == 0) == ((tid & stride) == 0);
      x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
    }
  }
  __syncthreads();  // took[] cleared by every thread
  if (tid < B) took[511 - static_cast<int>(x & 511ull)] = 1;
  __syncthreads();
  const bool taken = took[tid] != 0;
  const unsigned ball = __ballot_sync(0xFFFFFFFFu, taken);
  const int tc = __popc((ball >> ((tid & 31) & ~3)) & 0xFu);
  if (j == 0) {
    tcount[c] = tc;
    t_out[static_cast<size_t>(u) * kD + c] = static_cast<uint8_t>(tc);
    const float m = kmin[static_cast<size_t>(u) * kD + c];
    const float s = kstep[static_cast<size_t>(u) * kD + c];
    const float half = tc == 0 ? 7.5f : tc == 1 ? 3.5f : tc == 2 ? 1.5f : tc == 3 ? 0.5f : 0.f;
    cterm[c] = __fmul_rn(qb[c], __fadd_rn(m, __fmul_rn(s, half)));
  }
  __syncthreads();
  // exclusive prefix of t over channels (plane list is ascending in c*4 + p)
  if (tid < 32) {
    int v[4], run = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[e] = tcount[4 * tid + e];
      run += v[e];
    }
    int incl = run;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (tid >= d) incl += o;
    }
    int ex = incl - run;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      start[4 * tid + e] = ex;
      ex += v[e];
    }
  } else if (tid < 64) {
    // C = sum_c qbar_c (m_c + s_c (2^(4-t_c) - 1)/2), fixed tree order
    const int l = tid - 32;
    float a = __fadd_rn(__fadd_rn(cterm[l], cterm[l + 32]), __fadd_rn(cterm[l + 64], cterm[l + 96]));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) a = __fadd_rn(a, __shfl_down_sync(0xFFFFFFFFu, a, d));
    if (l == 0) C_out[u] = a;
  }
  __syncthreads();
  if (taken) {  // the taken events of a channel are its planes p = j < t_c
    const int slot = start[c] + j;
    const float s = kstep[static_cast<size_t>(u) * kD + c];
    plane_idx[static_cast<size_t>(u) * B + slot] = static_cast<uint16_t>(4 * c + j);
    plane_w[static_cast<size_t>(u) * B + slot] =
        __fmul_rn(__fmul_rn(qb[c], s), static_cast<float>(8 >> j));
  }
}

}  // namespace

kvs_status plan_bits_launch(const float* q, int H, const float* kmin, const float* kstep,
                            const float* kvar, int RG, int B, uint8_t* t, uint16_t* plane_idx,
                            float* plane_w, float* C, cudaStream_t s) {
  launch_chained(plan_bits_kernel, dim3(RG), dim3(512), 0, s, q, H, kmin, kstep, kvar, B, t, plane_idx,
                 plane_w, C);
  return check_launch("fathom_plan_bits");
}

}  // namespace kvs
