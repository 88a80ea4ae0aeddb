// scan_simple.cu -- a2, the Fathom bit-plane scan in its plainest GPU form
// ("Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
// Caches", abstract: the query reads only the planes its allocation chose).
//
// score_i = C + sum over the plan's B planes of W * bit(i). One thread owns a
// 32-key word, reads the B plane words for it (consecutive threads read
// consecutive words of a plane: coalesced) and keeps 32 accumulators. This is
// the reference kernel for the mapped host-memory index, where the host link,
// not the ALU, bounds the scan; the HBM-resident index uses the LUT kernel in
// scan_lut.cu. Inside decode_step it also writes the maximum of every 16-key
// group, so that the host-resident index takes the same top-k over scores as
// the HBM path (scan_topk.cu).
#include "internal.cuh"

namespace kvs {

namespace {

__global__ void __launch_bounds__(128) fathom_scan_simple_kernel(
    const uint32_t* __restrict__ planes, int W, int G, const uint16_t* __restrict__ plane_idx,
    const float* __restrict__ plane_w, const float* __restrict__ Cv, int B,
    const int32_t* __restrict__ n, int n_max, float* __restrict__ scores, float* __restrict__ gmax) {
  extern __shared__ unsigned char smem_raw[];
  float* wsm = reinterpret_cast<float*>(smem_raw);
  uint32_t* offs = reinterpret_cast<uint32_t*>(wsm + B);
  const int u = blockIdx.y;
  const int nr = n[u / G];
  for (int p = threadIdx.x; p < B; p += blockDim.x) {
    wsm[p] = plane_w[static_cast<size_t>(u) * B + p];
    offs[p] = static_cast<uint32_t>(plane_idx[static_cast<size_t>(u) * B + p]) * W;
  }
  __syncthreads();
  const float C = Cv[u];
  const uint32_t* pl = planes + static_cast<size_t>(u) * kD * 4 * W;
  float* out = scores + static_cast<size_t>(u) * n_max;
  const int words = (n_max + 31) / 32;
  for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < words; w += gridDim.x * blockDim.x) {
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.f;
    if (32 * w < nr) {
      for (int p = 0; p < B; ++p) {
        const uint32_t x = pl[offs[p] + w];
        const float wp = wsm[p];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] += ((x >> j) & 1u) ? wp : 0.f;
      }
    }
    const float ninf = -__int_as_float(0x7f800000);
    float m0 = ninf, m1 = ninf;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = 32 * w + j;
      const float v = i < nr ? C + acc[j] : ninf;
      if (i < n_max) out[i] = v;
      if (j < 16) m0 = fmaxf(m0, v);
      else m1 = fmaxf(m1, v);
    }
    if (gmax) {  // maxima of the 16-key groups 2w and 2w + 1 ([RG][ceil(n_max / 16)])
      float* gm = gmax + static_cast<size_t>(u) * ((n_max + 15) / 16);
      if (32 * w < n_max) gm[2 * w] = m0;
      if (32 * w + 16 < n_max) gm[2 * w + 1] = m1;
    }
  }
}

}  // namespace

kvs_status fathom_scan_simple_launch(const uint32_t* planes, int W, int R, int G,
                                     const uint16_t* plane_idx, const float* plane_w,
                                     const float* C, int B, const int32_t* n, int n_max,
                                     float* scores, cudaStream_t s, float* gmax) {
  const int words = (n_max + 31) / 32;
  const int blocks_x = max(1, min((words + 127) / 128, 4 * sm_count() / max(1, R * G) + 1));
  dim3 grid(blocks_x, R * G);
  const size_t smem = static_cast<size_t>(B) * 8;
  fathom_scan_simple_kernel<<<grid, 128, smem, s>>>(planes, W, G, plane_idx, plane_w, C, B, n,
                                                    n_max, scores, gmax);
  return check_launch("index_scan(fathom, simple)");
}

}  // namespace kvs
