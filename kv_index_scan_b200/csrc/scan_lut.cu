// scan_lut.cu -- a2, the Fathom bit-plane scan for an index resident in HBM
// ("Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
// Caches", abstract: each query reads only the planes its allocation chose,
// B bits per key).
//
// score_i = C + sum over the plan's planes of W * bit(i).
//
// Reading B planes costs B/8 bytes per key, but a naive "test a bit, add a
// weight" costs >= 2 ALU operations per (plane, key), far above what B200's
// ALUs deliver per HBM byte (about 0.7 operations per plane bit at full HBM
// bandwidth). This kernel does it in about one:
//
//  * Staging. A producer warp copies, for a chunk of 128 words (4096 keys) of
//    one (request, KV head) row, the planes of one "table set" into a shared
//    memory stage with 1-D TMA bulk copies (cp.async.bulk, 512 bytes per
//    plane), completing on the stage's mbarrier. Stages form a ring; consumer
//    warps release a stage when done with it. Every wait is bounded.
//  * Transpose. Two consumer threads share a 32-key word, 16 keys each. A
//    thread loads its 16-bit half of 32 plane words (conflict-free 2-byte
//    reads), pairs planes k and k + 16 in one register, and finishes the
//    32-plane x 16-key bit transpose in registers (one byte-permute stage,
//    three shift/select stages: ~0.25 operations per bit), giving per key a
//    word of 32 plane bits.
//  * Lookup. The planes are cut into G groups (8 or 16) of b bits (b <= 9);
//    group g has a 2^b-entry table of the sums of its weights. One lookup per
//    key per group replaces b multiply-adds. To keep the 32 lanes of a warp
//    on 32 different shared-memory banks without replicating tables per lane,
//    lane l reads its planes in an order rotated by l groups: at step g it
//    looks up group (g + l) mod G, whose table lives in bank
//    (g + l) mod G + G*(l div G). Tables cost 2^b * 128 bytes per set.
//  * Sets. Plans with more than 144 planes are cut into sets of 16 groups of
//    6 planes, processed one after another into the same accumulators.
//
// The scan writes f32 scores (-inf past n[r]); decode_step instead keeps
// top-k candidates on chip (scan_topk.cu shares this kernel's core).
#include "internal.cuh"
#include "scan_core.cuh"

namespace kvs {

namespace {

template <int G, int b>
__global__ void __launch_bounds__(kScanThreads, 1) fathom_scan_lut_kernel(ScanParams p) {
  ScanCore<G, b> core(p);
  core.run([&](int u, int w0, int nr, const float (&acc)[kKeysPerThread], int t) {
    // write the 16 scores of this thread's half word
    const int i0 = 32 * (w0 + (t >> 1)) + kKeysPerThread * (t & 1);
    if (i0 >= p.n_max) return;
    float* out = p.scores + static_cast<size_t>(u) * p.n_max;
    const float ninf = -__int_as_float(0x7f800000);
    if (i0 + kKeysPerThread <= p.n_max && (p.n_max & 3) == 0) {
#pragma unroll
      for (int j = 0; j < kKeysPerThread; j += 4) {
        float4 v;
        v.x = i0 + j + 0 < nr ? acc[j + 0] : ninf;
        v.y = i0 + j + 1 < nr ? acc[j + 1] : ninf;
        v.z = i0 + j + 2 < nr ? acc[j + 2] : ninf;
        v.w = i0 + j + 3 < nr ? acc[j + 3] : ninf;
        *reinterpret_cast<float4*>(out + i0 + j) = v;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kKeysPerThread; ++j)
        if (i0 + j < p.n_max) out[i0 + j] = i0 + j < nr ? acc[j] : ninf;
    }
  });
}

template <int G, int b>
kvs_status launch_gb(const ScanParams& p, cudaStream_t s) {
  const size_t smem = ScanCore<G, b>::smem_bytes(p.nsets);
  auto kern = fathom_scan_lut_kernel<G, b>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  const int chunks = p.RG * p.chunks_per_row;
  if (chunks <= 0) return KVS_OK;
  const int grid = min(chunks, sm_count());
  kern<<<grid, kScanThreads, smem, s>>>(p);
  return check_launch("index_scan(fathom, lut)");
}

}  // namespace

kvs_status fathom_scan_lut_launch(const ScanParams& p, cudaStream_t s) {
  if (p.G == 8) {
    switch (p.b) {
      case 1: return launch_gb<8, 1>(p, s);
      case 2: return launch_gb<8, 2>(p, s);
      case 3: return launch_gb<8, 3>(p, s);
      case 4: return launch_gb<8, 4>(p, s);
      case 5: return launch_gb<8, 5>(p, s);
      case 6: return launch_gb<8, 6>(p, s);
      case 7: return launch_gb<8, 7>(p, s);
      case 8: return launch_gb<8, 8>(p, s);
      case 9: return launch_gb<8, 9>(p, s);
    }
  } else {
    switch (p.b) {
      case 5: return launch_gb<16, 5>(p, s);
      case 6: return launch_gb<16, 6>(p, s);
      case 7: return launch_gb<16, 7>(p, s);
      case 8: return launch_gb<16, 8>(p, s);
      case 9: return launch_gb<16, 9>(p, s);
    }
  }
  return fail(KVS_EUNSUPPORTED, "index_scan: no LUT schedule for G=%d b=%d", p.G, p.b);
}

}  // namespace kvs
