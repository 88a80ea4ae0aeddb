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
//  * Staging. A producer warp copies, for a chunk of 16 words per consumer
//    warp (192 words, 6,144 keys, with 12 consumer warps) of one (request, KV
//    head) row, the planes of one "table set" into a shared memory stage with
//    1-D TMA bulk copies (cp.async.bulk, one per plane), completing on the
//    stage's mbarrier. Stages form a ring; consumer warps release a stage when
//    done with it. Every wait is bounded.
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
//    the thread pair of lanes (2i, 2i+1) reads its planes in an order rotated
//    by i groups: at step g it looks up group (g + i) mod G, in one of the
//    32/G replicas of the tables, so that the 32 lanes hit 32 distinct banks.
//    Tables cost 2^b * 128 bytes per set.
//  * Sets. Plans with more than 144 planes are cut into sets of 16 groups of
//    6 planes, processed one after another into the same accumulators.
//
// The scan writes f32 scores (-inf past n[r]); decode_step instead keeps
// top-k candidates on chip (scan_topk.cu shares this kernel's core).
#include "internal.cuh"
#include "scan_core.cuh"
#include "scan_prmt.cuh"

namespace kvs {

namespace {

template <int G, int b, int W>
__global__ void KVS_SCAN_BOUNDS(G, b, W) fathom_scan_lut_kernel(ScanParams p) {
  using Core = ScanCore<G, b, W>;
  Core core(p);
  core.run([&](int u, int c, int nr, const float (&acc)[kKeysPerThread], int t) {
    // write the 16 scores of this thread's half word
    const int i0 = 32 * (c * Core::CHUNK_WORDS + (t >> 1)) + kKeysPerThread * (t & 1);
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

struct LutLaunch {
  const ScanParams& p;
  cudaStream_t s;
  template <int G, int b, int W>
  kvs_status operator()() const {
    using Core = ScanCore<G, b, W>;
    const size_t smem = Core::smem_bytes(p.nsets);
    auto kern = fathom_scan_lut_kernel<G, b, W>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    ScanParams q = p;
    q.warps = W;
    q.chunks_per_row = scan_chunks_per_row(p.n_max, W);
    q.nstage = Core::nstages(p.nsets);
    const int chunks = q.RG * q.chunks_per_row;
    if (chunks <= 0) return KVS_OK;
    const int grid = min(chunks, sm_count());
    kern<<<grid, Core::THREADS, smem, s>>>(q);
    return check_launch("index_scan(fathom, lut)");
  }
};

// Plans of at most 144 planes: the byte-indexed lookup core (scan_prmt.cuh).
// Thread t writes the 16 consecutive scores of its half plane word.
__global__ void __launch_bounds__(kPThreads, 1) fathom_scan_prmt_kernel(ScanParams p) {
  pdl_wait();
  pdl_trigger();
  ScanCoreP core(p);
  core.run([&](int u, int c, int nr, const float (&acc)[kPKeys], int t) {
    const int i0 = ScanCoreP::key0(c, t);
    if (i0 >= p.n_max) return;
    float* out = p.scores + static_cast<size_t>(u) * p.n_max;
    const float ninf = -__int_as_float(0x7f800000);
    if (p.gmax) {
      float m = ninf;
#pragma unroll
      for (int j = 0; j < kPKeys; ++j) m = fmaxf(m, i0 + j < nr ? acc[j] : ninf);
      p.gmax[static_cast<size_t>(u) * ((p.n_max + kPKeys - 1) / kPKeys) + i0 / kPKeys] = m;
    }
    if (i0 + kPKeys <= p.n_max && (p.n_max & 3) == 0) {
#pragma unroll
      for (int j = 0; j < kPKeys; j += 4) {
        float4 v;
        v.x = i0 + j + 0 < nr ? acc[j + 0] : ninf;
        v.y = i0 + j + 1 < nr ? acc[j + 1] : ninf;
        v.z = i0 + j + 2 < nr ? acc[j + 2] : ninf;
        v.w = i0 + j + 3 < nr ? acc[j + 3] : ninf;
        *reinterpret_cast<float4*>(out + i0 + j) = v;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPKeys; ++j)
        if (i0 + j < p.n_max) out[i0 + j] = i0 + j < nr ? acc[j] : ninf;
    }
  });
}

}  // namespace

kvs_status fathom_scan_lut_launch(const ScanParams& p, cudaStream_t s) {
  if (p.B <= kPMaxB) {
    ScanParams q = p;
    q.chunks_per_row = prmt_chunks_per_row(p.n_max);
    q.nstage = prmt_nstages(p.B, 0);
    const int chunks = q.RG * q.chunks_per_row;
    if (chunks <= 0) return KVS_OK;
    const size_t smem = prmt_smem_bytes(p.B, q.nstage, 0);
    cudaFuncSetAttribute(fathom_scan_prmt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    launch_chained(fathom_scan_prmt_kernel, dim3(min(chunks, sm_count())), dim3(kPThreads), smem, s, q);
    return check_launch("index_scan(fathom, prmt)");
  }
  return dispatch_schedule(p, LutLaunch{p, s});
}

}  // namespace kvs
