/*
 * kvscan.h -- C ABI of libkvscan.so, the B200 (sm_100a) per-step top-k
 * sparse-attention decode path.
 *
 * One decode step, per request r and KV head g:
 *   a1  fathom_plan_bits   per-query bit allocation over the 4-bit K index
 *   a2  index_scan         score every cached key (Fathom bit-plane scan, or
 *                          the lightning-indexer variant)
 *   a3  topk_select        exact top-k of the scores
 *   a4  sparse_gather      fetch the selected K/V rows through the hot-buffer
 *                          slot map, counting misses
 *   a5  sparse_decode_attn GQA softmax attention over the selected rows only
 *   a6  decode_step        a1..a5 fused on one stream
 *   a0  kvs_build_fathom_index  (data preparation) quantise a bf16 K cache to
 *                          the 4-bit channel-major bit-plane index
 *
 * Sources (page title, then section):
 *   [FATHOM]   "Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded
 *              KV Caches", abstract: a 4-bit K copy laid out channel by channel
 *              as bit planes, whose first t planes per channel give the t-bit
 *              quantizer; each query splits a per-key bit budget among channels
 *              by reverse water-filling on variance-weighted importance.
 *   [XMSPARSE] "XM-Sparse: Pushing the Throughput Frontier of Sparse Attention
 *              with Netpreme X-Mem", Figure 1, the request-lifecycle list (the
 *              fetch of selected KV) and the modelled-throughput section: a hot
 *              KV buffer of 4096 tokens in HBM, 2048 entries selected per
 *              step, and a miss rate counting selected entries not in it.
 *   [MINIMAX]  "MiniMax-M3: share the sparse index top-k across layers and
 *              reuse the decode top-k buffer" (SGLang pull request 36527),
 *              description: a lightning indexer that picks KV blocks, one
 *              selection reused by a group of layers, and a fixed int32 output
 *              buffer owned by the caller so that graph capture allocates
 *              nothing.
 *
 * Conventions for every call.
 *   - Every buffer is owned by the caller. Pointers are device pointers (or,
 *     where stated, device aliases of mapped pinned host memory obtained with
 *     cudaHostGetDevicePointer). The library never allocates, frees or
 *     synchronises; it only enqueues kernels on `stream` (a cudaStream_t,
 *     NULL = the legacy default stream). Calls are therefore safe to capture
 *     in a CUDA graph, like the caller-owned top-k buffer of [MINIMAX].
 *   - Stream order holds as usual: a call's kernels start their memory
 *     accesses only after the work enqueued before them on `stream` has
 *     completed. The kernels of one decode_step (and the Fathom scan, the
 *     top-k over scores and the attention) are launched with programmatic
 *     stream serialization: the next kernel may be scheduled while its
 *     predecessor finishes, but waits for it (griddepcontrol.wait) before
 *     its first global access.
 *   - Scratch memory comes from the caller's workspace `ws` of `ws_bytes`
 *     bytes (16-byte aligned); its required size is returned by the matching
 *     kvs_*_workspace_size() query. ws_bytes too small -> KVS_EWORKSPACE.
 *   - Argument errors are found on the host before any launch; then nothing is
 *     written and the call returns KVS_EINVAL / KVS_EUNSUPPORTED. A failed
 *     launch returns KVS_ECUDA. kvs_last_error() gives a thread-local message.
 *   - `dev_status` (nullable) is a device int32 the kernels set to a non-zero
 *     kvs_status when they detect an error on the device (a bounded wait that
 *     ran out: KVS_ETIMEOUT). The caller reads it after its own synchronise;
 *     the library never resets it.
 *   - `n` is always a device int32[R] of per-request valid lengths; n_max
 *     (>= every n[r]) sets the strides. Keys i >= n[r] are never selected.
 *   - Outputs are fully overwritten, padding included.
 *   - bf16 tensors are passed as uint16_t bit patterns, e4m3 (OCP FP8 E4M3FN)
 *     as uint8_t.
 */
#ifndef KVSCAN_H
#define KVSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVS_ABI_VERSION 1

#if defined(__GNUC__)
#define KVS_API __attribute__((visibility("default")))
#else
#define KVS_API
#endif

typedef int32_t kvs_status;
enum {
  KVS_OK = 0,
  KVS_EINVAL = 1,       /* bad argument (null pointer, misalignment, size)     */
  KVS_EUNSUPPORTED = 2, /* valid but not built (e.g. head dim D != 128)        */
  KVS_ECUDA = 3,        /* a CUDA launch failed                                */
  KVS_EWORKSPACE = 4,   /* workspace smaller than the size query returns       */
  KVS_ETIMEOUT = 5,     /* (dev_status only) a bounded device wait ran out     */
  KVS_EBOUNDS = 6       /* (dev_status only) a device-side bounds check failed */
};

enum { KVS_F32 = 0, KVS_BF16 = 1 };              /* q dtypes              */
enum { KVS_SCAN_FATHOM = 0, KVS_SCAN_LIGHTNING = 1 };

/* Returns KVS_ABI_VERSION of the loaded library. */
KVS_API int32_t kvs_abi_version(void);
/* Thread-local text of the last error returned on this thread ("" if none). */
KVS_API const char* kvs_last_error(void);

/* ---------------------------------------------------------------------------
 * The Fathom K index [FATHOM].
 *
 * For every (r, g, channel c) the bf16 keys k_i (i < n[r]) are quantised to
 * 4-bit codes u_i = clamp(floor((k_i - m_c) / s_c + 1/2), 0, 15) (fp64) with
 * m_c = min_i k_i and s_c = f32((max_i k_i - m_c) / 15), the step as stored
 * (s_c = 0 -> all u = 0); so m_c + s_c*u_i is the stored level nearest k_i.
 * Plane p (0..3) of channel c holds bit (3 - p) of u (plane 0 = most
 * significant bit), so the first t planes of a channel hold u >> (4 - t): the
 * channel's t-bit quantizer. Plane words are little-endian bit vectors over
 * keys: bit j of word w is key 32*w + j; bits of keys >= n[r] are 0.
 *
 *   planes  u32 [R][G][D][4][W]   W = words per plane, a multiple of 4 (so each
 *                                 plane starts on a 16-byte boundary),
 *                                 32*W >= n_max
 *   kmin    f32 [R][G][D]         m_c
 *   kstep   f32 [R][G][D]         s_c
 *   kvar    f32 [R][G][D]         population variance over the n[r] keys of the
 *                                 dequantised values m_c + s_c*u, evaluated as
 *                                 f32( (s_c*s_c) * ((n*S2 - S1*S1) / (n*n)) ) in
 *                                 fp64 with S1 = sum u, S2 = sum u^2 (exact
 *                                 integers), s_c the stored f32 step.
 * `planes` may be a mapped pinned host pointer (host_mapped = 1): the scan then
 * reads the index over the host link, the regime [FATHOM] targets.
 * ------------------------------------------------------------------------- */
typedef struct {
  const uint32_t* planes;
  const float* kmin;
  const float* kstep;
  const float* kvar;
  int32_t R, G, D, W;
  int32_t host_mapped;
} kvs_fathom_index;

/* a0: quantise K (bf16 [R][G][n_max][D], token-major) into the index above.
 * D must be 128. Codes are decided in fp64 exactly as written above, so the
 * result is bit-reproducible. Workspace: kvs_build_index_workspace_size(). */
KVS_API kvs_status kvs_build_fathom_index(const uint16_t* K, const int32_t* n, int32_t R, int32_t G,
                                  int32_t n_max, int32_t D, int32_t W, uint32_t* planes,
                                  float* kmin, float* kstep, float* kvar, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream);
KVS_API size_t kvs_build_index_workspace_size(int32_t R, int32_t G, int32_t D);

/* ---------------------------------------------------------------------------
 * a1: per-query bit allocation [FATHOM]: reverse water-filling of the bit
 * budget over channels weighted by variance, read as a greedy integer
 * allocation of B bits per key over the channels, 0..4 bits each.
 *
 * Per (r, g): qbar_c = ((q0_c + q1_c) + q2_c) + q3_c over the H query heads
 * that share KV head g (f32, in this order), w_c = (qbar_c * qbar_c) * kvar_c
 * (f32, two roundings, no fused multiply-add). The 4*D "bit events" (c, j),
 * j = 0..3, have value w_c * 4^-j (exact); the B largest in the order
 * (value desc, c asc, j asc) are taken and t_c counts those of channel c.
 * This is the greedy "next bit to argmax_c w_c*4^-t_c, ties to the lowest c":
 * each bit divides a channel's quantisation-error variance by 4.
 *
 * Outputs (caller-owned):
 *   t          u8  [R][G][D]  bits read of each channel (sum = B)
 *   plane_idx  u16 [R][G][B]  the planes read, as c*4 + p, ascending
 *   plane_w    f32 [R][G][B]  their weights W = f32(qbar_c * s_c) * 2^(3-p)
 *   C          f32 [R][G]     sum_c qbar_c * (m_c + s_c * (2^(4-t_c) - 1) / 2)
 * so that the score of key i is C + sum over the B planes of W * bit(i): the
 * qbar-weighted dot product with each key reconstructed at the midpoint of its
 * t_c-bit quantizer cell. H in 1..8; B in 0..4D, else KVS_EINVAL. */
typedef struct {
  uint8_t* t;
  uint16_t* plane_idx;
  float* plane_w;
  float* C;
  int32_t B;
} kvs_plan;

KVS_API kvs_status fathom_plan_bits(const float* q /* f32 [R][G][H][D] */, int32_t H,
                            const kvs_fathom_index* ix, int32_t B, const kvs_plan* plan,
                            int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * a2: score every key.
 *
 * KVS_SCAN_FATHOM [FATHOM]: scores f32 [R][G][n_max],
 *   score_i = C + sum_{planes (c,p) of the plan} W_(c,p) * bit_(c,p)(i),
 *   for i < n[r]; entries i >= n[r] are written as -inf. The kernel reads
 *   exactly the B planes of the plan: B/8 bytes per key.
 *
 * KVS_SCAN_LIGHTNING [MINIMAX]: per request r and token i < n[r],
 *   S_i = sum_{h < Hi} w_h * max(0, q_h . k_i)
 *   with k_i = kidx e4m3 [R][n_max][Dl], q_h = qidx bf16 [R][Hi][Dl],
 *   w_h = widx f32 [R][Hi], computed on the tcgen05 tensor cores straight on
 *   the e4m3 keys (kind::f8f6f4) with f32 accumulation. Each request's q is
 *   scaled by a power of two and split into two e4m3 parts, hi and the
 *   residual lo, whose sum is q exactly except for components more than 2^10
 *   below the request's largest |q| (their bits below the e4m3 subnormal step
 *   are rounded away). With block > 1 the output is the block score
 *   scores f32 [R][ceil(n_max/block)], b_j = max of S_i over the valid tokens
 *   of block j (-inf for blocks past n[r]); with block == 1 it is S itself,
 *   [R][n_max]. Dl must be 128, Hi a multiple of 16 up to 128, block 1, 32,
 *   64 or 128, kidx 16-byte aligned and R * n_max below 2^31 (KVS_EINVAL /
 *   KVS_EUNSUPPORTED otherwise); KVS_ECUDA when the driver's tensor-map
 *   encoder cannot be reached.
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t kind;
  int32_t R, n_max;
  const int32_t* n;
  /* KVS_SCAN_FATHOM */
  const kvs_fathom_index* ix;
  const kvs_plan* plan;
  /* KVS_SCAN_LIGHTNING */
  const uint8_t* kidx;
  const uint16_t* qidx;
  const float* widx;
  int32_t Hi, Dl, block;
} kvs_scan_args;

KVS_API kvs_status index_scan(const kvs_scan_args* a, float* scores, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * a3: exact top-k [XMSPARSE: 2,048 entries chosen per layer and step;
 * MINIMAX: the block-level selection].
 *
 * block == 1: rows scores f32 [R][G][ld], row (r, g) valid for i < n[r];
 *   selects the k_eff = min(k, n[r]) keys first in the order (score desc,
 *   index asc). idx i32 [R][G][k] receives them ascending by index, then -1.
 * block > 1: rows are block scores [R][G][ld], valid for j < ceil(n[r]/block);
 *   the k/block best blocks in the order (score desc, block asc) are taken
 *   and expanded to their tokens < n[r], ascending; the rest of idx is -1.
 *   k must be a multiple of block.
 * vals (nullable) f32 [R][G][k]: the score of each output (token score, or
 *   the block's score in block mode), -inf for padding.
 * NaN scores are not supported. Workspace: kvs_topk_workspace_size(). */
KVS_API kvs_status topk_select(const float* scores, int64_t ld, const int32_t* n, int32_t R, int32_t G,
                       int32_t k, int32_t block, int32_t* idx, float* vals, void* ws,
                       size_t ws_bytes, int32_t* dev_status, void* stream);
KVS_API size_t kvs_topk_workspace_size(int32_t R, int32_t G, int32_t n_max, int32_t k, int32_t block);

/* ---------------------------------------------------------------------------
 * a4: gather the selected K/V rows [XMSPARSE, Figure 1 and the lifecycle
 * item on fetching selected KV: look each entry up in the local hot buffer and
 * bring in only the absent ones].
 *
 * For each (r, g, j < k) with i = idx[r][g][j] >= 0: s = slot_map[r][g][i];
 *   s >= 0 -> row hotK/hotV[r][g][s] (a hit), s == -1 -> row
 *   fullK/fullV[r][g][i] (a miss). gK/gV[r][g][j] receive the row, slots
 *   receives s, misses[r][g] the number of misses. Padding entries (idx = -1)
 *   get zero rows and slot -2. Hot rows hold bit-identical copies of the full
 *   rows, so the gathered rows do not depend on hit or miss.
 *   idx i32 [R][G][k]; slot_map i32 [R][G][n_max]; hot bf16 [R][G][S][D];
 *   full bf16 [R][G][n_max][D]; gK/gV bf16 [R][G][k][D]; slots i32 [R][G][k];
 *   misses i32 [R][G]. D = 128. */
KVS_API kvs_status sparse_gather(const int32_t* idx, int32_t k, const int32_t* slot_map,
                         const uint16_t* hotK, const uint16_t* hotV, int32_t S,
                         const uint16_t* fullK, const uint16_t* fullV, const int32_t* n,
                         int32_t n_max, int32_t R, int32_t G, int32_t D, uint16_t* gK,
                         uint16_t* gV, int32_t* slots, int32_t* misses, int32_t* dev_status,
                         void* stream);

/* ---------------------------------------------------------------------------
 * a5: GQA decode attention over the selected rows only.
 *
 * For each (r, g, h < H): l_j = scale * (q_h . K_j) over the k_eff rows
 * j < k_eff[r][g] (k when k_eff is NULL), o = sum_j softmax(l)_j V_j, with an
 * online softmax in f32. q f32 or bf16 [R][G][H][D]; K, V bf16 [R][G][k][D];
 * out f32 [R][G][H][D]; lse (nullable) f32 [R][G][H] = log sum_j exp(l_j)
 * (natural log). A head with k_eff = 0 gets out = 0 and lse = -inf.
 * D = 128, H in 1..8. Workspace: kvs_attn_workspace_size(). */
KVS_API kvs_status sparse_decode_attn(const void* q, int32_t q_dtype, const uint16_t* K,
                              const uint16_t* V, const int32_t* k_eff, int32_t R, int32_t G,
                              int32_t H, int32_t D, int32_t k, float scale, float* out,
                              float* lse, void* ws, size_t ws_bytes, int32_t* dev_status,
                              void* stream);
KVS_API size_t kvs_attn_workspace_size(int32_t R, int32_t G, int32_t H, int32_t k);

/* sparse_decode_attn_noalloc: the same computation as sparse_decode_attn
 * (same arguments except that there is no workspace), for callers that cannot
 * allocate device memory: code that runs where cudaMalloc is not allowed or
 * would stall the device (inside a stream being captured into a CUDA graph,
 * allocator-free runtimes that hand the library only their input and output
 * buffers, or latency-critical serving loops that forbid allocation after
 * start-up). The pages have no counterpart: this is a library convenience.
 *
 * Its scratch (the split-K partial results) is one fixed 4 MiB device array
 * inside this library, which every GPU that loads the library holds until the
 * process exits. Each call cuts the k rows into the cheapest number of splits
 * whose partial results fit in that array (R*G*splits*H*132 floats; a single
 * split per (r, g) needs none), so every size is accepted: sizes for which
 * sparse_decode_attn would use more splits than fit run with fewer, at some
 * cost in speed. KVS_EINVAL with a message is returned only for argument
 * errors (and, defensively, if a split ever needed more than the array). The
 * call allocates nothing and calls no allocator. The first call on each
 * device looks up that device's address of the array (with the device
 * current) and caches it for the life of the process (the cache does not
 * survive cudaDeviceReset); make that first call before any stream capture.
 * Every call shares the array: nothing in it has to start at zero (each split
 * writes its whole partial before the merge reads it), but calls that overlap
 * on the same GPU (other streams, other host threads) race on it and must be
 * serialised by the caller. */
KVS_API kvs_status sparse_decode_attn_noalloc(const void* q, int32_t q_dtype, const uint16_t* K,
                                              const uint16_t* V, const int32_t* k_eff, int32_t R,
                                              int32_t G, int32_t H, int32_t D, int32_t k,
                                              float scale, float* out, float* lse,
                                              int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * a6: one fused decode step for all (r, g), on one stream.
 *
 * idx_in == NULL: a1 (plan into `plan`), then a2 and a3. For plans of at
 *   most 144 planes the scan writes every score and the maximum of every
 *   16-key group into the workspace, and a per-row top-k kernel bounds the
 *   k-th score by the k-th largest group maximum, reads back only the groups
 *   that can hold a selected key and selects exactly (ties to the lower
 *   index), writing idx, the slots and the miss counts. For longer plans the
 *   scan keeps top-k candidates per chunk on chip and a per-row merge selects
 *   from them. Then a5 reads K/V straight through slot_map (a4 without
 *   staging), misses counted.
 * idx_in != NULL: the selection is reused and a1..a3 are skipped -- the layer
 *   sharing of [MINIMAX], where a group's first layer selects and the others
 *   reuse it. idx_shared = 1 means idx_in is [R][k], one row per request
 *   shared by all G heads (the lightning indexer's block selection);
 *   otherwise [R][G][k].
 * slot_map == NULL: rows come straight from fullK/fullV (no hot buffer).
 * fullK/fullV may be page-locked host memory mapped into the device's address
 *   space (the full store in the host tier, [XMSPARSE] Figure 1): the step
 *   then reads the missing selected rows over the host link into a staging
 *   area of the workspace and the attention reads every row from HBM (hits
 *   from the hot buffer, misses from the staging); the results are those of
 *   the all-in-HBM step, bit for bit. The workspace must then be
 *   kvs_decode_step_workspace_size_host() bytes (KVS_EWORKSPACE otherwise).
 *
 * Outputs: out f32 [R][G][H][D]; lse (nullable) [R][G][H]; idx (written only
 * when idx_in == NULL) [R][G][k]; slots (nullable) [R][G][k]; misses
 * (nullable) [R][G]. Workspace: kvs_decode_step_workspace_size(). */
typedef struct {
  const void* q;
  int32_t q_dtype, H;
  const kvs_fathom_index* ix;
  const kvs_plan* plan;
  int32_t k;
  const int32_t* n;
  int32_t n_max;
  const int32_t* slot_map;
  const uint16_t* hotK;
  const uint16_t* hotV;
  int32_t S;
  const uint16_t* fullK;
  const uint16_t* fullV;
  const int32_t* idx_in;
  int32_t idx_shared;
  float scale;
  float* out;
  float* lse;
  int32_t* idx;
  int32_t* slots;
  int32_t* misses;
} kvs_decode_args;

KVS_API kvs_status decode_step(const kvs_decode_args* a, void* ws, size_t ws_bytes, int32_t* dev_status,
                       void* stream);
KVS_API size_t kvs_decode_step_workspace_size(int32_t R, int32_t G, int32_t H, int32_t n_max, int32_t k,
                                      int32_t B);
/* Workspace of decode_step when fullK/fullV are in host memory: the above
 * plus two [R][G][k][D] bf16 staging buffers for the fetched misses. */
KVS_API size_t kvs_decode_step_workspace_size_host(int32_t R, int32_t G, int32_t H, int32_t n_max,
                                                   int32_t k, int32_t B);

/* ---------------------------------------------------------------------------
 * kvs_append_token -- the per-step write-back after a decode step: the token
 * just generated joins every (request, KV head) row [XMSPARSE, the request
 * lifecycle list: the generated KV is written back at each step; FATHOM: the
 * 4-bit bit-plane K copy the scan reads].
 *
 * For each request r with i = n[r] < n_max: channel c of KV head g gets the
 * code u = clamp(floor((k - m_c) / s_c + 1/2), 0, 15), computed in fp64 from
 * the bf16 key Knew[r][g][c] with the row's stored kmin/kstep (s_c = 0 -> 0):
 * the quantiser of kvs_build_fathom_index, not re-fitted (kmin, kstep and
 * kvar are left as they are, so a key outside the row's range takes the end
 * code). The four plane bits of key i are set to u's bits (plane 0 = MSB),
 * fullK/fullV[r][g][i] receive Knew/Vnew[r][g], and n[r] grows by one.
 * Slot map and hot buffer (all nullable): without hot_slot, slot_map[r][g][i]
 * (if given) is set to -1 (a miss until a hot-buffer policy brings it in);
 * with hot_slot [R][G], a slot s = hot_slot[r][g] >= 0 receives the new rows
 * in hotK/hotV[r][g][s], the token it held before (hot_tok[r][g][s], -1 when
 * empty) leaves the slot map (slot_map = -1), and hot_tok[r][g][s] = i,
 * slot_map[r][g][i] = s. A request already at n[r] == n_max is left
 * unchanged and KVS_EBOUNDS is written to dev_status.
 *   Knew, Vnew bf16 [R][G][D]; n device int32 [R] (read and advanced);
 *   planes u32 [R][G][D][4][W] (written); kmin, kstep f32 [R][G][D];
 *   fullK, fullV bf16 [R][G][n_max][D]; slot_map i32 [R][G][n_max];
 *   hot_slot i32 [R][G]; hot_tok i32 [R][G][S]; hotK, hotV bf16 [R][G][S][D].
 * D = 128, G <= 8. The pages define no such call signature; it is the
 * write-back step of their request lifecycle. */
KVS_API kvs_status kvs_append_token(const uint16_t* Knew, const uint16_t* Vnew, int32_t* n, int32_t R,
                                    int32_t G, int32_t D, int32_t n_max, uint32_t* planes, int32_t W,
                                    const float* kmin, const float* kstep, uint16_t* fullK,
                                    uint16_t* fullV, int32_t* slot_map, const int32_t* hot_slot,
                                    int32_t* hot_tok, uint16_t* hotK, uint16_t* hotV, int32_t S,
                                    int32_t* dev_status, void* stream);

/* kvs_selftest_scan_timeout -- a check of the bounded waits, without a GPU
 * fault: runs the HBM Fathom scan of index_scan (index in HBM, a plan of
 * 1..144 planes) with one producer warp of every block withholding its
 * arrival on its first chunk and every wait bounded by wait_cycles
 * (1e3 .. 2e9 SM cycles; the library's waits are otherwise bounded by 2e9,
 * about one second). The consumers' wait for that chunk runs out: they write
 * KVS_ETIMEOUT to dev_status (required here), stop waiting, the producers
 * see the block's abort flag, and every block returns with no copy in
 * flight, leaving the context usable. The scores it writes are not
 * meaningful. For tests of the failure path only; the pages define no such
 * call. */
KVS_API kvs_status kvs_selftest_scan_timeout(const kvs_fathom_index* ix, const kvs_plan* plan,
                                             const int32_t* n, int32_t n_max, float* scores,
                                             int64_t wait_cycles, int32_t* dev_status, void* stream);

/* decode_step_timed -- decode_step that also records caller-created CUDA
 * events (cudaEvent_t handles, passed as void*) on `stream` at the boundaries
 * of its stages, so that a caller can time each stage on the device:
 *   events[0] before the bit allocation (a1),
 *   events[1] after it,
 *   events[2] after the scan (a2; on the fused path, the scan kernel that
 *             keeps top-k candidates on chip),
 *   events[3] after the selection (a3: the candidate merge, or the top-k over
 *             scores, and the slot lookup),
 *   events[4] after the attention (a5).
 * With idx_in the skipped stages record their events back to back. Results,
 * workspace and errors are exactly those of decode_step; n_events must be
 * KVS_DECODE_STAGES + 1 and no event may be null (KVS_EINVAL). The events are
 * only recorded, never waited on or destroyed. The pages define no such call;
 * it exists to measure the path. */
#define KVS_DECODE_STAGES 4
KVS_API kvs_status decode_step_timed(const kvs_decode_args* a, void* ws, size_t ws_bytes,
                                     int32_t* dev_status, void* stream, void* const* events,
                                     int32_t n_events);

#ifdef __cplusplus
}
#endif

#endif /* KVSCAN_H */
