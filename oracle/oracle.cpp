// oracle.cpp -- plain CPU reference of the per-step top-k sparse-attention
// decode path (Fathom bit-plane scan, top-k, hot-buffer gather, sparse GQA
// attention, and the lightning-indexer variant).
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this code:
// only the tests, the smoke check and the benchmark's CPU-baseline leg load
// it. It shares no code, header or table with the CUDA library.
//
// Every function is the plain definition, computed in fp64 unless a step is
// defined in f32 (the bit allocation's weights, so that the integer decision
// it takes is reproducible). No blocking, fusion or reordering beyond the
// definition. Sources (page title, section):
//   [FATHOM]   "Fathom: Per-Query Read Depth for Sparse Decoding over
//              Offloaded KV Caches", abstract.
//   [XMSPARSE] "XM-Sparse: Pushing the Throughput Frontier of Sparse Attention
//              with Netpreme X-Mem", Figure 1, "KV management follows the
//              request lifecycle", and the 20% / 40% miss-rate study.
//   [MINIMAX]  "MiniMax-M3: share the sparse index top-k across layers and
//              reuse the decode top-k buffer", description.
// Readings of points the pages leave open are stated where they are used.
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math -std=c++17 -shared -fPIC
// (contraction off keeps every f32 / fp64 operation a single IEEE rounding).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// bf16 bit pattern -> value (bf16 is the top half of an IEEE binary32).
double bf16_to_double(uint16_t h) {
  uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

// OCP FP8 E4M3FN -> value: sign, 4 exponent bits (bias 7), 3 mantissa bits;
// exponent 0 is subnormal (m/8 * 2^-6); 0x7F / 0xFF are NaN; no infinities.
double e4m3_to_double(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
  if (e == 0xF && m == 7) return std::numeric_limits<double>::quiet_NaN();
  double v = (e == 0) ? std::ldexp(static_cast<double>(m), -9)
                      : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

template <typename F>
void parallel_for(int n_items, int nthreads, F fn) {
  if (nthreads <= 1 || n_items <= 1) {
    for (int i = 0; i < n_items; ++i) fn(i);
    return;
  }
  nthreads = std::min(nthreads, n_items);
  std::vector<std::thread> pool;
  for (int t = 0; t < nthreads; ++t)
    pool.emplace_back([&, t]() {
      for (int i = t; i < n_items; i += nthreads) fn(i);
    });
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

int32_t oracle_version(void) { return 1; }

// ---------------------------------------------------------------------------
// O0. The 4-bit channel-major bit-plane K index [FATHOM, abstract: the 4-bit
// K copy is laid out channel by channel as bit planes, and reading the first t
// planes of a channel yields its t-bit quantizer].
// Reading: asymmetric per-channel quantiser over the n keys of this
// (request, KV head): m = min k, s = f32((max k - m)/15) (the step as stored),
// u = floor((k-m)/s + 1/2) in fp64, clamped to 0..15 (s = 0 -> u = 0). Plane p holds bit (3-p) of u, so plane 0
// is the most significant bit and the first t planes hold u >> (4-t). Bit j
// of word w of a plane is key 32w+j; bits of keys >= n are zero.
// var is the population variance of the dequantised values m + s*u, written as
// s^2 * (n*S2 - S1^2)/n^2 with exact integer sums S1 = sum u, S2 = sum u^2,
// and s the stored f32 step.
//   K bf16 [n][D] (row-major, one row per key); planes u32 [D][4][W].
void oracle_build_index(const uint16_t* K, int64_t n, int32_t D, int32_t W, uint32_t* planes,
                        float* kmin, float* kstep, float* kvar) {
  std::memset(planes, 0, sizeof(uint32_t) * static_cast<size_t>(D) * 4 * W);
  for (int32_t c = 0; c < D; ++c) {
    double m = 0.0, M = 0.0;
    for (int64_t i = 0; i < n; ++i) {
      double k = bf16_to_double(K[i * D + c]);
      if (i == 0 || k < m) m = k;
      if (i == 0 || k > M) M = k;
    }
    // the step is stored in f32; codes are decided with the stored step so
    // that m + s*u with the stored (m, s) is the level nearest to each key
    const float s32 = static_cast<float>((M - m) / 15.0);
    const double s = static_cast<double>(s32);
    int64_t S1 = 0, S2 = 0;
    for (int64_t i = 0; i < n; ++i) {
      int64_t u = 0;
      if (s != 0.0) {
        double k = bf16_to_double(K[i * D + c]);
        double x = std::floor((k - m) / s + 0.5);
        u = x < 0.0 ? 0 : (x > 15.0 ? 15 : static_cast<int64_t>(x));
      }
      S1 += u;
      S2 += u * u;
      for (int p = 0; p < 4; ++p)
        if ((u >> (3 - p)) & 1)
          planes[(static_cast<size_t>(c) * 4 + p) * W + static_cast<size_t>(i / 32)] |=
              1u << (i % 32);
    }
    kmin[c] = static_cast<float>(m);
    kstep[c] = s32;
    double var = 0.0;
    if (n > 0) {
      double num = static_cast<double>(n * S2 - S1 * S1);
      double den = static_cast<double>(n) * static_cast<double>(n);
      double s2 = static_cast<double>(s32) * static_cast<double>(s32);
      var = s2 * (num / den);
    }
    kvar[c] = static_cast<float>(var);
  }
}

// ---------------------------------------------------------------------------
// O0b. Per-step write-back of one new token into a row [XMSPARSE, the request
// lifecycle list: the KV generated at each step is written back; FATHOM,
// abstract: the 4-bit bit-plane K copy]. Reading: the new key is coded with
// the row's stored quantiser (m, s), not a re-fitted one -- u = floor((k-m)/s
// + 1/2) in fp64, clamped to 0..15, s = 0 -> u = 0 -- and its four plane bits
// at position i are set to u's bits (plane 0 = MSB); its K and V rows go to
// the full store at i. With a hot slot (slot >= 0) the rows are also copied
// into that slot, the slot's previous token (hot_tok[slot], -1 if none) leaves
// the slot map and the new token takes the slot; without one the new token's
// slot-map entry is -1. kmin, kstep and kvar are left unchanged.
//   knew, vnew bf16 [D]; planes u32 [D][4][W]; full bf16 [n_max][D];
//   slot_map [n_max], hot_tok [S], hot bf16 [S][D] (nullable when slot < 0).
void oracle_append_token(const uint16_t* knew, const uint16_t* vnew, int64_t i, int32_t D, int32_t W,
                         uint32_t* planes, const float* kmin, const float* kstep, uint16_t* fullK,
                         uint16_t* fullV, int32_t* slot_map, int32_t slot, int32_t* hot_tok,
                         uint16_t* hotK, uint16_t* hotV) {
  for (int32_t c = 0; c < D; ++c) {
    const double m = static_cast<double>(kmin[c]);
    const double s = static_cast<double>(kstep[c]);
    int64_t u = 0;
    if (s != 0.0) {
      const double x = std::floor((bf16_to_double(knew[c]) - m) / s + 0.5);
      u = x < 0.0 ? 0 : (x > 15.0 ? 15 : static_cast<int64_t>(x));
    }
    for (int p = 0; p < 4; ++p) {
      uint32_t& w = planes[(static_cast<size_t>(c) * 4 + p) * W + static_cast<size_t>(i / 32)];
      const uint32_t bit = 1u << (i % 32);
      w = ((u >> (3 - p)) & 1) ? (w | bit) : (w & ~bit);
    }
    fullK[static_cast<size_t>(i) * D + c] = knew[c];
    fullV[static_cast<size_t>(i) * D + c] = vnew[c];
    if (slot >= 0) {
      hotK[static_cast<size_t>(slot) * D + c] = knew[c];
      hotV[static_cast<size_t>(slot) * D + c] = vnew[c];
    }
  }
  if (slot_map) {
    if (slot >= 0) {
      if (hot_tok[slot] >= 0) slot_map[hot_tok[slot]] = -1;
      hot_tok[slot] = static_cast<int32_t>(i);
      slot_map[i] = slot;
    } else {
      slot_map[i] = -1;
    }
  }
}

// ---------------------------------------------------------------------------
// O1. Per-query bit allocation [FATHOM, abstract: each query divides its bit
// budget among the key channels by reverse water-filling, with each channel's
// importance weighted by its variance]. Reading: one allocation per (request, KV head) for the summed
// query qbar = ((q0 + q1) + q2) + q3 of its H query heads (the summed raw
// scores sum_h q_h.k = qbar.k), weights w_c = (qbar_c * qbar_c) * var_c in f32,
// and a greedy integer allocation of B bits, 0..4 per channel: each added bit
// divides the channel's quantisation-error variance by 4, so the next bit goes
// to argmax_c w_c * 4^-t_c, ties to the lowest channel. Because each
// channel's values w_c * 4^-j fall with j, the greedy takes exactly the B
// largest events (c, j) in the order (value desc, c asc, j asc); that is what
// is computed here, with the event values formed exactly in fp64.
// Returns 0, or -1 when B is outside 0..4D.
int32_t oracle_plan_bits(const float* q, int32_t H, int32_t D, const float* kvar, int32_t B,
                         uint8_t* t, float* qbar) {
  if (B < 0 || B > 4 * D || H < 1) return -1;
  std::vector<float> w(D);
  for (int32_t c = 0; c < D; ++c) {
    float acc = q[c];
    for (int32_t h = 1; h < H; ++h) acc = acc + q[static_cast<size_t>(h) * D + c];
    qbar[c] = acc;
    float sq = acc * acc;
    w[c] = sq * kvar[c];
  }
  struct Event {
    double value;
    int32_t c, j;
  };
  std::vector<Event> ev;
  ev.reserve(static_cast<size_t>(D) * 4);
  for (int32_t c = 0; c < D; ++c)
    for (int32_t j = 0; j < 4; ++j)
      ev.push_back({std::ldexp(static_cast<double>(w[c]), -2 * j), c, j});
  std::sort(ev.begin(), ev.end(), [](const Event& a, const Event& b) {
    if (a.value != b.value) return a.value > b.value;
    if (a.c != b.c) return a.c < b.c;
    return a.j < b.j;
  });
  for (int32_t c = 0; c < D; ++c) t[c] = 0;
  for (int32_t e = 0; e < B; ++e) t[ev[e].c] += 1;
  return 0;
}

// ---------------------------------------------------------------------------
// O2. The Fathom scan [FATHOM, abstract: a scan over all keys in which the
// query chooses, per channel, how many bits of that channel it reads]: each
// key's score is qbar . khat,
// with channel c of the key read from its first t_c planes only (the t_c-bit
// code v = u >> (4 - t_c)) and reconstructed at the midpoint of that t_c-bit
// quantizer cell: khat = m + s * (2^(4-t) * v + (2^(4-t) - 1) / 2).
// (Reading: the midpoint; any other reconstruction point moves every score by
// the same constant, so the ranking -- and the top-k -- is the same.)
//   planes u32 [D][4][W]; scores fp64 [n].
void oracle_scan(const uint32_t* planes, int32_t D, int32_t W, const float* kmin,
                 const float* kstep, const float* qbar, const uint8_t* t, int64_t n,
                 double* scores) {
  for (int64_t i = 0; i < n; ++i) scores[i] = 0.0;
  for (int32_t c = 0; c < D; ++c) {
    const int tc = t[c];
    const double cell = std::ldexp(1.0, 4 - tc);
    const double m = kmin[c], s = kstep[c], qb = qbar[c];
    for (int64_t i = 0; i < n; ++i) {
      int64_t v = 0;
      for (int p = 0; p < tc; ++p) {
        uint32_t word = planes[(static_cast<size_t>(c) * 4 + p) * W + static_cast<size_t>(i / 32)];
        v = 2 * v + ((word >> (i % 32)) & 1u);
      }
      double khat = m + s * (cell * static_cast<double>(v) + (cell - 1.0) / 2.0);
      scores[i] += qb * khat;
    }
  }
}

// ---------------------------------------------------------------------------
// O3. Exact top-k [XMSPARSE, modelled-throughput section: every request picks
// 2,048 KV entries per layer in each decode step]. Reading: the k_eff = min(k, n) keys first in the
// order (score desc, index asc), output ascending by index, padded with -1.
// Returns k_eff.
}  // extern "C"

template <typename T>
static int32_t topk_impl(const T* scores, int64_t n, int32_t k, int32_t* idx) {
  int64_t k_eff = std::min<int64_t>(k, n);
  std::vector<int64_t> order(static_cast<size_t>(n));
  for (int64_t i = 0; i < n; ++i) order[i] = i;
  auto better = [scores](int64_t a, int64_t b) {
    if (scores[a] != scores[b]) return scores[a] > scores[b];
    return a < b;
  };
  std::nth_element(order.begin(), order.begin() + k_eff, order.end(), better);
  std::sort(order.begin(), order.begin() + k_eff);
  for (int64_t j = 0; j < k; ++j) idx[j] = j < k_eff ? static_cast<int32_t>(order[j]) : -1;
  return static_cast<int32_t>(k_eff);
}

extern "C" {

int32_t oracle_topk(const double* scores, int64_t n, int32_t k, int32_t* idx) {
  return topk_impl(scores, n, k, idx);
}

int32_t oracle_topk_f32(const float* scores, int64_t n, int32_t k, int32_t* idx) {
  return topk_impl(scores, n, k, idx);
}

// ---------------------------------------------------------------------------
// O4. Hot-buffer gather [XMSPARSE, Figure 1 and the lifecycle item on fetching
// selected KV: the decode GPU looks each selected entry up in its own hot
// buffer and brings in only the absent ones; the miss rate counts the selected
// entries not found there]. Reading: slot_map[i] >= 0 is the hot slot holding key i, -1 means
// absent (a miss, served from the full store). Padding (idx -1) gives a zero
// row and slot -2. Returns the miss count.
//   slot_map i32 [n_max]; hot bf16 [S][D]; full bf16 [n_max][D]; g bf16 [k][D].
int32_t oracle_gather(const int32_t* idx, int32_t k, const int32_t* slot_map,
                      const uint16_t* hotK, const uint16_t* hotV, const uint16_t* fullK,
                      const uint16_t* fullV, int32_t D, uint16_t* gK, uint16_t* gV,
                      int32_t* slots) {
  int32_t misses = 0;
  for (int32_t j = 0; j < k; ++j) {
    uint16_t* dk = gK + static_cast<size_t>(j) * D;
    uint16_t* dv = gV + static_cast<size_t>(j) * D;
    int32_t i = idx[j];
    if (i < 0) {
      std::memset(dk, 0, sizeof(uint16_t) * D);
      std::memset(dv, 0, sizeof(uint16_t) * D);
      slots[j] = -2;
      continue;
    }
    int32_t s = slot_map[i];
    slots[j] = s;
    const uint16_t* sk;
    const uint16_t* sv;
    if (s >= 0) {
      sk = hotK + static_cast<size_t>(s) * D;
      sv = hotV + static_cast<size_t>(s) * D;
    } else {
      sk = fullK + static_cast<size_t>(i) * D;
      sv = fullV + static_cast<size_t>(i) * D;
      ++misses;
    }
    std::memcpy(dk, sk, sizeof(uint16_t) * D);
    std::memcpy(dv, sv, sizeof(uint16_t) * D);
  }
  return misses;
}

// ---------------------------------------------------------------------------
// O5. Sparse decode attention over the selected rows only [XMSPARSE, opening
// paragraph: per decode step, attention touches only the chosen KV entries]:
// for each
// query head, l_j = scale * q . K_j over the k_eff rows, o = sum_j softmax(l)_j
// V_j. Naive two-pass softmax in fp64. k_eff = 0 -> o = 0, lse = -inf.
//   q f32 [H][D]; K, V bf16 [k_eff][D]; out fp64 [H][D]; lse fp64 [H].
void oracle_attention(const float* q, int32_t H, int32_t D, const uint16_t* K,
                      const uint16_t* V, int32_t k_eff, double scale, double* out, double* lse) {
  std::vector<double> l(static_cast<size_t>(std::max(k_eff, 0)));
  for (int32_t h = 0; h < H; ++h) {
    double* o = out + static_cast<size_t>(h) * D;
    for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
    if (k_eff <= 0) {
      lse[h] = -std::numeric_limits<double>::infinity();
      continue;
    }
    double mx = -std::numeric_limits<double>::infinity();
    for (int32_t j = 0; j < k_eff; ++j) {
      double dot = 0.0;
      for (int32_t d = 0; d < D; ++d)
        dot += static_cast<double>(q[static_cast<size_t>(h) * D + d]) *
               bf16_to_double(K[static_cast<size_t>(j) * D + d]);
      l[j] = scale * dot;
      mx = std::max(mx, l[j]);
    }
    double den = 0.0;
    for (int32_t j = 0; j < k_eff; ++j) den += std::exp(l[j] - mx);
    for (int32_t j = 0; j < k_eff; ++j) {
      double p = std::exp(l[j] - mx) / den;
      for (int32_t d = 0; d < D; ++d) o[d] += p * bf16_to_double(V[static_cast<size_t>(j) * D + d]);
    }
    lse[h] = mx + std::log(den);
  }
}

// ---------------------------------------------------------------------------
// O6. Lightning-indexer score [MINIMAX, description: every sparse layer runs a
// lightning-indexer pass whose output picks the top-k KV blocks]. Reading (the
// pages give no formula): S_i = sum_h w_h * max(0, q_h . k_i) over the index heads, with
// the e4m3 keys and bf16 queries decoded exactly and summed in fp64.
//   kidx e4m3 [n][Dl]; qidx bf16 [Hi][Dl]; w f32 [Hi]; scores fp64 [n].
void oracle_lightning_scores(const uint8_t* kidx, int64_t n, int32_t Dl, const uint16_t* qidx,
                             int32_t Hi, const float* w, double* scores) {
  for (int64_t i = 0; i < n; ++i) {
    double S = 0.0;
    for (int32_t h = 0; h < Hi; ++h) {
      double dot = 0.0;
      for (int32_t d = 0; d < Dl; ++d)
        dot += bf16_to_double(qidx[static_cast<size_t>(h) * Dl + d]) *
               e4m3_to_double(kidx[static_cast<size_t>(i) * Dl + d]);
      S += static_cast<double>(w[h]) * std::max(0.0, dot);
    }
    scores[i] = S;
  }
}

// Block score = max of the token scores of the block's valid tokens (reading:
// a partial last block takes the max over its tokens < n).
void oracle_block_max(const double* scores, int64_t n, int32_t block, double* bscores) {
  int64_t nb = (n + block - 1) / block;
  for (int64_t b = 0; b < nb; ++b) {
    double mx = -std::numeric_limits<double>::infinity();
    for (int64_t i = b * block; i < std::min<int64_t>(n, (b + 1) * block); ++i)
      mx = std::max(mx, scores[i]);
    bscores[b] = mx;
  }
}

// Block top-k [MINIMAX, description: the selection is made over KV blocks]: the
// kb = k / block best blocks in the order (score desc, block asc), expanded
// to their tokens < n, ascending, padded with -1. Returns the token count.
}  // extern "C"

template <typename T>
static int32_t block_topk_impl(const T* bscores, int64_t n, int32_t block, int32_t k,
                               int32_t* idx) {
  int64_t nb = (n + block - 1) / block;
  int32_t kb = k / block;
  std::vector<int32_t> bidx(static_cast<size_t>(kb));
  int32_t kbe = topk_impl(bscores, nb, kb, bidx.data());
  int32_t cnt = 0;
  for (int32_t j = 0; j < kbe; ++j)
    for (int64_t i = static_cast<int64_t>(bidx[j]) * block;
         i < std::min<int64_t>(n, (static_cast<int64_t>(bidx[j]) + 1) * block); ++i)
      idx[cnt++] = static_cast<int32_t>(i);
  for (int32_t j = cnt; j < k; ++j) idx[j] = -1;
  return cnt;
}

extern "C" {

int32_t oracle_block_topk(const double* bscores, int64_t n, int32_t block, int32_t k,
                          int32_t* idx) {
  return block_topk_impl(bscores, n, block, k, idx);
}

int32_t oracle_block_topk_f32(const float* bscores, int64_t n, int32_t block, int32_t k,
                              int32_t* idx) {
  return block_topk_impl(bscores, n, block, k, idx);
}

// ---------------------------------------------------------------------------
// Batch drivers: the steps above applied to many (request, KV head) rows,
// spread over threads (one row per task). Row u = r*G + g.

// O0 over every row. K bf16 [R][G][n_max][D]; outputs as in oracle_build_index
// with row strides D*4*W (planes) and D (kmin, kstep, kvar).
void oracle_build_index_batch(const uint16_t* K, const int32_t* n, int32_t R, int32_t G,
                              int32_t n_max, int32_t D, int32_t W, uint32_t* planes,
                              float* kmin, float* kstep, float* kvar, int32_t nthreads) {
  parallel_for(R * G, nthreads, [&](int u) {
    int r = u / G;
    oracle_build_index(K + static_cast<size_t>(u) * n_max * D, n[r], D, W,
                       planes + static_cast<size_t>(u) * D * 4 * W, kmin + static_cast<size_t>(u) * D,
                       kstep + static_cast<size_t>(u) * D, kvar + static_cast<size_t>(u) * D);
  });
}

// The Fathom decode step O1 -> O2 -> O3 -> O4 -> O5 for the listed rows
// (rows == NULL: all R*G rows). Outputs are written at each row's position.
//   q f32 [R][G][H][D]; planes [R][G][D][4][W]; kmin/kstep/kvar [R][G][D];
//   slot_map [R][G][n_max] (NULL: every key is read from the full store);
//   hot bf16 [R][G][S][D]; full bf16 [R][G][n_max][D].
//   t [R][G][D]; idx, slots [R][G][k]; misses [R][G]; out [R][G][H][D];
//   lse [R][G][H]; scores (nullable) [R][G][n_max].
// Returns 0, or -1 on a bad budget.
int32_t oracle_decode_batch(const float* q, int32_t R, int32_t G, int32_t H, int32_t D,
                            const uint32_t* planes, int32_t W, const float* kmin,
                            const float* kstep, const float* kvar, const int32_t* n,
                            int32_t n_max, int32_t B, int32_t k, const int32_t* slot_map,
                            const uint16_t* hotK, const uint16_t* hotV, int32_t S,
                            const uint16_t* fullK, const uint16_t* fullV, double scale,
                            const int32_t* rows, int32_t n_rows, int32_t nthreads, uint8_t* t,
                            int32_t* idx, int32_t* slots, int32_t* misses, double* out,
                            double* lse, double* scores) {
  if (B < 0 || B > 4 * D) return -1;
  if (rows == nullptr) n_rows = R * G;
  parallel_for(n_rows, nthreads, [&](int task) {
    const int u = rows ? rows[task] : task;
    const int r = u / G;
    const int64_t nr = n[r];
    std::vector<float> qbar(D);
    uint8_t* tu = t + static_cast<size_t>(u) * D;
    oracle_plan_bits(q + static_cast<size_t>(u) * H * D, H, D, kvar + static_cast<size_t>(u) * D, B,
                     tu, qbar.data());
    std::vector<double> sc(static_cast<size_t>(nr));
    oracle_scan(planes + static_cast<size_t>(u) * D * 4 * W, D, W, kmin + static_cast<size_t>(u) * D,
                kstep + static_cast<size_t>(u) * D, qbar.data(), tu, nr, sc.data());
    if (scores)
      for (int64_t i = 0; i < n_max; ++i)
        scores[static_cast<size_t>(u) * n_max + i] =
            i < nr ? sc[i] : -std::numeric_limits<double>::infinity();
    int32_t* iu = idx + static_cast<size_t>(u) * k;
    int32_t k_eff = oracle_topk(sc.data(), nr, k, iu);
    std::vector<uint16_t> gK(static_cast<size_t>(k) * D), gV(static_cast<size_t>(k) * D);
    std::vector<int32_t> none(static_cast<size_t>(n_max), -1);
    const int32_t* sm = slot_map ? slot_map + static_cast<size_t>(u) * n_max : none.data();
    const uint16_t* hk = hotK ? hotK + static_cast<size_t>(u) * S * D : nullptr;
    const uint16_t* hv = hotV ? hotV + static_cast<size_t>(u) * S * D : nullptr;
    misses[u] = oracle_gather(iu, k, sm, hk, hv, fullK + static_cast<size_t>(u) * n_max * D,
                              fullV + static_cast<size_t>(u) * n_max * D, D, gK.data(), gV.data(),
                              slots + static_cast<size_t>(u) * k);
    oracle_attention(q + static_cast<size_t>(u) * H * D, H, D, gK.data(), gV.data(), k_eff, scale,
                     out + static_cast<size_t>(u) * H * D, lse + static_cast<size_t>(u) * H);
  });
  return 0;
}

// The lightning selection O6 for the listed requests (NULL: all R): token
// scores, block max and block top-k, one selection per request.
//   kidx e4m3 [R][n_max][Dl]; qidx bf16 [R][Hi][Dl]; w f32 [R][Hi];
//   bscores (nullable) fp64 [R][ceil(n_max/block)]; idx [R][k].
void oracle_lightning_batch(const uint8_t* kidx, const uint16_t* qidx, const float* w, int32_t R,
                            int32_t Hi, int32_t Dl, const int32_t* n, int32_t n_max,
                            int32_t block, int32_t k, const int32_t* reqs, int32_t n_reqs,
                            int32_t nthreads, double* bscores, int32_t* idx) {
  if (reqs == nullptr) n_reqs = R;
  const int64_t nbmax = (n_max + block - 1) / block;
  parallel_for(n_reqs, nthreads, [&](int task) {
    const int r = reqs ? reqs[task] : task;
    const int64_t nr = n[r];
    std::vector<double> s(static_cast<size_t>(nr));
    oracle_lightning_scores(kidx + static_cast<size_t>(r) * n_max * Dl, nr, Dl,
                            qidx + static_cast<size_t>(r) * Hi * Dl, Hi, w + static_cast<size_t>(r) * Hi,
                            s.data());
    std::vector<double> bs(static_cast<size_t>(nbmax), -std::numeric_limits<double>::infinity());
    oracle_block_max(s.data(), nr, block, bs.data());
    if (bscores)
      for (int64_t b = 0; b < nbmax; ++b) bscores[static_cast<size_t>(r) * nbmax + b] = bs[b];
    oracle_block_topk(bs.data(), nr, block, k, idx + static_cast<size_t>(r) * k);
  });
}

// O5 for every listed (request, KV head) row over a selection shared by all G
// heads of a request (idx [R][k], -1 padded; the lightning path's layer-group
// reuse reads it twice). q f32 [R][G][H][D]; K, V bf16 [R][G][n_max][D].
void oracle_shared_attention_batch(const float* q, int32_t R, int32_t G, int32_t H, int32_t D,
                                   const uint16_t* K, const uint16_t* V, int32_t n_max,
                                   const int32_t* idx, int32_t k, double scale,
                                   const int32_t* rows, int32_t n_rows, int32_t nthreads,
                                   double* out, double* lse) {
  if (rows == nullptr) n_rows = R * G;
  parallel_for(n_rows, nthreads, [&](int task) {
    const int u = rows ? rows[task] : task;
    const int r = u / G;
    const int32_t* iu = idx + static_cast<size_t>(r) * k;
    std::vector<uint16_t> gK, gV;
    int32_t k_eff = 0;
    for (int32_t j = 0; j < k; ++j) {
      if (iu[j] < 0) continue;
      const uint16_t* sk = K + (static_cast<size_t>(u) * n_max + iu[j]) * D;
      const uint16_t* sv = V + (static_cast<size_t>(u) * n_max + iu[j]) * D;
      gK.insert(gK.end(), sk, sk + D);
      gV.insert(gV.end(), sv, sv + D);
      ++k_eff;
    }
    oracle_attention(q + static_cast<size_t>(u) * H * D, H, D, gK.data(), gV.data(), k_eff, scale,
                     out + static_cast<size_t>(u) * H * D, lse + static_cast<size_t>(u) * H);
  });
}

}  // extern "C"
