"""Shared comparison rules of the GPU parity tests.

Tolerances (derived from the f32 arithmetic of the kernels):
  * Fathom scores: the kernels evaluate C + sum_p W_p bit_p(i) in f32 with
    W_p = f32(qbar_c * s_c) * 2^(3-p); against the oracle's fp64 value the
    error is at most (2B + 2D + 16) * 2^-24 * S, where
    S = sum_c |qbar_c| (|m_c| + 15 s_c) bounds |C| + sum_p |W_p|.
  * Selection: identical, or differing only on entries whose oracle score lies
    within a band of the oracle's k-th score: every extra GPU entry has
    S_i >= S_(k) - tol and every missing oracle entry has S_i <= S_(k) + tol,
    tol = 1e-4 * max |S| (the acceptance rule for float-decided selections).
  * Attention: 2e-3 max-abs (f32 accumulation from bf16 K/V).
"""
import numpy as np
import torch

import oracle

ATTN_TOL = 2e-3
LSE_TOL = 1e-3


def fathom_score_tol(qbar, kmin, kstep, B: int, D: int = 128) -> float:
    qbar = np.abs(np.asarray(qbar, np.float64))
    S = float(np.sum(qbar * (np.abs(np.asarray(kmin, np.float64)) + 15 * np.asarray(kstep, np.float64))))
    return (2 * B + 2 * D + 16) * 2.0 ** -24 * S


def check_selection(gpu_idx, ref_idx, ref_scores, k_eff: int, rel=1e-4):
    """Returns the number of differing entries; raises if any lies outside the band."""
    g = np.asarray(gpu_idx)
    r = np.asarray(ref_idx)
    assert np.all(g[k_eff:] == -1), "padding must be -1"
    gs = g[:k_eff]
    assert np.all(np.diff(gs) > 0), "selection must be strictly ascending"
    if np.array_equal(g, r):
        return 0
    s = np.asarray(ref_scores, np.float64)
    rs = r[:k_eff]
    kth = np.min(s[rs])
    tol = rel * np.max(np.abs(s[np.isfinite(s)]))
    extra = np.setdiff1d(gs, rs)
    missing = np.setdiff1d(rs, gs)
    assert extra.size == missing.size
    assert np.all(s[extra] >= kth - tol), (s[extra], kth, tol)
    assert np.all(s[missing] <= kth + tol), (s[missing], kth, tol)
    return int(extra.size)


def check_row_over_selection(idx, slots, misses, out, lse, q, K, V, slot_map, hotK, hotV,
                             k_eff: int, scale: float):
    """One (request, KV head) row of a GPU step against the oracle's gather and
    attention run over the GPU's own selection `idx` (so that rows whose
    selection differs from the oracle's inside the tie band are still checked):
    slots and the miss count bit for bit, out within ATTN_TOL, lse within
    LSE_TOL. slot_map None: every row comes from the full store (all misses).
    q f32/bf16 [H][D]; K, V bf16 [n_max][D]; hotK, hotV bf16 [S][D]."""
    D = K.shape[-1]
    sm = np.full(K.shape[0], -1, np.int32) if slot_map is None else np.asarray(slot_map)
    hK = torch.zeros(1, D, dtype=torch.bfloat16) if hotK is None else hotK
    hV = torch.zeros(1, D, dtype=torch.bfloat16) if hotV is None else hotV
    gK, gV, rs, rm = oracle.gather(np.asarray(idx, np.int32), sm, hK, hV, K, V)
    if slots is not None:
        assert np.array_equal(np.asarray(slots), rs), "slots differ"
    if misses is not None:
        assert int(misses) == rm, (int(misses), rm)
    ro, rl = oracle.attention(q.float(), gK, gV, k_eff, scale)
    err = float(np.max(np.abs(np.asarray(out) - ro)))
    assert err < ATTN_TOL, err
    if lse is not None and k_eff:
        assert float(np.max(np.abs(np.asarray(lse) - rl))) < LSE_TOL
    return err
