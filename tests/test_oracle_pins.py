"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, brute force on tiny inputs, an invariant, or a library routine (numpy,
torch's own format conversions). No test here needs a GPU.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth

D = 128


def _codes_from_planes(planes, n):
    """Decode 4-bit codes [D][n] from planes [D][4][W] with numpy's bit unpacking
    (little bit order: bit j of word w is key 32w+j; plane 0 = MSB)."""
    Dd, _, W = planes.shape
    bits = np.unpackbits(planes.view(np.uint8).reshape(Dd, 4, W * 4), axis=-1, bitorder="little")
    bits = bits.astype(np.int64)
    u = 8 * bits[:, 0] + 4 * bits[:, 1] + 2 * bits[:, 2] + bits[:, 3]
    return u[:, :n], bits


def _kv(n, seed=0, G=1):
    K, V, _ = synth.fathom_kv(1, G, D, n, seed=seed)
    return K, V


def _bf16_np(t):
    return t.float().numpy().astype(np.float64)


# ----------------------------------------------------------------------------- O0 quantiser

@pytest.mark.parametrize("n", [1, 33, 1000, 4096])
def test_index_is_a_nearest_level_4bit_quantiser(n):
    K, _ = _kv(n, seed=11)
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index(K[0, 0], D, W)
    u, bits = _codes_from_planes(planes, n)
    k = _bf16_np(K[0, 0]).T  # [D][n]
    assert u.min() >= 0 and u.max() <= 15
    # keys past n have zero bits in every plane
    assert not bits[:, :, n:].any()
    m = kmin.astype(np.float64)[:, None]
    s = kstep.astype(np.float64)[:, None]
    # nearest of the 16 stored levels m + s*u: within half a step
    err = np.abs(k - (m + s * u))
    assert np.all(err <= s / 2 * (1 + 1e-12) + 1e-30)
    # the range endpoints map to the end codes
    assert np.array_equal(kmin.astype(np.float64), k.min(axis=1))
    if n > 1:
        rows = np.arange(D)
        assert np.all(u[rows, k.argmin(axis=1)] == 0)
        assert np.all(u[rows, k.argmax(axis=1)] == 15)
        assert np.array_equal(kstep, ((k.max(axis=1) - k.min(axis=1)) / 15).astype(np.float32))
    # monotone: a larger key never gets a smaller code
    for c in range(0, D, 17):
        o = np.argsort(k[c], kind="stable")
        assert np.all(np.diff(u[c, o]) >= 0)
    # var = population variance of the dequantised values (numpy's np.var)
    deq = m + s * u
    ref = deq.var(axis=1)
    assert np.allclose(kvar.astype(np.float64), ref, rtol=4e-7, atol=1e-30)


def test_index_degenerate_channel():
    n = 100
    K, _ = _kv(n, seed=3)
    K[0, 0, :, 5] = 1.5  # a constant channel
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index(K[0, 0], D, W)
    assert kstep[5] == 0 and kvar[5] == 0 and kmin[5] == 1.5
    assert not planes[5].any()


# ----------------------------------------------------------------------------- O1 allocation

def _alloc(w, B):
    """Allocation for exact weights w (H = 1, q = 1 so that w_c = 1*1*var_c exactly)."""
    w = np.asarray(w, np.float32)
    q = np.ones((1, w.size), np.float32)
    t, _ = oracle.plan_bits(q, w, B)
    return t.astype(np.int64)


def _objective(w, t):
    return float(np.sum(np.asarray(w, np.float64) * np.power(4.0, -np.asarray(t, np.float64))))


@pytest.mark.parametrize("B", [0, 1, 4, 68, 92, 136, 511, 512])
def test_alloc_sums_to_budget_and_is_monotone(B):
    rng = np.random.default_rng(B)
    for trial in range(5):
        q = rng.standard_normal((4, D)).astype(np.float32)
        var = np.exp(rng.standard_normal(D) * 1.4).astype(np.float32)
        t, qbar = oracle.plan_bits(q, var, B)
        t = t.astype(np.int64)
        assert t.sum() == B and t.min() >= 0 and t.max() <= 4
        # qbar is the f32 sum of the 4 query heads in order
        assert np.array_equal(qbar, ((q[0] + q[1]) + q[2]) + q[3])
        w = (qbar * qbar) * var  # numpy f32, for the ordering only
        o = np.argsort(-w.astype(np.float64), kind="stable")
        # sorted by weight desc (ties by channel asc), t never increases
        assert np.all(np.diff(t[o]) <= 0)


def test_alloc_closed_forms():
    rng = np.random.default_rng(7)
    w = np.exp(rng.standard_normal(D)).astype(np.float32)
    assert np.all(_alloc(w, 4 * D) == 4)
    assert np.all(_alloc(w, 0) == 0)
    # equal weights: each bit lowers its channel's value by 4x, so the bits go
    # round-robin over the channels (ties to the lowest), B // D each plus one
    # more for the first B % D channels -- the even spread that minimises the
    # convex objective sum_c w 4^-t_c
    eq = np.full(D, 0.75, np.float32)
    for B in [1, 3, 4, 5, 92, 137, 300, 511]:
        t = _alloc(eq, B)
        exp = np.full(D, B // D, np.int64) + (np.arange(D) < B % D)
        assert np.array_equal(t, exp), B
    with pytest.raises(ValueError):
        _alloc(w, 4 * D + 1)


def test_alloc_zero_weights_follow_channel_order():
    w = np.zeros(D, np.float32)
    w[10] = 2.0
    t = _alloc(w, 9)
    exp = np.zeros(D, np.int64)
    exp[10] = 4  # the only positive weight takes its 4 bits first
    exp[0] = 4   # then zero-valued events go by channel, then bit
    exp[1] = 1
    assert np.array_equal(t, exp)


@pytest.mark.parametrize("Dt", [1, 2, 3, 5, 6])
def test_alloc_is_optimal_by_brute_force(Dt):
    """Reverse water-filling: the allocation minimises sum_c w_c 4^-t_c under
    sum t_c = B, 0 <= t_c <= 4 (exhaustive over {0..4}^D)."""
    rng = np.random.default_rng(100 + Dt)
    combos = np.array(list(itertools.product(range(5), repeat=Dt)), np.int64)
    for trial in range(20):
        if trial % 4 == 3:  # ties: powers-of-4 related and equal weights
            w = np.array([4.0 ** rng.integers(-2, 3) for _ in range(Dt)], np.float32)
        else:
            w = np.exp(rng.standard_normal(Dt) * 2).astype(np.float32)
        obj_all = (w.astype(np.float64)[None, :] * np.power(4.0, -combos)).sum(axis=1)
        for B in range(0, 4 * Dt + 1):
            t = _alloc(w, B)
            best = obj_all[combos.sum(axis=1) == B].min()
            assert t.sum() == B
            assert math.isclose(_objective(w, t), best, rel_tol=1e-12, abs_tol=0)


def test_alloc_ties_break_to_lower_channel():
    # w = (1, 4, 1): events 4, 1(c0), 1(c1,j=1), 1(c2), 0.25(c0)...; with B=2 the
    # second bit goes to channel 0 (value 1 at c0 < c1's j=1 event < c2)
    t = _alloc([1.0, 4.0, 1.0], 2)
    assert list(t) == [1, 1, 0]
    t = _alloc([1.0, 4.0, 1.0], 3)
    assert list(t) == [1, 2, 0]
    t = _alloc([1.0, 4.0, 1.0], 4)
    assert list(t) == [1, 2, 1]


# ----------------------------------------------------------------------------- O2 scan

def _setup_row(n, seed=5, H=4):
    K, V = _kv(n, seed=seed)
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index(K[0, 0], D, W)
    q = synth.queries(1, 1, H, D, seed=seed)[0, 0].numpy()
    return K, V, planes, kmin, kstep, kvar, q


@pytest.mark.parametrize("n", [32, 33, 4095, 4096])
def test_full_budget_scan_is_the_dequantised_dot_product(n):
    K, _, planes, kmin, kstep, kvar, q = _setup_row(n)
    t, qbar = oracle.plan_bits(q, kvar, 4 * D)
    s = oracle.scan(planes, kmin, kstep, qbar, t, n)
    u, _ = _codes_from_planes(planes, n)
    deq = kmin.astype(np.float64)[:, None] + kstep.astype(np.float64)[:, None] * u
    ref = qbar.astype(np.float64) @ deq
    scale = np.abs(qbar.astype(np.float64)) @ np.abs(deq)
    assert np.all(np.abs(s - ref) <= 1e-12 * scale)
    # and within half a quantisation step of the exact dot product with K
    k = _bf16_np(K[0, 0]).T
    exact = qbar.astype(np.float64) @ k
    bound = np.abs(qbar.astype(np.float64)) @ (kstep.astype(np.float64) / 2)
    assert np.all(np.abs(s - exact) <= bound * (1 + 1e-6))


@pytest.mark.parametrize("tt", [0, 1, 2, 3, 4])
def test_prefix_of_t_planes_is_the_t_bit_quantiser(tt):
    """One channel at a time (qbar = e_c): the score is the channel's
    reconstruction from its first t planes. It must be the midpoint of a cell of
    2^(4-t) merged 4-bit levels, hold the key within half that cell, and be a
    monotone function of the key."""
    n = 777
    K, _, planes, kmin, kstep, kvar, _ = _setup_row(n, seed=9)
    k = _bf16_np(K[0, 0]).T
    u, _ = _codes_from_planes(planes, n)
    for c in [0, 3, 64, 127]:
        qbar = np.zeros(D, np.float32)
        qbar[c] = 1.0
        t = np.zeros(D, np.uint8)
        t[c] = tt
        khat = oracle.scan(planes, kmin, kstep, qbar, t, n)
        m, s = float(kmin[c]), float(kstep[c])
        cell = 2 ** (4 - tt)
        v = (khat - m) / s / cell - (cell - 1) / (2 * cell)
        assert np.allclose(v, np.round(v), atol=1e-9)
        v = np.round(v).astype(np.int64)
        assert np.array_equal(v, u[c] >> (4 - tt))
        assert np.all(np.abs(k[c] - khat) <= s * cell / 2 * (1 + 1e-6))
        o = np.argsort(k[c], kind="stable")
        assert np.all(np.diff(khat[o]) >= 0)


def test_zero_budget_scores_are_constant_and_topk_is_first_indices():
    n = 1000
    _, _, planes, kmin, kstep, kvar, q = _setup_row(n)
    t, qbar = oracle.plan_bits(q, kvar, 0)
    s = oracle.scan(planes, kmin, kstep, qbar, t, n)
    C = float(np.sum(qbar.astype(np.float64) * (kmin.astype(np.float64) + kstep.astype(np.float64) * 7.5)))
    assert np.allclose(s, C, rtol=1e-12, atol=1e-12)
    assert np.all(s == s[0])
    idx, k_eff = oracle.topk(s, 64)
    assert k_eff == 64 and np.array_equal(idx, np.arange(64))


def test_scan_is_linear_in_qbar_and_reads_only_allocated_planes():
    n = 500
    _, _, planes, kmin, kstep, kvar, q = _setup_row(n)
    t, qbar = oracle.plan_bits(q, kvar, 92)
    s = oracle.scan(planes, kmin, kstep, qbar, t, n)
    # flipping bits of planes beyond each channel's t_c cannot change the scores
    p2 = planes.copy()
    for c in range(D):
        for p in range(t[c], 4):
            p2[c, p] ^= np.uint32(0xFFFFFFFF)
    assert np.array_equal(oracle.scan(p2, kmin, kstep, qbar, t, n), s)
    # flipping a bit inside the prefix changes that key's score by +-W
    c = int(np.argmax(t))
    p3 = planes.copy()
    p3[c, 0, 0] ^= np.uint32(1)
    d = oracle.scan(p3, kmin, kstep, qbar, t, n) - s
    Wc0 = float(qbar[c]) * float(kstep[c]) * 8
    assert math.isclose(abs(d[0]), abs(Wc0), rel_tol=1e-9) and np.all(d[1:] == 0)


# ----------------------------------------------------------------------------- O3 top-k

def _brute_topk(scores, k):
    n = scores.size
    order = np.lexsort((np.arange(n), -scores))  # score desc, index asc
    sel = np.sort(order[: min(k, n)])
    out = np.full(k, -1, np.int64)
    out[: sel.size] = sel
    return out


@pytest.mark.parametrize("n,k", [(1, 1), (10, 3), (37, 37), (37, 50), (1000, 256), (4096, 256)])
def test_topk_matches_full_sort(n, k):
    rng = np.random.default_rng(n * 31 + k)
    for dtype in (np.float64, np.float32):
        s = np.round(rng.standard_normal(n) * 4).astype(dtype)  # many ties
        idx, k_eff = oracle.topk(s, k)
        assert k_eff == min(k, n)
        assert np.array_equal(idx, _brute_topk(s.astype(np.float64), k))


def test_topk_equal_scores_take_lowest_indices():
    s = np.full(300, 2.5)
    idx, _ = oracle.topk(s[np.random.default_rng(0).permutation(300)], 17)
    assert np.array_equal(idx, np.arange(17))


# ----------------------------------------------------------------------------- O4 gather

def test_gather_reads_hot_or_full_rows_and_counts_misses():
    R, G, n, k, S = 1, 2, 3000, 256, 512
    K, V, _ = synth.fathom_kv(R, G, D, n, seed=4)
    rng = np.random.default_rng(1)
    sel = np.stack([np.sort(rng.choice(n, k, replace=False)) for _ in range(G)])[None]
    slot_map, hot_tok = synth.slot_map_from_selection(sel, n, n, S, 0.2, seed=4)
    hotK = synth.hot_rows(K, hot_tok)
    hotV = synth.hot_rows(V, hot_tok)
    for g in range(G):
        gK, gV, slots, m = oracle.gather(sel[0, g], slot_map[0, g], hotK[0, g], hotV[0, g],
                                         K[0, g], V[0, g])
        assert m == round(0.2 * k) == int((slots == -1).sum())
        Kn = K[0, g].view(torch.int16).numpy().view(np.uint16)
        Vn = V[0, g].view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(gK, Kn[sel[0, g]]) and np.array_equal(gV, Vn[sel[0, g]])
        hit = slots >= 0
        assert np.array_equal(hot_tok[0, g][slots[hit]], sel[0, g][hit])
    # padding rows are zero with slot -2
    idx = np.array([5, -1, 7], np.int32)
    gK, gV, slots, m = oracle.gather(idx, slot_map[0, 0], hotK[0, 0], hotV[0, 0], K[0, 0], V[0, 0])
    assert slots[1] == -2 and not gK[1].any() and not gV[1].any()


# ----------------------------------------------------------------------------- O5 attention

def test_attention_over_all_rows_is_dense_softmax_attention():
    n, H = 300, 4
    K, V = _kv(n, seed=21)
    q = synth.queries(1, 1, H, D, seed=21)[0, 0].numpy()
    scale = 1 / math.sqrt(D)
    out, lse = oracle.attention(q, K[0, 0], V[0, 0], n, scale)
    Kf, Vf = _bf16_np(K[0, 0]), _bf16_np(V[0, 0])
    logits = (q.astype(np.float64) @ Kf.T) * scale
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    ref = (p / p.sum(axis=1, keepdims=True)) @ Vf
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, (mx[:, 0] + np.log(p.sum(axis=1))), rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    n, H = 50, 4
    K, V = _kv(n, seed=22)
    q = synth.queries(1, 1, H, D, seed=22)[0, 0].numpy()
    Vf = _bf16_np(V[0, 0])
    out, _ = oracle.attention(q, K[0, 0], V[0, 0], 1, 0.1)
    assert np.array_equal(out, np.tile(Vf[0], (H, 1)))  # one row: exactly V_0
    out, _ = oracle.attention(np.zeros_like(q), K[0, 0], V[0, 0], n, 0.1)
    assert np.allclose(out, np.tile(Vf.mean(axis=0), (H, 1)), rtol=1e-12, atol=1e-13)
    perm = np.random.default_rng(0).permutation(n)
    o1, l1 = oracle.attention(q, K[0, 0], V[0, 0], n, 0.1)
    o2, l2 = oracle.attention(q, K[0, 0][perm], V[0, 0][perm], n, 0.1)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-13) and np.allclose(l1, l2, rtol=1e-13)
    out, lse = oracle.attention(q, K[0, 0], V[0, 0], 0, 0.1)
    assert not out.any() and np.all(np.isneginf(lse))


# ----------------------------------------------------------------------------- O6 lightning

def test_e4m3_and_bf16_decoding_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    finite = ~np.isnan(ref)
    one = torch.tensor([[1.0]], dtype=torch.bfloat16)
    for sign in (1.0, -1.0):
        q = (one * sign)
        s = oracle.lightning_scores(codes[:, None], q, np.ones(1, np.float32))
        assert np.array_equal(s[finite], np.maximum(0.0, sign * ref[finite]))
    # bf16 queries decode exactly: a one-hot key times every bf16 value
    vals = torch.randn(64, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    kone = np.zeros((1, 64), np.uint8)
    for j in range(0, 64, 7):
        kone[:] = 0
        kone[0, j] = 0x38  # e4m3 1.0
        s = oracle.lightning_scores(kone, vals[None, :], np.ones(1, np.float32))
        assert s[0] == max(0.0, float(vals[j]))


def test_lightning_one_hot_weight_is_one_relu_dot():
    R, n, Hi = 1, 200, 8
    kidx, qidx, w, _ = synth.lightning_inputs(R, n, Hi=Hi, seed=5)
    kf = kidx[0].view(torch.float8_e4m3fn).double().numpy()
    qf = qidx[0].double().numpy()
    for h in [0, 3, 7]:
        wh = np.zeros(Hi, np.float32)
        wh[h] = 1.0
        s = oracle.lightning_scores(kidx[0], qidx[0], wh)
        assert np.allclose(s, np.maximum(0.0, kf @ qf[h]), rtol=1e-13, atol=1e-15)
    s = oracle.lightning_scores(kidx[0], qidx[0], w[0])
    ref = np.maximum(0.0, kf @ qf.T) @ w[0].double().numpy()
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-14)


def test_block_max_and_block_topk():
    rng = np.random.default_rng(3)
    n, block, k = 1000, 64, 256
    s = rng.standard_normal(n)
    bm = oracle.block_max(s, block)
    pad = np.full(16 * block, -np.inf)
    pad[:n] = s
    assert np.array_equal(bm, pad.reshape(16, block).max(axis=1))
    idx, cnt = oracle.block_topk(bm, n, block, k)
    top = _brute_topk(bm, k // block)
    exp = np.concatenate([np.arange(b * block, min(n, (b + 1) * block)) for b in np.sort(top)])
    assert cnt == exp.size and np.array_equal(idx[:cnt], exp) and np.all(idx[cnt:] == -1)
    # block = 1 reduces to the token top-k
    idx1, c1 = oracle.block_topk(s, n, 1, 100)
    assert np.array_equal(idx1, oracle.topk(s, 100)[0])


# ----------------------------------------------------------------------------- pipeline

def test_decode_batch_composes_the_steps():
    R, G, H, n, B, k, S = 2, 2, 4, 2000, 92, 128, 256
    K, V, nl = synth.fathom_kv(R, G, D, [n, 1500], n_max=n, seed=8)
    q = synth.queries(R, G, H, D, seed=8)
    W = synth.plane_words(n)
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, W)
    res = oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, k, None, None, None, K, V,
                              1 / math.sqrt(D), want_scores=True)
    for r in range(R):
        for g in range(G):
            p1, m1, s1, v1 = oracle.build_index(K[r, g, : nl[r]], D, W)
            assert np.array_equal(p1, planes[r, g]) and np.array_equal(v1, kvar[r, g])
            t, qbar = oracle.plan_bits(q[r, g], kvar[r, g], B)
            assert np.array_equal(t, res["t"][r, g])
            sc = oracle.scan(planes[r, g], kmin[r, g], kstep[r, g], qbar, t, nl[r])
            assert np.array_equal(sc, res["scores"][r, g, : nl[r]])
            idx, k_eff = oracle.topk(sc, k)
            assert np.array_equal(idx, res["idx"][r, g])
            out, lse = oracle.attention(q[r, g], K[r, g][idx], V[r, g][idx], k_eff, 1 / math.sqrt(D))
            assert np.array_equal(out, res["out"][r, g])
            assert res["misses"][r, g] == k_eff  # no hot buffer: every row is a miss


def _lightning_numpy(kidx, qidx, w, nr, block, k):
    """Lightning selection for one request written out with numpy/torch alone:
    e4m3 and bf16 decoded by torch, S = relu(K Q^T) w in fp64, block max over
    the valid tokens, top (k / block) blocks by (score desc, block asc)."""
    kf = kidx[:nr].view(torch.float8_e4m3fn).double().numpy()
    qf = qidx.double().numpy()
    s = np.maximum(0.0, kf @ qf.T) @ w.double().numpy()
    nb = (nr + block - 1) // block
    pad = np.full(nb * block, -np.inf)
    pad[:nr] = s
    bm = pad.reshape(nb, block).max(axis=1) if nb else np.zeros(0)
    order = np.lexsort((np.arange(nb), -bm))[: k // block]
    toks = [np.arange(b * block, min(nr, (b + 1) * block)) for b in np.sort(order)]
    idx = np.full(k, -1, np.int64)
    if toks:
        t = np.concatenate(toks)
        idx[: t.size] = t
    return bm, idx


def test_lightning_batch_is_the_per_request_selection():
    """Every request of the batch driver equals the selection written out with
    numpy on that request's own slices (ragged lengths, different data per
    request), and a request subset fills only its own rows."""
    nl = [700, 333, 320, 0, 65]
    R, Hi, block, k = len(nl), 16, 64, 256
    kidx, qidx, w, _ = synth.lightning_inputs(R, nl, Hi=Hi, n_max=700, seed=17)
    bs, idx = oracle.lightning_batch(kidx, qidx, w, nl, block, k)
    nbmax = (700 + block - 1) // block
    assert bs.shape == (R, nbmax) and idx.shape == (R, k)
    for r in range(R):
        bm, ref = _lightning_numpy(kidx[r], qidx[r], w[r], nl[r], block, k)
        nb = bm.size
        assert np.allclose(bs[r, :nb], bm, rtol=1e-12, atol=0)
        assert np.all(np.isneginf(bs[r, nb:]))
        assert np.array_equal(idx[r], ref), r
    # the same requests through the subset argument, in another order
    bs2, idx2 = oracle.lightning_batch(kidx, qidx, w, nl, block, k, reqs=[2, 0])
    assert np.array_equal(bs2[[0, 2]], bs[[0, 2]]) and np.array_equal(idx2[[0, 2]], idx[[0, 2]])
    assert not idx2[[1, 3, 4]].any() and not bs2[[1, 3, 4]].any()


def test_shared_attention_batch_reads_each_requests_selection():
    """Every (request, KV head) row attends, with numpy's dense softmax, over
    the rows that request's own selection names in that head's own K/V
    (different selections per request, -1 padding skipped); a row subset fills
    only its rows."""
    R, G, H, n_max, k = 3, 2, 4, 500, 64
    K, V, _ = synth.fathom_kv(R, G, D, [500, 410, 77], n_max=n_max, seed=29)
    q = synth.queries(R, G, H, D, seed=29)
    rng = np.random.default_rng(29)
    idx = np.full((R, k), -1, np.int32)
    for r, (kk, hi) in enumerate([(64, 500), (50, 410), (9, 77)]):
        idx[r, :kk] = np.sort(rng.choice(hi, kk, replace=False))
    scale = 1 / math.sqrt(D)
    out, lse = oracle.shared_attention_batch(q, K, V, idx, scale)
    for r in range(R):
        sel = idx[r][idx[r] >= 0]
        for g in range(G):
            Kf, Vf = _bf16_np(K[r, g])[sel], _bf16_np(V[r, g])[sel]
            logits = (q[r, g].double().numpy() @ Kf.T) * scale
            mx = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - mx)
            assert np.allclose(out[r, g], (p / p.sum(axis=1, keepdims=True)) @ Vf, rtol=1e-12,
                               atol=1e-13)
            assert np.allclose(lse[r, g], mx[:, 0] + np.log(p.sum(axis=1)), rtol=1e-13)
    rows = [5, 0]  # (r=2, g=1) and (r=0, g=0)
    out2, lse2 = oracle.shared_attention_batch(q, K, V, idx, scale, rows=rows)
    for u in range(R * G):
        r, g = divmod(u, G)
        if u in rows:
            assert np.array_equal(out2[r, g], out[r, g]) and np.array_equal(lse2[r, g], lse[r, g])
        else:
            assert not out2[r, g].any()


# ----------------------------------------------------------------------------- O0b append

def test_append_equals_the_build_over_the_longer_row():
    """Appending a key that lies inside the row's per-channel range (so the
    quantiser of the longer row is the same) gives exactly the planes that
    building the index over the longer row gives."""
    n = 700
    K, V = _kv(n + 1, seed=41)
    K[0, 0, n] = ((K[0, 0, :n].float().amax(0) + K[0, 0, :n].float().amin(0)) / 2).to(torch.bfloat16)
    W = synth.plane_words(n + 1)
    planes_n, kmin, kstep, _ = oracle.build_index(K[0, 0, :n], D, W)
    planes_n1, kmin1, kstep1, _ = oracle.build_index(K[0, 0, : n + 1], D, W)
    assert np.array_equal(kmin, kmin1) and np.array_equal(kstep, kstep1)
    fullK = np.zeros((n + 1, D), np.uint16)
    fullV = np.zeros((n + 1, D), np.uint16)
    out = oracle.append_token(K[0, 0, n], V[0, 0, n], n, planes_n, kmin, kstep, fullK, fullV)
    assert np.array_equal(out[0], planes_n1)
    assert np.array_equal(out[1][n], K[0, 0, n].view(torch.int16).numpy().view(np.uint16))


def test_append_copies_an_existing_keys_codes_and_clamps_outside_the_range():
    n = 300
    K, V = _kv(n, seed=42)
    W = synth.plane_words(n + 3)
    planes, kmin, kstep, _ = oracle.build_index(K[0, 0], D, W)
    fullK = np.zeros((n + 3, D), np.uint16)
    fullV = np.zeros((n + 3, D), np.uint16)
    # a copy of key 17 gets key 17's codes
    p1 = oracle.append_token(K[0, 0, 17], V[0, 0, 17], n, planes, kmin, kstep, fullK, fullV)[0]
    u17, _ = _codes_from_planes(p1, n + 1)
    assert np.array_equal(u17[:, n], u17[:, 17])
    # far below every channel's minimum -> 0, far above its maximum -> 15
    lo = torch.full((D,), -1e4, dtype=torch.bfloat16)
    hi = torch.full((D,), 1e4, dtype=torch.bfloat16)
    p2 = oracle.append_token(lo, lo, n + 1, p1, kmin, kstep, fullK, fullV)[0]
    p3 = oracle.append_token(hi, hi, n + 2, p2, kmin, kstep, fullK, fullV)[0]
    u, _ = _codes_from_planes(p3, n + 3)
    assert np.all(u[:, n + 1] == 0) and np.all(u[:, n + 2] == 15)
    assert np.array_equal(u[:, :n + 1], u17)  # earlier keys untouched


def test_append_hot_slot_evicts_the_previous_token():
    n, S = 100, 8
    K, V = _kv(n + 1, seed=43)
    W = synth.plane_words(n + 1)
    planes, kmin, kstep, _ = oracle.build_index(K[0, 0, :n], D, W)
    slot_map = np.full(n + 1, -1, np.int32)
    hot_tok = np.full(S, -1, np.int32)
    slot_map[5], hot_tok[3] = 3, 5
    hotK = np.zeros((S, D), np.uint16)
    hotV = np.zeros((S, D), np.uint16)
    fullK = np.zeros((n + 1, D), np.uint16)
    fullV = np.zeros((n + 1, D), np.uint16)
    _, fK, _, sm, ht, hK, hV = oracle.append_token(K[0, 0, n], V[0, 0, n], n, planes, kmin, kstep, fullK,
                                                   fullV, slot_map, 3, hot_tok, hotK, hotV)
    assert sm[5] == -1 and sm[n] == 3 and ht[3] == n
    assert np.array_equal(hK[3], fK[n]) and np.array_equal(hV[3], V[0, 0, n].view(torch.int16).numpy().view(np.uint16))
    _, _, _, sm2, _, _, _ = oracle.append_token(K[0, 0, n], V[0, 0, n], n, planes, kmin, kstep, fullK, fullV,
                                                slot_map, -1, hot_tok, hotK, hotV)
    assert sm2[n] == -1 and sm2[5] == 3  # no slot: a miss, the hot buffer untouched
