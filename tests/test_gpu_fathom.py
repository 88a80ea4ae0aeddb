"""GPU parity of the Fathom path against the CPU oracle, through the C ABI.

Integer work (index codes, bit allocation, top-k on identical scores, slots,
misses) is compared bit for bit; float work within the tolerances of
tests/_parity.py. Sizes span several tiles and a ragged tail.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import ATTN_TOL, check_row_over_selection, check_selection, fathom_score_tol

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_index_scan_b200
    return kv_index_scan_b200


DEV = "cuda"


def _np(t):
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return t.numpy()


# ----------------------------------------------------------------------------- a0 index

@pytest.mark.parametrize("R,G,nl,n_max", [(1, 1, [4096], 4096), (2, 3, [1000, 33], 1030),
                                          (1, 2, [32], 32), (2, 1, [0, 5000], 5000)])
def test_index_build_bit_exact(kvs, R, G, nl, n_max):
    K, _, _ = synth.fathom_kv(R, G, D, nl, n_max=n_max, seed=21, with_v=False)
    W = kvs.plane_words(n_max)
    ix = kvs.build_fathom_index(K.to(DEV), nl, W)
    torch.cuda.synchronize()
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, W)
    assert np.array_equal(_np(ix.planes).view(np.uint32), planes)
    assert np.array_equal(_np(ix.kmin), kmin)
    assert np.array_equal(_np(ix.kstep), kstep)
    assert np.array_equal(_np(ix.kvar), kvar)


# ----------------------------------------------------------------------------- a1 allocation

@pytest.mark.parametrize("B", [0, 1, 4, 68, 92, 136, 511, 512])
def test_plan_bits_bit_exact(kvs, B):
    R, G, H, n = 2, 4, 4, 3000
    K, _, nl = synth.fathom_kv(R, G, D, n, seed=B + 1, with_v=False)
    q = synth.queries(R, G, H, D, seed=B + 1)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    plan = kvs.fathom_plan_bits(q.to(DEV), ix, B)
    torch.cuda.synchronize()
    kvar, kmin, kstep = _np(ix.kvar), _np(ix.kmin), _np(ix.kstep)
    t_gpu = _np(plan.t)
    for r in range(R):
        for g in range(G):
            t, qbar = oracle.plan_bits(q[r, g], kvar[r, g], B)
            assert np.array_equal(t_gpu[r, g], t)
            if B == 0:
                continue
            pidx = _np(plan.plane_idx)[r, g, :B].view(np.uint16).astype(np.int64)
            exp = np.array([4 * c + p for c in range(D) for p in range(t[c])], np.int64)
            assert np.array_equal(pidx, exp)
            c, p = exp // 4, exp % 4
            wref = qbar[c].astype(np.float64) * kstep[r, g][c].astype(np.float64) * 2.0 ** (3 - p)
            assert np.allclose(_np(plan.plane_w)[r, g, :B], wref, rtol=2 ** -23, atol=0)
            cref = np.sum(qbar.astype(np.float64) * (kmin[r, g].astype(np.float64) + kstep[r, g].astype(np.float64)
                                                     * (2.0 ** (4 - t.astype(np.float64)) - 1) / 2))
            tol = fathom_score_tol(qbar, kmin[r, g], kstep[r, g], 0)
            assert abs(float(_np(plan.C)[r, g]) - cref) <= tol


@pytest.mark.parametrize("B", [1, 37, 92, 136, 300, 511])
def test_plan_bits_bit_exact_with_tied_and_zero_weights(kvs, B):
    """Channels with equal variances and queries with few distinct values give
    many equal weights w_c (ties go to the lowest channel), constant channels
    give w_c = 0, and weights 4x apart tie across bit positions."""
    R, G, H, n = 1, 4, 4, 256
    gen = torch.Generator().manual_seed(B)
    base = torch.randn(n, generator=gen)
    scale = torch.tensor([1.0, 2.0, 0.5, 0.0])[torch.randint(0, 4, (R, G, D), generator=gen)]
    K = (base.view(1, 1, n, 1) * scale.view(R, G, 1, D)).to(torch.bfloat16).contiguous()
    q = torch.tensor([-1.0, 0.5, 1.0, 2.0])[torch.randint(0, 4, (R, G, H, D), generator=gen)]
    q[0, 3] = 0.0
    q[0, 3, 0] = torch.pow(2.0, torch.randint(-3, 4, (D,), generator=gen).float())
    ix = kvs.build_fathom_index(K.to(DEV), [n] * R)
    plan = kvs.fathom_plan_bits(q.to(DEV), ix, B)
    torch.cuda.synchronize()
    kvar, t_gpu = _np(ix.kvar), _np(plan.t)
    for g in range(G):
        t, _ = oracle.plan_bits(q[0, g], kvar[0, g], B)
        assert np.array_equal(t_gpu[0, g], t), g
        pidx = _np(plan.plane_idx)[0, g, :B].view(np.uint16).astype(np.int64)
        assert np.array_equal(pidx, [4 * c + p for c in range(D) for p in range(t[c])])


# ----------------------------------------------------------------------------- a2 scan

@pytest.mark.parametrize("B", [0, 1, 7, 33, 68, 72, 73, 92, 136, 144, 145, 300, 512])
@pytest.mark.parametrize("nl,n_max", [([4096, 4095], 4096), ([33, 1], 64), ([20000, 12345], 20000),
                                      ([0, 70000], 70001)])
def test_fathom_scan_within_f32_error(kvs, B, nl, n_max):
    R, G, H = 2, 2, 4
    K, _, _ = synth.fathom_kv(R, G, D, nl, n_max=n_max, seed=7, with_v=False)
    q = synth.queries(R, G, H, D, seed=7)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    plan = kvs.fathom_plan_bits(q.to(DEV), ix, B)
    sc = kvs.index_scan_fathom(ix, plan, nl, n_max)
    torch.cuda.synchronize()
    sc = _np(sc)
    planes, kmin, kstep, kvar = (_np(ix.planes).view(np.uint32), _np(ix.kmin), _np(ix.kstep), _np(ix.kvar))
    for r in range(R):
        for g in range(G):
            t, qbar = oracle.plan_bits(q[r, g], kvar[r, g], B)
            ref = oracle.scan(planes[r, g], kmin[r, g], kstep[r, g], qbar, t, nl[r])
            tol = fathom_score_tol(qbar, kmin[r, g], kstep[r, g], B)
            assert np.max(np.abs(sc[r, g, : nl[r]] - ref), initial=0) <= tol
            assert np.all(np.isneginf(sc[r, g, nl[r]:]))


# ----------------------------------------------------------------------------- a3 top-k

@pytest.mark.parametrize("n,k", [(1, 1), (100, 7), (4096, 256), (4097, 2048), (131072, 2048),
                                 (70000, 3000), (50, 64)])
def test_topk_bit_exact_on_identical_scores(kvs, n, k):
    rng = np.random.default_rng(n + k)
    R, G = 2, 3
    nl = [n, max(1, n // 3)]
    s = np.round(rng.standard_normal((R, G, n)) * 50).astype(np.float32)  # many ties
    s[:, :, ::97] = s[:, :, 0:1]  # more exact ties
    st = torch.from_numpy(s).to(DEV)
    idx, vals = kvs.topk_select(st, nl, k, want_vals=True)
    torch.cuda.synchronize()
    idx, vals = _np(idx), _np(vals)
    for r in range(R):
        for g in range(G):
            ref, ke = oracle.topk(s[r, g, : nl[r]].copy(), k)
            assert np.array_equal(idx[r, g], ref)
            assert np.array_equal(vals[r, g, :ke], s[r, g][ref[:ke]])
            assert np.all(np.isneginf(vals[r, g, ke:]))


@pytest.mark.parametrize("n,block,k", [(80000, 64, 2048), (1000, 64, 256), (4096, 32, 2048),
                                       (100, 64, 2048)])
def test_block_topk_bit_exact(kvs, n, block, k):
    rng = np.random.default_rng(n)
    R = 3
    nl = [n, n - 17, max(1, n // 5)]
    nb = (n + block - 1) // block
    s = np.round(rng.standard_normal((R, nb)) * 20).astype(np.float32)
    idx = _np(kvs.topk_select(torch.from_numpy(s).to(DEV), nl, k, block=block))
    for r in range(R):
        nbr = (nl[r] + block - 1) // block
        ref, cnt = oracle.block_topk(s[r, :nbr].copy(), nl[r], block, k)
        assert np.array_equal(idx[r], ref)


# ----------------------------------------------------------------------------- a4 gather

def test_gather_bit_exact(kvs):
    R, G, n, k, S = 2, 3, 5000, 512, 1024
    K, V, nl = synth.fathom_kv(R, G, D, [n, 3000], n_max=n, seed=5)
    rng = np.random.default_rng(0)
    sel = np.full((R, G, k), -1, np.int32)
    for r in range(R):
        for g in range(G):
            kk = k if r == 0 else k - 100  # ragged selections with -1 padding
            sel[r, g, :kk] = np.sort(rng.choice(nl[r], kk, replace=False))
    slot_map, hot_tok = synth.slot_map_from_selection(sel, nl, n, S, 0.2, seed=5)
    hotK, hotV = synth.hot_rows(K, hot_tok), synth.hot_rows(V, hot_tok)
    gK, gV, slots, misses = kvs.sparse_gather(torch.from_numpy(sel).to(DEV),
                                              torch.from_numpy(slot_map).to(DEV), hotK.to(DEV),
                                              hotV.to(DEV), K.to(DEV), V.to(DEV), nl)
    torch.cuda.synchronize()
    for r in range(R):
        for g in range(G):
            rK, rV, rs, rm = oracle.gather(sel[r, g], slot_map[r, g], hotK[r, g], hotV[r, g], K[r, g], V[r, g])
            assert np.array_equal(_np(gK[r, g]).view(np.uint16), rK)
            assert np.array_equal(_np(gV[r, g]).view(np.uint16), rV)
            assert np.array_equal(_np(slots[r, g]), rs)
            assert int(misses[r, g]) == rm


# ----------------------------------------------------------------------------- a5 attention

@pytest.mark.parametrize("H", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("k", [1, 64, 100, 2048])
@pytest.mark.parametrize("qdt", [torch.float32, torch.bfloat16])
def test_attention_within_tolerance(kvs, H, k, qdt):
    R, G = 2, 3
    K, V, _ = synth.fathom_kv(R, G, D, k, seed=H + k)
    q = synth.queries(R, G, H, D, seed=H + k, dtype=qdt)
    k_eff = torch.tensor([[k, max(1, k // 2), 0], [k, 1, k]], dtype=torch.int32)
    out, lse = kvs.sparse_decode_attn(q.to(DEV), K.to(DEV), V.to(DEV), k_eff.to(DEV))
    torch.cuda.synchronize()
    out, lse = _np(out), _np(lse)
    for r in range(R):
        for g in range(G):
            ke = int(k_eff[r, g])
            ro, rl = oracle.attention(q[r, g].float(), K[r, g], V[r, g], ke, 1 / math.sqrt(D))
            assert np.max(np.abs(out[r, g] - ro)) < ATTN_TOL
            if ke:
                assert np.max(np.abs(lse[r, g] - rl)) < 1e-3
            else:
                assert np.all(np.isneginf(lse[r, g])) and not out[r, g].any()


# ----------------------------------------------------------------------------- a6 decode step

def _decode_case(kvs, R, G, H, nl, n_max, B, k, S, seed, rows=None):
    K, V, _ = synth.fathom_kv(R, G, D, nl, n_max=n_max, seed=seed)
    q = synth.queries(R, G, H, D, seed=seed)
    W = kvs.plane_words(n_max)
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, W)
    scale = 1 / math.sqrt(D)
    ref0 = oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, k, None, None, None, K, V, scale,
                               rows=rows)
    slot_map, hot_tok = synth.slot_map_from_selection(ref0["idx"], nl, n_max, S, 0.2, seed=seed)
    hotK, hotV = synth.hot_rows(K, hot_tok), synth.hot_rows(V, hot_tok)
    ref = oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, k, slot_map, hotK, hotV, K, V,
                              scale, rows=rows, want_scores=True)
    ref.update(q=q, K=K, V=V, slot_map=slot_map, hotK=hotK, hotV=hotV, scale=scale)
    ix = kvs.build_fathom_index(K.to(DEV), nl, W)
    step = kvs.DecodeStep(ix, nl, n_max, H, B, k, K.to(DEV), V.to(DEV),
                          torch.from_numpy(slot_map).to(DEV), hotK.to(DEV), hotV.to(DEV))
    step(q.to(DEV))
    torch.cuda.synchronize()
    return ref, step


def _check_decode(ref, step, R, G, nl, k, rows=None, max_diff_frac=1e-3):
    """Every listed row: allocation bit-exact, selection equal to the oracle's
    or differing only inside the tie band, and slots, misses and attention
    against the oracle's gather and attention over the GPU's own selection
    (rows whose selection differs are checked too). Returns the number of
    differing selected entries, which is printed and bounded."""
    t, idx, slots, misses = _np(step.plan.t), _np(step.idx), _np(step.slots), _np(step.misses)
    out, lse = _np(step.out), _np(step.lse)
    rows = range(R * G) if rows is None else rows
    diffs = diff_rows = entries = 0
    for u in rows:
        r, g = divmod(u, G)
        ke = min(k, nl[r])
        assert np.array_equal(t[r, g], ref["t"][r, g])
        d = check_selection(idx[r, g], ref["idx"][r, g], ref["scores"][r, g, : nl[r]], ke)
        diffs += d
        diff_rows += d > 0
        entries += ke
        if d == 0:
            assert np.array_equal(slots[r, g], ref["slots"][r, g])
            assert misses[r, g] == ref["misses"][r, g]
        check_row_over_selection(idx[r, g], slots[r, g], misses[r, g], out[r, g], lse[r, g],
                                 ref["q"][r, g], ref["K"][r, g], ref["V"][r, g],
                                 ref["slot_map"][r, g], ref["hotK"][r, g], ref["hotV"][r, g], ke,
                                 ref["scale"])
    print(f"selection: {diff_rows} of {len(rows)} rows differ from the oracle inside the tie band "
          f"({diffs} of {entries} entries)")
    assert diffs <= max(2, max_diff_frac * entries)
    return diffs


def test_decode_step_tiny_config(kvs):
    """1 request, 1 KV head of 4 query heads, 4096 keys, B = 92, top-256, 512 slots at 80% hits."""
    ref, step = _decode_case(kvs, 1, 1, 4, [4096], 4096, 92, 256, 512, seed=0)
    assert _check_decode(ref, step, 1, 1, [4096], 256) == 0
    assert int(step.misses[0, 0]) == round(0.2 * 256)


@pytest.mark.parametrize("B", [1, 20, 68, 92, 136, 512])
def test_decode_step_ragged_batch(kvs, B):
    nl = [20000, 7777, 2048, 1000]
    ref, step = _decode_case(kvs, 4, 2, 4, nl, 20000, B, 2048, 4096, seed=B)
    _check_decode(ref, step, 4, 2, nl, 2048)


def test_decode_step_layer_sharing_reuses_selection(kvs):
    """idx_in: the second layer of a group reads the first layer's selection
    ("MiniMax-M3: share the sparse index top-k across layers", description).
    Layer 1 selects; layer 2 has its own queries, K/V caches and hot buffers
    (built around that selection at 20% misses) and attends over the same
    selection. Layer 2's slots, misses and attention are checked against the
    oracle's gather and attention over layer 1's selection in layer 2's
    caches; the selection buffer is not written by the reusing call."""
    R, G, H, n_max, k, S = 2, 2, 4, 6000, 512, 1024
    nl = [6000, 5000]
    ref, step = _decode_case(kvs, R, G, H, nl, n_max, 92, k, S, seed=3)
    _check_decode(ref, step, R, G, nl, k)
    idx1 = step.idx.clone()
    K2, V2, _ = synth.fathom_kv(R, G, D, nl, n_max=n_max, seed=3, layer=1)
    q2 = synth.queries(R, G, H, D, seed=3, layer=1)
    sel = idx1.cpu().numpy()
    slot_map2, hot_tok2 = synth.slot_map_from_selection(sel, nl, n_max, S, 0.2, seed=4)
    hotK2, hotV2 = synth.hot_rows(K2, hot_tok2), synth.hot_rows(V2, hot_tok2)
    ix2 = kvs.build_fathom_index(K2.to(DEV), nl)  # not read when a selection is given
    step2 = kvs.DecodeStep(ix2, nl, n_max, H, 92, k, K2.to(DEV), V2.to(DEV),
                           torch.from_numpy(slot_map2).to(DEV), hotK2.to(DEV), hotV2.to(DEV))
    step2.idx.fill_(-7)
    step2(q2.to(DEV), idx_in=idx1)
    torch.cuda.synchronize()
    assert torch.all(step2.idx == -7)  # not written when a selection is given
    for r in range(R):
        for g in range(G):
            ke = min(k, nl[r])
            check_row_over_selection(sel[r, g], _np(step2.slots)[r, g], _np(step2.misses)[r, g],
                                     _np(step2.out)[r, g], _np(step2.lse)[r, g], q2[r, g],
                                     K2[r, g], V2[r, g], slot_map2[r, g], hotK2[r, g],
                                     hotV2[r, g], ke, 1 / math.sqrt(D))
            assert int(step2.misses[r, g]) == round(0.2 * ke)


def test_decode_step_all_scores_tied_takes_first_indices(kvs):
    """Degenerate keys: every key of a row equal -> zero quantiser step, all
    codes 0, every score equal -> the top-k is the first k indices."""
    R, G, H, n, k, S = 2, 2, 4, 9000, 2048, 4096
    K = torch.full((R, G, n, D), 0.5, dtype=torch.bfloat16)
    V = synth.fathom_kv(R, G, D, n, seed=31)[1]
    q = synth.queries(R, G, H, D, seed=31)
    ix = kvs.build_fathom_index(K.to(DEV), [n, n])
    step = kvs.DecodeStep(ix, [n, n], n, H, 92, k, K.to(DEV), V.to(DEV))
    step(q.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(step.idx.cpu(), torch.arange(k, dtype=torch.int32).expand(R, G, k))
    assert torch.all(step.misses == k)


def test_decode_step_all_tied_long_rows_cut_to_first_indices(kvs):
    """All scores equal on rows long enough that a scan block holds more than
    four 4096-key chunks of one row: its candidate buffer fills, is cut to the
    k best by (score, index), and later ties must lose to the held ones; the
    top-k is still the first k indices of every row."""
    R, G, H, n, k = 4, 2, 4, 327680, 2048
    K = torch.full((R, G, n, D), -1.25, dtype=torch.bfloat16)
    V = torch.zeros((R, G, n, D), dtype=torch.bfloat16)
    q = synth.queries(R, G, H, D, seed=32)
    ix = kvs.build_fathom_index(K.to(DEV), [n] * R)
    step = kvs.DecodeStep(ix, [n] * R, n, H, 92, k, K.to(DEV), V.to(DEV))
    step(q.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(step.idx.cpu(), torch.arange(k, dtype=torch.int32).expand(R, G, k))


@pytest.mark.parametrize("B", [20, 92, 136])
def test_decode_step_selection_is_exact_topk_of_its_scores(kvs, B):
    """On ordinary rows (ragged: 100,000 and 131,072 keys) the step's top-k is
    exactly the k largest of the same scan's scores, ties to the lower index."""
    R, G, H, n, k = 2, 4, 4, 131072, 2048
    nl = [100000, n]
    K, V, _ = synth.fathom_kv(R, G, D, nl, n_max=n, seed=81 + B)
    q = synth.queries(R, G, H, D, seed=81 + B)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    step = kvs.DecodeStep(ix, nl, n, H, B, k, K.to(DEV), V.to(DEV))
    step(q.to(DEV))
    sc = kvs.index_scan_fathom(ix, step.plan, nl, n)
    torch.cuda.synchronize()
    order = torch.sort(sc.cpu(), dim=2, descending=True, stable=True).indices[:, :, :k]
    expect = torch.sort(order, dim=2).values.to(torch.int32)
    assert torch.equal(step.idx.cpu(), expect)


def test_decode_step_high_block_overflows_warp_lists(kvs):
    """The first 8,192 keys of each row are one key far above the rest: their
    512 groups are all candidates, and the warps given them collect about
    1,024 keys each (more than a warp's on-chip list holds) while the number of
    candidate groups still fits on chip, so the row is selected over global
    memory. The scores of those keys agree up to the scan's summation order;
    the selection must be exactly the top-2048 of the same scores (score desc,
    index asc), all inside the block."""
    R, G, H, n, k, blk, B = 1, 2, 4, 131072, 2048, 8192, 92
    K, V, nl = synth.fathom_kv(R, G, D, n, seed=71)
    q = synth.queries(R, G, H, D, seed=71)
    s = synth.channel_scales(71, 0, G, D)
    for g in range(G):
        K[0, g, :blk] = (3.0 * s[g] * torch.sign(q[0, g].sum(0))).to(torch.bfloat16)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    step = kvs.DecodeStep(ix, nl, n, H, B, k, K.to(DEV), V.to(DEV))
    step(q.to(DEV))
    sc = kvs.index_scan_fathom(ix, step.plan, nl, n)
    torch.cuda.synchronize()
    order = torch.sort(sc.cpu(), dim=2, descending=True, stable=True).indices[:, :, :k]
    expect = torch.sort(order, dim=2).values.to(torch.int32)
    assert torch.equal(step.idx.cpu(), expect)
    assert int(step.idx.max()) < blk


@pytest.mark.parametrize("B", [68, 92])
def test_host_mapped_index_scan_and_decode(kvs, B):
    """The index planes in mapped pinned host memory, read over the host link
    by the same call: scores within the f32 bound of the oracle, and the same
    selection as the oracle (up to ties inside the band)."""
    R, G, n = 2, 2, 20000
    K, V, nl = synth.fathom_kv(R, G, D, n, seed=61)
    q = synth.queries(R, G, 4, D, seed=61)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    hix = kvs.MappedHostIndex(ix)
    plan = kvs.fathom_plan_bits(q.to(DEV), hix, B)
    sc = kvs.index_scan_fathom(hix, plan, nl, n).cpu().numpy()
    step = kvs.DecodeStep(hix, nl, n, 4, B, 512, K.to(DEV), V.to(DEV))
    step(q.to(DEV))
    torch.cuda.synchronize()
    planes, kmin, kstep, kvar = oracle.build_index_batch(K, nl, kvs.plane_words(n))
    ref = oracle.decode_batch(q, planes, kmin, kstep, kvar, nl, B, 512, None, None, None, K, V,
                              1 / math.sqrt(D), want_scores=True)
    for r in range(R):
        for g in range(G):
            t, qbar = oracle.plan_bits(q[r, g], kvar[r, g], B)
            tol = fathom_score_tol(qbar, kmin[r, g], kstep[r, g], B)
            assert np.max(np.abs(sc[r, g] - ref["scores"][r, g])) <= tol
            gi = step.idx[r, g].cpu().numpy()
            check_selection(gi, ref["idx"][r, g], ref["scores"][r, g], 512)
            # no hot buffer: every selected row is read from the full store
            check_row_over_selection(gi, None, _np(step.misses)[r, g], _np(step.out)[r, g],
                                     _np(step.lse)[r, g], q[r, g], K[r, g], V[r, g], None, None,
                                     None, min(512, nl[r]), 1 / math.sqrt(D))


def test_decode_step_timed_matches_and_records_stages(kvs):
    """decode_step_timed gives the same results as decode_step and records its
    five stage events in order on the stream."""
    R, G, n, B, k = 2, 4, 30000, 92, 512
    K, V, nl = synth.fathom_kv(R, G, D, n, seed=71)
    q = synth.queries(R, G, 4, D, seed=71).to(DEV)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    step = kvs.DecodeStep(ix, nl, n, 4, B, k, K.to(DEV), V.to(DEV))
    step(q)
    torch.cuda.synchronize()
    out0, idx0 = step.out.clone(), step.idx.clone()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(step.DECODE_STAGES) + 1)]
    step.timed(q, ev)
    torch.cuda.synchronize()
    assert torch.equal(step.out, out0) and torch.equal(step.idx, idx0)
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(step.DECODE_STAGES))]
    assert all(t >= 0 for t in times) and times[1] > 0 and times[3] > 0
    with pytest.raises(ValueError):
        step.timed(q, ev[:3])


# ----------------------------------------------------------------------------- write-back

def test_append_token_matches_the_oracle(kvs):
    """kvs_append_token against the oracle's append, row by row: two tokens
    appended in turn to ragged rows (the second request starts one short of
    n_max, so its second append is refused with KVS_EBOUNDS and leaves the row
    as it was), with a hot slot for some rows (the previous occupant evicted)
    and none for the others."""
    R, G, S, n_max = 3, 2, 16, 5000
    nl = [3000, n_max - 1, 1]
    K, V, _ = synth.fathom_kv(R, G, D, nl, n_max=n_max, seed=51)
    Knew, Vnew, _ = synth.fathom_kv(R, G, D, 2, seed=52)
    W = kvs.plane_words(n_max)
    ix = kvs.build_fathom_index(K.to(DEV), nl, W)
    rng = np.random.default_rng(51)
    slot_map = np.full((R, G, n_max), -1, np.int32)
    hot_tok = np.full((R, G, S), -1, np.int32)
    for r in range(R):
        for g in range(G):
            toks = rng.choice(nl[r], min(S // 2, nl[r]), replace=False)
            hot_tok[r, g, : toks.size] = toks
            slot_map[r, g, toks] = np.arange(toks.size)
    hotK, hotV = synth.hot_rows(K, hot_tok), synth.hot_rows(V, hot_tok)
    hot_slot = np.array([[2, -1], [15, 0], [-1, 1]], np.int32)
    dK, dV = K.clone().to(DEV), V.clone().to(DEV)
    d_sm, d_ht = torch.from_numpy(slot_map).to(DEV), torch.from_numpy(hot_tok).to(DEV)
    d_hK, d_hV = hotK.clone().to(DEV), hotV.clone().to(DEV)
    n = torch.tensor(nl, dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    ref = dict(planes=_np(ix.planes).view(np.uint32).copy(), K=_np(K).view(np.uint16).copy(),
               V=_np(V).view(np.uint16).copy(), sm=slot_map.copy(), ht=hot_tok.copy(),
               hK=_np(hotK).view(np.uint16).copy(), hV=_np(hotV).view(np.uint16).copy())
    kmin, kstep = _np(ix.kmin), _np(ix.kstep)
    pos = list(nl)
    for step in range(2):
        kvs.append_token(ix, Knew[:, :, step].to(DEV), Vnew[:, :, step].to(DEV), n, dK, dV, d_sm,
                         torch.from_numpy(hot_slot).to(DEV), d_ht, d_hK, d_hV, dev_status=st)
        torch.cuda.synchronize()
        for r in range(R):
            if pos[r] >= n_max:
                continue
            for g in range(G):
                out = oracle.append_token(Knew[r, g, step], Vnew[r, g, step], pos[r], ref["planes"][r, g],
                                          kmin[r, g], kstep[r, g], ref["K"][r, g], ref["V"][r, g],
                                          ref["sm"][r, g], int(hot_slot[r, g]), ref["ht"][r, g],
                                          ref["hK"][r, g], ref["hV"][r, g])
                for key, val in zip(["planes", "K", "V", "sm", "ht", "hK", "hV"], out):
                    ref[key][r, g] = val
            pos[r] += 1
    assert int(st.item()) == kvs.KVS_EBOUNDS  # request 1 was full at the second step
    assert n.cpu().tolist() == pos == [nl[0] + 2, n_max, 3]
    assert np.array_equal(_np(ix.planes).view(np.uint32), ref["planes"])
    assert np.array_equal(_np(dK).view(np.uint16), ref["K"]) and np.array_equal(_np(dV).view(np.uint16), ref["V"])
    assert np.array_equal(_np(d_sm), ref["sm"]) and np.array_equal(_np(d_ht), ref["ht"])
    assert np.array_equal(_np(d_hK).view(np.uint16), ref["hK"])
    assert np.array_equal(_np(d_hV).view(np.uint16), ref["hV"])


# ----------------------------------------------------------------------------- failure detection

def test_scan_bounded_wait_runs_out_and_the_context_stays_usable(kvs):
    """A producer warp of every block of the HBM scan withholds its arrival on
    its first chunk (kvs_selftest_scan_timeout), with every wait bounded by
    2e6 cycles: the consumers' wait runs out, KVS_ETIMEOUT reaches the status
    word, the kernel returns within milliseconds, and the next decode step on
    the same context is exact."""
    import time
    R, G, H, n, B, k = 2, 4, 4, 70000, 92, 2048
    K, V, nl = synth.fathom_kv(R, G, D, n, seed=61)
    q = synth.queries(R, G, H, D, seed=61).to(DEV)
    ix = kvs.build_fathom_index(K.to(DEV), nl)
    plan = kvs.fathom_plan_bits(q, ix, B)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    kvs.selftest_scan_timeout(ix, plan, nl, n, 2_000_000, st)
    torch.cuda.synchronize()
    assert int(st.item()) == kvs.KVS_ETIMEOUT
    assert time.perf_counter() - t0 < 5.0
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    step = kvs.DecodeStep(ix, nl, n, H, B, k, K.to(DEV), V.to(DEV))
    step(q, dev_status=st2)
    sc = kvs.index_scan_fathom(ix, step.plan, nl, n, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == kvs.KVS_OK
    order = torch.sort(sc.cpu(), dim=2, descending=True, stable=True).indices[:, :, :k]
    assert torch.equal(step.idx.cpu(), torch.sort(order, dim=2).values.to(torch.int32))


# ----------------------------------------------------------------------------- host tier

@pytest.mark.parametrize("miss", [0.2, 0.4, 1.0])
def test_full_store_in_host_memory_equals_the_hbm_step(kvs, miss):
    """The full K/V store in mapped pinned host memory: the step fetches only
    the missing selected rows over the host link into HBM before the
    attention. Its outputs equal those of the same step with the store in HBM,
    bit for bit, at 20% and 40% misses and with no hot buffer at all (every
    selected row a miss); a second layer reusing the selection (idx_in) too."""
    R, G, H, n, B, k, S = 2, 4, 4, 30000, 92, 512, 1024
    K, V, nl = synth.fathom_kv(R, G, D, [n, 21000], n_max=n, seed=71)
    q = synth.queries(R, G, H, D, seed=71).to(DEV)
    Kd, Vd = K.to(DEV), V.to(DEV)
    ix = kvs.build_fathom_index(Kd, nl)
    if miss < 1.0:
        warm = kvs.DecodeStep(ix, nl, n, H, B, k, Kd, Vd)
        warm(q)
        torch.cuda.synchronize()
        slot_map, hot_tok = synth.slot_map_from_selection(warm.idx.cpu().numpy(), nl, n, S, miss, seed=72)
        sm, hK, hV = (torch.from_numpy(slot_map).to(DEV), synth.hot_rows(Kd, hot_tok),
                      synth.hot_rows(Vd, hot_tok))
    else:
        sm = hK = hV = None
    ref = kvs.DecodeStep(ix, nl, n, H, B, k, Kd, Vd, sm, hK, hV)
    hostK, hostV = kvs.MappedHostStore(Kd), kvs.MappedHostStore(Vd)
    step = kvs.DecodeStep(ix, nl, n, H, B, k, hostK, hostV, sm, hK, hV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    ref(q)
    step(q, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for name in ("out", "lse", "idx", "slots", "misses"):
        assert torch.equal(getattr(step, name), getattr(ref, name)), name
    expect = round(miss * k) if miss < 1.0 else k
    assert torch.all(step.misses == expect)
    # a second layer of a group reusing the selection, store in host memory
    q2 = synth.queries(R, G, H, D, seed=73).to(DEV)
    o_ref = ref(q2, idx_in=ref.idx).clone()
    o_host = step(q2, idx_in=ref.idx)
    torch.cuda.synchronize()
    assert torch.equal(o_host, o_ref)
