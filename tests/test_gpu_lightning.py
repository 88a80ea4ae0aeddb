"""GPU parity of the lightning-indexer variant (tcgen05 tensor cores) against
the CPU oracle, through the C ABI: block scores within 1e-4 * max|S| of the
fp64 scores, block selections equal up to ties inside that band, and the
selection reused by every KV head and by the second layer of a group."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests._parity import ATTN_TOL

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_index_scan_b200
    return kv_index_scan_b200


@pytest.mark.parametrize("block", [1, 32, 64, 128])
@pytest.mark.parametrize("Hi", [64, 16, 128, 48, 96])
def test_lightning_scores_within_tolerance(kvs, block, Hi):
    nl = [5000, 1000, 129, 0]
    n_max = 5000
    R = len(nl)
    kidx, qidx, w, _ = synth.lightning_inputs(R, nl, Hi=Hi, n_max=n_max, seed=block + Hi)
    bs = kvs.index_scan_lightning(kidx.to(DEV), qidx.to(DEV), w.to(DEV), nl, block=block)
    torch.cuda.synchronize()
    bs = bs.cpu().numpy()
    nb = (n_max + block - 1) // block
    for r in range(R):
        s = oracle.lightning_scores(kidx[r, : nl[r]], qidx[r], w[r])
        ref = oracle.block_max(s, block) if block > 1 else s
        nbr = (nl[r] + block - 1) // block
        if nbr:
            tol = 1e-4 * max(1e-30, float(np.max(np.abs(ref))))
            assert np.max(np.abs(bs[r, :nbr] - ref)) <= tol, (r, np.max(np.abs(bs[r, :nbr] - ref)), tol)
        assert np.all(np.isneginf(bs[r, nbr:nb]))


def test_lightning_one_hot_weights_single_head(kvs):
    R, n, Hi = 1, 777, 64
    kidx, qidx, w, nl = synth.lightning_inputs(R, n, Hi=Hi, seed=9)
    for h in [0, 17, 63]:
        wh = torch.zeros(R, Hi)
        wh[0, h] = 1.0
        s = kvs.index_scan_lightning(kidx.to(DEV), qidx.to(DEV), wh.to(DEV), nl, block=1)
        ref = oracle.lightning_scores(kidx[0], qidx[0], wh[0])
        assert np.max(np.abs(s.cpu().numpy()[0] - ref)) <= 1e-5 * max(1e-30, np.max(np.abs(ref)))


def test_lightning_layer_pair_block_topk_and_shared_attention(kvs):
    """Scores -> top-32 of 64-token blocks -> attention of every KV head over the
    one selection, run for two layers of a group with the same idx."""
    R, n, Hi, G, H, k, block = 4, 8000, 64, 8, 4, 2048, 64
    kidx, qidx, w, nl = synth.lightning_inputs(R, n, Hi=Hi, seed=3)
    bs = kvs.index_scan_lightning(kidx.to(DEV), qidx.to(DEV), w.to(DEV), nl, block=block)
    idx = kvs.topk_select(bs, nl, k, block=block)  # [R][k], one selection per request
    torch.cuda.synchronize()
    ref_bs, ref_idx = oracle.lightning_batch(kidx, qidx, w, nl, block, k)
    nb = (n + block - 1) // block
    for r in range(R):
        g_blocks = np.unique(idx.cpu().numpy()[r] // block)
        o_blocks = np.unique(ref_idx[r] // block)
        if not np.array_equal(g_blocks, o_blocks):  # only ties inside the band may differ
            s = ref_bs[r, :nb]
            kth = np.sort(s[o_blocks])[0]
            tol = 1e-4 * np.max(np.abs(s))
            assert np.all(s[np.setdiff1d(g_blocks, o_blocks)] >= kth - tol)
            assert np.all(s[np.setdiff1d(o_blocks, g_blocks)] <= kth + tol)
    # attention for two layers of the group, each reading the same selection
    scale = 1 / math.sqrt(D)
    for layer in range(2):
        K, V, _ = synth.fathom_kv(R, G, D, n, seed=40 + layer)
        q = synth.queries(R, G, H, D, seed=40 + layer, dtype=torch.bfloat16)
        ix = kvs.build_fathom_index(K.to(DEV), nl)  # the index is not read when idx_in is given
        step = kvs.DecodeStep(ix, nl, n, H, 92, k, K.to(DEV), V.to(DEV), q_dtype=torch.bfloat16)
        step(q.to(DEV), idx_in=idx, idx_shared=True)
        torch.cuda.synchronize()
        out_ref, lse_ref = oracle.shared_attention_batch(q.float(), K, V, idx.cpu().numpy(), scale)
        assert np.max(np.abs(step.out.cpu().numpy() - out_ref)) < ATTN_TOL
        assert np.all(step.misses.cpu().numpy() == k)


def _check_block_selection(g_idx, o_idx, s_blocks, block):
    """The GPU's block selection equals the oracle's, or differs only on blocks
    whose oracle score lies within 1e-4 max|S| of the oracle's last selected
    block. Returns the number of differing blocks."""
    g_blocks = np.unique(g_idx[g_idx >= 0] // block)
    o_blocks = np.unique(o_idx[o_idx >= 0] // block)
    assert g_blocks.size == o_blocks.size
    if np.array_equal(g_blocks, o_blocks):
        return 0
    kth = np.min(s_blocks[o_blocks])
    tol = 1e-4 * np.max(np.abs(s_blocks[np.isfinite(s_blocks)]))
    extra, missing = np.setdiff1d(g_blocks, o_blocks), np.setdiff1d(o_blocks, g_blocks)
    assert np.all(s_blocks[extra] >= kth - tol)
    assert np.all(s_blocks[missing] <= kth + tol)
    return int(extra.size)


def _lightning_vs_oracle(kvs, R, nl, n_max, Hi, block, k, reqs, seed):
    kidx, qidx, w, _ = synth.lightning_inputs(R, nl, Hi=Hi, n_max=n_max, seed=seed, device=DEV)
    bs = kvs.index_scan_lightning(kidx, qidx, w, nl, block=block)
    idx = kvs.topk_select(bs, nl, k, block=block)
    torch.cuda.synchronize()
    bs, idx = bs.cpu().numpy(), idx.cpu().numpy()
    sub = torch.tensor(reqs, dtype=torch.long, device=DEV)
    ref_bs, ref_idx = oracle.lightning_batch(kidx[sub].cpu(), qidx[sub].cpu(), w[sub].cpu(),
                                             [nl[r] for r in reqs], block, k)
    diffs = 0
    for j, r in enumerate(reqs):
        nbr = (nl[r] + block - 1) // block
        if nbr:
            ref = ref_bs[j, :nbr]
            tol = 1e-4 * max(1e-30, float(np.max(np.abs(ref))))
            err = float(np.max(np.abs(bs[r, :nbr] - ref)))
            assert err <= tol, (r, err, tol)
        assert np.all(np.isneginf(bs[r, nbr:]))
        diffs += _check_block_selection(idx[r], ref_idx[j], ref_bs[j, :nbr], block)
    print(f"block selection: {diffs} blocks differ from the oracle inside the tie band over "
          f"{len(reqs)} requests")
    return diffs


def test_lightning_full_size_sampled_requests(kvs):
    """The lightning layer at its full size (32 requests x 80000 tokens, 64
    index heads, 64-token blocks, top-2048 tokens): every block of the kernel's
    grid runs about 135 tiles, so its raw-tile and accumulator rings wrap many
    times. Four sampled requests (the last one included) against the oracle."""
    R, n = 32, 80000
    _lightning_vs_oracle(kvs, R, [n] * R, n, 64, 64, 2048, reqs=[0, 9, 22, 31], seed=5)


def test_lightning_many_short_requests_cross_boundaries(kvs):
    """600 requests of at most 384 tokens (ragged, some empty): about 12 tiles
    per block of the grid, each block crossing three or more request
    boundaries, so the query buffers, head-weight slots and rings all rotate.
    Every request against the oracle."""
    R, n_max = 600, 384
    rng = np.random.default_rng(11)
    nl = [int(x) for x in rng.integers(1, n_max + 1, size=R)]
    nl[0], nl[17], nl[599], nl[300] = n_max, 0, n_max, 1
    _lightning_vs_oracle(kvs, R, nl, n_max, 64, 64, 128, reqs=list(range(R)), seed=6)
