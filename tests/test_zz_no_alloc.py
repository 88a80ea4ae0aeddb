"""sparse_decode_attn_noalloc through the C ABI, against sparse_decode_attn.

The no-allocation variant serves callers that cannot call cudaMalloc (inside a
stream capture, or runtimes that only lend the library their input and output
buffers): its split-K scratch is a fixed device array inside the library. This
file is collected last so that a run stopping at the first failure has already
run every other test; it must pass alone in a fresh process too.
"""
import math

import numpy as np
import pytest
import torch

import synth
from tests._parity import ATTN_TOL

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module")
def kvs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_index_scan_b200
    return kv_index_scan_b200


def _case(seed, R, G, H, k, qdt):
    K, V, _ = synth.fathom_kv(R, G, D, k, seed=seed, device="cuda")
    q = synth.queries(R, G, H, D, seed=seed, device="cuda", dtype=qdt)
    k_eff = torch.randint(0, k + 1, (R, G), generator=torch.Generator().manual_seed(seed),
                          dtype=torch.int32).cuda()
    k_eff[0, 0] = k
    return q, K, V, k_eff


def test_noalloc_matches_workspace_attention_on_two_calls_in_a_row(kvs):
    cases = [(11, 16, 8, 4, 2048, torch.float32), (12, 3, 5, 8, 700, torch.bfloat16)]
    outs = []
    for seed, R, G, H, k, qdt in cases:
        q, K, V, k_eff = _case(seed, R, G, H, k, qdt)
        need = kvs._lib.kvs_attn_workspace_size(R, G, H, k)
        assert 0 < need <= 4 << 20  # these sizes use the split-K scratch
        out = torch.empty(R, G, H, D, dtype=torch.float32, device="cuda")
        lse = torch.empty(R, G, H, dtype=torch.float32, device="cuda")
        kvs.sparse_decode_attn_noalloc(q, K, V, out, lse, k_eff=k_eff)
        ref_out, ref_lse = kvs.sparse_decode_attn(q, K, V, k_eff=k_eff)
        torch.cuda.synchronize()
        assert float((out - ref_out).abs().max()) < ATTN_TOL
        fin = torch.isfinite(ref_lse)
        assert torch.equal(fin, torch.isfinite(lse))
        assert float((lse[fin] - ref_lse[fin]).abs().max()) < 1e-3
        outs.append(out)


def test_noalloc_sizes_beyond_the_workspace_split_run_with_fewer_splits(kvs):
    """At H = 4, k = 2048 the workspace attention cuts the rows of 593 and 2073
    (request, KV head) pairs into splits whose partial results need more than
    the fixed 4 MiB array (7.2 and 8.8 MiB on a 148-SM B200). The no-allocation
    call runs them with fewer splits, and matches, twice in a row."""
    H, k, G = 4, 2048, 1
    for RG in (593, 2073):
        assert kvs._lib.kvs_attn_workspace_size(RG, G, H, k) > 4 << 20
        q, K, V, k_eff = _case(RG, RG, G, H, k, torch.float32)
        ref_out, ref_lse = kvs.sparse_decode_attn(q, K, V, k_eff=k_eff)
        for _ in range(2):
            out = torch.full((RG, G, H, D), float("nan"), device="cuda")
            lse = torch.full((RG, G, H), float("nan"), device="cuda")
            kvs.sparse_decode_attn_noalloc(q, K, V, out, lse, k_eff=k_eff)
            torch.cuda.synchronize()
            assert float((out - ref_out).abs().max()) < ATTN_TOL
            fin = torch.isfinite(ref_lse)
            assert torch.equal(fin, torch.isfinite(lse))
            assert float((lse[fin] - ref_lse[fin]).abs().max()) < 1e-3


def test_noalloc_checks_caller_outputs(kvs):
    """The binding refuses output buffers that the kernels would overrun."""
    q, K, V, k_eff = _case(13, 2, 3, 4, 64, torch.float32)
    bad = [torch.empty(2, 3, 4, D, dtype=torch.bfloat16, device="cuda"),
           torch.empty(2, 3, 4, D + 1, device="cuda")[..., :D],
           torch.empty(2, 3, 3, D, device="cuda")]
    for out in bad:
        with pytest.raises(ValueError):
            kvs.sparse_decode_attn_noalloc(q, K, V, out)
    out = torch.empty(2, 3, 4, D, device="cuda")
    with pytest.raises(ValueError):
        kvs.sparse_decode_attn_noalloc(q, K, V, out, torch.empty(2, 3, 5, device="cuda"))
    with pytest.raises(ValueError):
        kvs.sparse_decode_attn_noalloc(q, K, V, out, k_eff=k_eff.long())
