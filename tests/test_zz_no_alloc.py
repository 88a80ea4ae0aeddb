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


def test_noalloc_rejects_sizes_beyond_its_array(kvs):
    H, k, G = 8, 2048, 4
    sizes = [R for R in range(1, 400)
             if kvs._lib.kvs_attn_workspace_size(R, G, H, k) > 4 << 20]
    if not sizes:
        pytest.skip("no size needs more than the fixed array on this GPU")
    R = sizes[0]
    q = torch.zeros(R, G, H, D, device="cuda")
    K = torch.zeros(R, G, 8, D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(R, G, H, D, device="cuda")
    st = kvs._lib.sparse_decode_attn_noalloc(q.data_ptr(), 0, K.data_ptr(), K.data_ptr(), None, R,
                                             G, H, D, k, 0.1, out.data_ptr(), None, None,
                                             torch.cuda.current_stream().cuda_stream)
    assert st == kvs.KVS_EINVAL
    assert b"fixed" in kvs._lib.kvs_last_error()
