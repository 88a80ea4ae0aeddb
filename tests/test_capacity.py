"""The throughput and capacity model ("XM-Sparse: Pushing the Throughput
Frontier of Sparse Attention with Netpreme X-Mem", the modelled-throughput
section, Figures 2-3) against the page's own batch limits, and its basic
invariants. No GPU needed."""
import math

import pytest

from kv_index_scan_b200 import capacity as cm


def test_page_batch_limits_from_the_page_footprints():
    """Footprints fitted to three of the page's batch limits (128K with 1 TB:
    36; 128K and 1M with 24 TB: 109 and 20) reproduce them, and predict the
    other two: 1M with 1 TB (the page: 4) and 16K, where the page reports
    batch 241 per GPU using 0.85 TB of the 1 TB budget."""
    fp = cm.glm_footprint_from_page()
    pcie, cxl = cm.LINKS["pcie"], cm.LINKS["cxl"]
    assert cm.batch_max(fp, 131072, cm.HBM_BUDGET, pcie["capacity"]) == 36
    assert cm.batch_max(fp, 131072, cm.HBM_BUDGET, cxl["capacity"]) == 109
    assert cm.batch_max(fp, 1048576, cm.HBM_BUDGET, cxl["capacity"]) == 20
    assert cm.batch_max(fp, 1048576, cm.HBM_BUDGET, pcie["capacity"]) == 4
    b16 = cm.batch_max(fp, 16384, cm.HBM_BUDGET, pcie["capacity"])
    assert abs(b16 - 241) / 241 < 0.03
    # 241 requests of 16K over 4 GPUs: the page's 0.85 TB of full KV
    assert abs(4 * 241 * fp.full_bytes(16384) / 1e12 - 0.85) < 0.03


def test_step_time_is_compute_plus_fetch():
    fp = cm.qwen3_8b_like()
    t = cm.step_seconds(1e-3, fp, batch=16, k=2048, miss_rate=0.2, link_bytes_per_s=64e9)
    fetch = 16 * 36 * 2048 * 0.2 * (8 * 2 * 128 * 2) / 64e9
    assert math.isclose(t, 1e-3 + fetch, rel_tol=1e-12)
    # more misses or a slower link cost time; a faster link recovers it
    assert cm.step_seconds(1e-3, fp, 16, 2048, 0.4, 64e9) > t
    assert cm.step_seconds(1e-3, fp, 16, 2048, 0.2, 900e9) < t
    assert cm.step_seconds(1e-3, fp, 16, 2048, 0.0, 64e9) == 1e-3


def test_footprint_of_the_decode_layer():
    """4-bit index: 512 bytes per token and layer over 8 KV heads of 128
    channels; bf16 K and V: 4 KB per token and layer; hot buffers of 4096
    entries: 16 MiB per layer."""
    fp = cm.qwen3_8b_like()
    assert fp.hbm_per_token == 36 * 512 and fp.full_per_token == 36 * 4096
    assert fp.hbm_fixed == 36 * 8 * 4096 * 512
    assert fp.entry_bytes == 4096


@pytest.mark.parametrize("n", [16384, 131072, 1048576])
def test_batch_limit_is_the_tighter_memory(n):
    fp = cm.qwen3_8b_like()
    for link in cm.LINKS.values():
        b = cm.batch_max(fp, n, cm.HBM_BUDGET, link["capacity"])
        assert fp.hbm_bytes(n) * b <= cm.HBM_BUDGET and fp.full_bytes(n) * b <= link["capacity"]
        assert fp.hbm_bytes(n) * (b + 1) > cm.HBM_BUDGET or fp.full_bytes(n) * (b + 1) > link["capacity"]
