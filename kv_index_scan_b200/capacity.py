"""Decode throughput and capacity model of the offloaded sparse-attention
system, fed with measured decode-step times ("XM-Sparse: Pushing the
Throughput Frontier of Sparse Attention with Netpreme X-Mem", the
modelled-throughput section and Figures 2-3).

The page states the model in words; its equations were not preserved. The
plain reading used here:

  * The full KV cache of every request lives in external memory (host DRAM,
    CXL, a scale-up memory node); HBM holds, per request, the hot KV buffer
    and the K-index.
  * One decode step of a batch takes the measured compute time plus the time
    to fetch the missing selected KV entries over the link, with no overlap:
        T_step(b) = T_compute(b) + b * layers * k * miss_rate * entry_bytes / BW
  * The batch is capped by both memories, per GPU:
        b_max = min(floor(HBM budget / HBM bytes per request),
                    floor(external capacity / full KV bytes per request))
  * Throughput is b / T_step(b) output tokens per second per GPU.

Host-side arithmetic only; nothing here runs on the GPU.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class Footprint:
    """Per-request memory of a model: bytes as a + b * context length."""
    hbm_fixed: float        # hot KV buffers (all layers)
    hbm_per_token: float    # K-index (all layers)
    full_per_token: float   # the full KV cache (all layers)
    layers: int
    entry_bytes: float      # bytes of one selected KV entry of one layer

    def hbm_bytes(self, n: int) -> float:
        return self.hbm_fixed + self.hbm_per_token * n

    def full_bytes(self, n: int) -> float:
        return self.full_per_token * n


def qwen3_8b_like(k_bits: int = 4, hot_slots: int = 4096, layers: int = 36, kv_heads: int = 8,
                  head_dim: int = 128) -> Footprint:
    """The decode layer this library runs: bf16 K and V of kv_heads x head_dim
    per token and layer; the 4-bit bit-plane K-index; a hot buffer of
    hot_slots entries per (request, layer, KV head)."""
    row = 2 * head_dim * 2  # K and V, bf16
    return Footprint(hbm_fixed=layers * kv_heads * hot_slots * row,
                     hbm_per_token=layers * kv_heads * head_dim * k_bits / 8,
                     full_per_token=layers * kv_heads * row, layers=layers,
                     entry_bytes=kv_heads * row)


def batch_max(fp: Footprint, n: int, hbm_budget: float, ext_capacity: float) -> int:
    """The largest batch both memories hold (per GPU)."""
    if n <= 0:
        return 0
    return int(min(math.floor(hbm_budget / fp.hbm_bytes(n)), math.floor(ext_capacity / fp.full_bytes(n))))


def fetch_seconds(fp: Footprint, batch: int, k: int, miss_rate: float, link_bytes_per_s: float) -> float:
    """Time to fetch one step's missing selected entries over the link."""
    return batch * fp.layers * k * miss_rate * fp.entry_bytes / link_bytes_per_s


def step_seconds(t_compute: float, fp: Footprint, batch: int, k: int, miss_rate: float,
                 link_bytes_per_s: float) -> float:
    """Compute plus fetch, not overlapped."""
    return t_compute + fetch_seconds(fp, batch, k, miss_rate, link_bytes_per_s)


def tokens_per_s(t_compute: float, fp: Footprint, batch: int, k: int, miss_rate: float,
                 link_bytes_per_s: float) -> float:
    """Output tokens per second per GPU at this batch (one token per request and step)."""
    return batch / step_seconds(t_compute, fp, batch, k, miss_rate, link_bytes_per_s)


# The link and capacity settings the page models, per GPU of a 4-GPU instance
# (capacities are the instance's budgets divided by 4).
LINKS = {
    "pcie": dict(bandwidth=64e9, capacity=1e12 / 4),
    "cxl": dict(bandwidth=64e9, capacity=24e12 / 4),
    "nvlink_c2c": dict(bandwidth=225e9, capacity=1e12 / 4),
    "scale_up": dict(bandwidth=900e9, capacity=24e12 / 4),
}
HBM_BUDGET = 60 * 2 ** 30  # hot KV buffer + K-index per GPU (the page's allocation)


def glm_footprint_from_page() -> Footprint:
    """The GLM-5.3 footprints the page's own batch limits imply: 1 TB over 4
    GPUs holds batch 36 of 128K-token full caches (full KV per token), and the
    60 GiB HBM budget holds batch 109 at 128K and 20 at 1M (hot buffers plus
    a K-index growing with the context). Derived constants, for checking the
    model against the page's other points."""
    full_per_token = (1e12 / 4) / 36 / 131072
    b128, b1m = HBM_BUDGET / 109, HBM_BUDGET / 20
    per_token = (b1m - b128) / (1048576 - 131072)
    fixed = b128 - per_token * 131072
    return Footprint(hbm_fixed=fixed, hbm_per_token=per_token, full_per_token=full_per_token, layers=1,
                     entry_bytes=0.0)
