"""Seeded synthetic inputs shaped like the workloads of the kv_index_scan pages.

This module holds no arithmetic of the method itself. It only draws random
numbers, converts the draws to the storage formats (f32 -> bf16 / e4m3 through
torch's own conversions), and builds a hot-buffer slot map around a selection
it is given. The CUDA path's tests and benchmark and the CPU oracle both take
their inputs from here; neither side's arithmetic lives here.

Shapes follow the pages' workloads: GQA with G KV heads of H query heads each
and head dim D = 128 (Qwen3-8B-like); per-channel key scales s_c drawn
log-normal(0, 0.7) per (layer, KV head, channel) and shared by all requests
(a few outlier channels); K ~ N(0, s_c^2) and V ~ N(0, 1) stored as bf16;
queries N(0, 1) in f32. The lightning-indexer variant stores e4m3 keys drawn
N(0, 1)/sqrt(128), bf16 index queries N(0, 1) and head weights U(0, 1).

Every (request, KV head) row has its own generator, seeded from
(workload seed, layer, r, g, tag), so a row can be drawn alone and the draws
do not depend on the batch shape. Rows past a request's length are zero.
"""
from __future__ import annotations

import math

import numpy as np
import torch

_M64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _M64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def row_seed(*parts: int) -> int:
    """Mix integer parts into one 63-bit seed (SplitMix64 chain)."""
    h = 0x243F6A8885A308D3
    for p in parts:
        h = _splitmix64(h ^ (int(p) & _M64))
    return h & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(row_seed(*parts))
    return g


TAG_SCALE, TAG_K, TAG_V, TAG_Q, TAG_KIDX, TAG_QIDX, TAG_W, TAG_SLOTS, TAG_LEN = range(1, 10)


def channel_scales(seed: int, layer: int, G: int, D: int) -> torch.Tensor:
    """s_c = exp(0.7 * N(0,1)) per (KV head, channel): f32 [G][D] on the CPU."""
    out = torch.empty(G, D, dtype=torch.float32)
    for g in range(G):
        z = torch.randn(D, generator=_gen("cpu", seed, layer, g, TAG_SCALE), dtype=torch.float64)
        out[g] = torch.exp(0.7 * z).to(torch.float32)
    return out


def as_lengths(n, R: int) -> list[int]:
    if isinstance(n, int):
        return [n] * R
    n = [int(x) for x in n]
    assert len(n) == R
    return n


def fathom_kv(R: int, G: int, D: int, n, n_max: int | None = None, seed: int = 0,
              layer: int = 0, device="cpu", with_v: bool = True):
    """K (and V) caches: bf16 [R][G][n_max][D] with K ~ N(0, s_c^2), V ~ N(0, 1).

    Returns (K, V, n_list); V is None when with_v is False.
    """
    n_list = as_lengths(n, R)
    n_max = max(n_list) if n_max is None else n_max
    assert n_max >= max(n_list)
    s = channel_scales(seed, layer, G, D).to(device)
    K = torch.zeros(R, G, n_max, D, dtype=torch.bfloat16, device=device)
    V = torch.zeros(R, G, n_max, D, dtype=torch.bfloat16, device=device) if with_v else None
    for r in range(R):
        nr = n_list[r]
        for g in range(G):
            z = torch.randn(nr, D, generator=_gen(device, seed, layer, r, g, TAG_K),
                            dtype=torch.float32, device=device)
            K[r, g, :nr] = (z * s[g]).to(torch.bfloat16)
            if with_v:
                v = torch.randn(nr, D, generator=_gen(device, seed, layer, r, g, TAG_V),
                                dtype=torch.float32, device=device)
                V[r, g, :nr] = v.to(torch.bfloat16)
    return K, V, n_list


def queries(R: int, G: int, H: int, D: int, seed: int = 0, layer: int = 0, device="cpu",
            dtype=torch.float32) -> torch.Tensor:
    """Decode queries N(0, 1): [R][G][H][D] (f32, or bf16 by conversion)."""
    q = torch.empty(R, G, H, D, dtype=torch.float32, device=device)
    for r in range(R):
        for g in range(G):
            q[r, g] = torch.randn(H, D, generator=_gen(device, seed, layer, r, g, TAG_Q),
                                  dtype=torch.float32, device=device)
    return q.to(dtype)


def ragged_lengths(batch: int, seed: int, lo: int = 16384, hi: int = 131072) -> list[int]:
    """Context lengths floor(exp(U(ln lo, ln hi))), one per request."""
    rng = np.random.default_rng(row_seed(seed, TAG_LEN))
    u = rng.uniform(math.log(lo), math.log(hi), size=batch)
    return [int(math.floor(math.exp(x))) for x in u]


def slot_map_from_selection(sel, n, n_max: int, S: int, miss_frac: float, seed: int):
    """Hot-buffer contents built around a given selection.

    sel: int [R][G][k] token indices (-1 = padding). Of the k_eff selected
    tokens of each row, k_eff - round(miss_frac * k_eff) are placed in the hot
    buffer (chosen uniformly); the other slots hold uniformly drawn tokens that
    were not selected; the slot order is a random permutation. Slots left over
    when a row has too few tokens hold token -1.

    Returns (slot_map int32 [R][G][n_max] with -1 for absent tokens,
             hot_tok int32 [R][G][S], the token held by each slot or -1).
    """
    sel = np.asarray(sel.cpu() if torch.is_tensor(sel) else sel)
    R, G, _ = sel.shape
    n_list = as_lengths(n, R)
    slot_map = np.full((R, G, n_max), -1, dtype=np.int32)
    hot_tok = np.full((R, G, S), -1, dtype=np.int32)
    for r in range(R):
        for g in range(G):
            rng = np.random.default_rng(row_seed(seed, r, g, TAG_SLOTS))
            chosen = sel[r, g][sel[r, g] >= 0].astype(np.int64)
            k_eff = chosen.size
            n_hit = min(S, k_eff - int(round(miss_frac * k_eff)))
            hits = rng.choice(chosen, size=n_hit, replace=False) if n_hit > 0 else chosen[:0]
            mask = np.ones(n_list[r], dtype=bool)
            mask[chosen] = False
            pool = np.nonzero(mask)[0]
            n_fill = min(S - n_hit, pool.size)
            fill = rng.choice(pool, size=n_fill, replace=False) if n_fill > 0 else pool[:0]
            toks = np.concatenate([hits, fill])
            order = rng.permutation(S)[: toks.size]
            hot_tok[r, g, order] = toks
            slot_map[r, g, toks] = order
    return slot_map, hot_tok


def hot_rows(full: torch.Tensor, hot_tok) -> torch.Tensor:
    """Copies of the full rows held by each slot: [R][G][S][D] (zero rows for empty slots)."""
    ht = torch.as_tensor(np.asarray(hot_tok), device=full.device).long()
    R, G, S = ht.shape
    D = full.shape[-1]
    idx = ht.clamp(min=0).unsqueeze(-1).expand(R, G, S, D)
    out = torch.gather(full, 2, idx)
    out[ht < 0] = 0
    return out


def lightning_inputs(R: int, n, Hi: int = 64, Dl: int = 128, n_max: int | None = None,
                     seed: int = 3, device="cpu"):
    """Lightning-indexer inputs.

    kidx: e4m3 codes (uint8) [R][n_max][Dl] of N(0,1)/sqrt(128) (torch's
    float8_e4m3fn conversion), qidx: bf16 [R][Hi][Dl] N(0,1), w: f32 [R][Hi]
    U(0,1). Rows past n[r] are zero codes.
    """
    n_list = as_lengths(n, R)
    n_max = max(n_list) if n_max is None else n_max
    kidx = torch.zeros(R, n_max, Dl, dtype=torch.uint8, device=device)
    qidx = torch.empty(R, Hi, Dl, dtype=torch.bfloat16, device=device)
    w = torch.empty(R, Hi, dtype=torch.float32, device=device)
    for r in range(R):
        nr = n_list[r]
        z = torch.randn(nr, Dl, generator=_gen(device, seed, r, TAG_KIDX), dtype=torch.float32,
                        device=device) / math.sqrt(128.0)
        kidx[r, :nr] = z.to(torch.float8_e4m3fn).view(torch.uint8)
        qidx[r] = torch.randn(Hi, Dl, generator=_gen(device, seed, r, TAG_QIDX),
                              dtype=torch.float32, device=device).to(torch.bfloat16)
        w[r] = torch.rand(Hi, generator=_gen(device, seed, r, TAG_W), dtype=torch.float32,
                          device=device)
    return kidx, qidx, w, n_list


def plane_words(n_max: int) -> int:
    """Words per bit plane: ceil(n_max / 32) rounded up to a multiple of 4."""
    w = (n_max + 31) // 32
    return (w + 3) // 4 * 4
