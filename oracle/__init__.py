"""CPU oracle for the per-step top-k sparse-attention decode path.

TEST INFRASTRUCTURE ONLY: imported by tests/, the smoke check and the
benchmark's CPU-baseline leg, never by the product package. The arithmetic is
plain C++ in oracle.cpp (fp64, each step the plain definition, with the page it
follows cited there); this file only compiles it and marshals numpy arrays.
It shares no code with the CUDA library and imports nothing from it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (contraction and fast-math off)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared",
               "-fPIC", "-pthread", _SRC, "-o", _LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        _declare(_lib)
    return _lib


P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
F64 = ctypes.c_double


def _declare(L):
    L.oracle_version.restype = I32
    L.oracle_build_index.argtypes = [P, I64, I32, I32, P, P, P, P]
    L.oracle_plan_bits.argtypes = [P, I32, I32, P, I32, P, P]
    L.oracle_plan_bits.restype = I32
    L.oracle_scan.argtypes = [P, I32, I32, P, P, P, P, I64, P]
    L.oracle_topk.argtypes = [P, I64, I32, P]
    L.oracle_topk.restype = I32
    L.oracle_topk_f32.argtypes = [P, I64, I32, P]
    L.oracle_topk_f32.restype = I32
    L.oracle_gather.argtypes = [P, I32, P, P, P, P, P, I32, P, P, P]
    L.oracle_gather.restype = I32
    L.oracle_append_token.argtypes = [P, P, I64, I32, I32, P, P, P, P, P, P, I32, P, P, P]
    L.oracle_attention.argtypes = [P, I32, I32, P, P, I32, F64, P, P]
    L.oracle_lightning_scores.argtypes = [P, I64, I32, P, I32, P, P]
    L.oracle_block_max.argtypes = [P, I64, I32, P]
    L.oracle_block_topk.argtypes = [P, I64, I32, I32, P]
    L.oracle_block_topk.restype = I32
    L.oracle_block_topk_f32.argtypes = [P, I64, I32, I32, P]
    L.oracle_block_topk_f32.restype = I32
    L.oracle_build_index_batch.argtypes = [P, P, I32, I32, I32, I32, I32, P, P, P, P, I32]
    L.oracle_decode_batch.argtypes = [P, I32, I32, I32, I32, P, I32, P, P, P, P, I32, I32, I32,
                                      P, P, P, I32, P, P, F64, P, I32, I32, P, P, P, P, P, P, P]
    L.oracle_decode_batch.restype = I32
    L.oracle_lightning_batch.argtypes = [P, P, P, I32, I32, I32, P, I32, I32, I32, P, I32, I32,
                                         P, P]
    L.oracle_shared_attention_batch.argtypes = [P, I32, I32, I32, I32, P, P, I32, P, I32, F64, P,
                                                I32, I32, P, P]


def _arr(a, dtype):
    """Contiguous numpy array of dtype; torch tensors are moved to the CPU first
    (bf16 tensors are reinterpreted as their uint16 bit patterns)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16)
            a = a.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(a)
    if a.dtype != dtype:
        if dtype == np.uint16 and a.dtype == np.int16:
            a = a.view(np.uint16)
        else:
            a = a.astype(dtype)
    return np.ascontiguousarray(a)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def nthreads_default() -> int:
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- single rows

def build_index(K, D: int, W: int):
    """O0 for one (request, KV head): K bf16 [n][D] -> planes [D][4][W], kmin, kstep, kvar."""
    K = _arr(K, np.uint16)
    n = K.shape[0]
    planes = np.zeros((D, 4, W), np.uint32)
    kmin, kstep, kvar = (np.zeros(D, np.float32) for _ in range(3))
    lib().oracle_build_index(_p(K), n, D, W, _p(planes), _p(kmin), _p(kstep), _p(kvar))
    return planes, kmin, kstep, kvar


def append_token(knew, vnew, i: int, planes, kmin, kstep, fullK, fullV, slot_map=None, slot: int = -1,
                 hot_tok=None, hotK=None, hotV=None):
    """O0b for one row, on copies: returns (planes, fullK, fullV, slot_map,
    hot_tok, hotK, hotV) after writing token i (see oracle.cpp)."""
    planes = _arr(planes, np.uint32).copy()
    D, _, W = planes.shape
    fullK = _arr(fullK, np.uint16).copy()
    fullV = _arr(fullV, np.uint16).copy()
    sm = None if slot_map is None else _arr(slot_map, np.int32).copy()
    ht = None if hot_tok is None else _arr(hot_tok, np.int32).copy()
    hK = None if hotK is None else _arr(hotK, np.uint16).copy()
    hV = None if hotV is None else _arr(hotV, np.uint16).copy()
    lib().oracle_append_token(_p(_arr(knew, np.uint16)), _p(_arr(vnew, np.uint16)), i, D, W, _p(planes),
                              _p(_arr(kmin, np.float32)), _p(_arr(kstep, np.float32)), _p(fullK),
                              _p(fullV), _p(sm), slot, _p(ht), _p(hK), _p(hV))
    return planes, fullK, fullV, sm, ht, hK, hV


def plan_bits(q, kvar, B: int):
    """O1 for one row: q f32 [H][D], kvar f32 [D] -> (t u8 [D], qbar f32 [D])."""
    q = _arr(q, np.float32)
    kvar = _arr(kvar, np.float32)
    H, D = q.shape
    t = np.zeros(D, np.uint8)
    qbar = np.zeros(D, np.float32)
    rc = lib().oracle_plan_bits(_p(q), H, D, _p(kvar), B, _p(t), _p(qbar))
    if rc != 0:
        raise ValueError(f"bad bit budget B={B} for D={D}")
    return t, qbar


def scan(planes, kmin, kstep, qbar, t, n: int):
    """O2 for one row: fp64 scores [n]."""
    planes = _arr(planes, np.uint32)
    D, _, W = planes.shape
    out = np.zeros(n, np.float64)
    lib().oracle_scan(_p(planes), D, W, _p(_arr(kmin, np.float32)), _p(_arr(kstep, np.float32)),
                      _p(_arr(qbar, np.float32)), _p(_arr(t, np.uint8)), n, _p(out))
    return out


def topk(scores, k: int):
    """O3: (idx int32 [k] ascending, -1 padded; k_eff). fp64 or f32 scores."""
    s = np.asarray(scores)
    idx = np.zeros(k, np.int32)
    if s.dtype == np.float32:
        s = np.ascontiguousarray(s)
        k_eff = lib().oracle_topk_f32(_p(s), s.size, k, _p(idx))
    else:
        s = _arr(s, np.float64)
        k_eff = lib().oracle_topk(_p(s), s.size, k, _p(idx))
    return idx, k_eff


def gather(idx, slot_map, hotK, hotV, fullK, fullV):
    """O4 for one row -> (gK, gV uint16 [k][D], slots int32 [k], misses)."""
    idx = _arr(idx, np.int32)
    k = idx.size
    fullK = _arr(fullK, np.uint16)
    D = fullK.shape[-1]
    gK = np.zeros((k, D), np.uint16)
    gV = np.zeros((k, D), np.uint16)
    slots = np.zeros(k, np.int32)
    m = lib().oracle_gather(_p(idx), k, _p(_arr(slot_map, np.int32)), _p(_arr(hotK, np.uint16)),
                            _p(_arr(hotV, np.uint16)), _p(fullK), _p(_arr(fullV, np.uint16)), D,
                            _p(gK), _p(gV), _p(slots))
    return gK, gV, slots, m


def attention(q, K, V, k_eff: int, scale: float):
    """O5 for one row: q f32 [H][D], K/V bf16 [>=k_eff][D] -> (out fp64 [H][D], lse fp64 [H])."""
    q = _arr(q, np.float32)
    H, D = q.shape
    K = _arr(K, np.uint16)
    V = _arr(V, np.uint16)
    out = np.zeros((H, D), np.float64)
    lse = np.zeros(H, np.float64)
    lib().oracle_attention(_p(q), H, D, _p(K), _p(V), k_eff, scale, _p(out), _p(lse))
    return out, lse


def lightning_scores(kidx, qidx, w):
    """O6 token scores for one request: kidx u8 [n][Dl], qidx bf16 [Hi][Dl], w [Hi] -> fp64 [n]."""
    kidx = _arr(kidx, np.uint8)
    qidx = _arr(qidx, np.uint16)
    n, Dl = kidx.shape
    Hi = qidx.shape[0]
    out = np.zeros(n, np.float64)
    lib().oracle_lightning_scores(_p(kidx), n, Dl, _p(qidx), Hi, _p(_arr(w, np.float32)), _p(out))
    return out


def block_max(scores, block: int):
    s = _arr(scores, np.float64)
    nb = (s.size + block - 1) // block
    out = np.zeros(nb, np.float64)
    lib().oracle_block_max(_p(s), s.size, block, _p(out))
    return out


def block_topk(bscores, n: int, block: int, k: int):
    """Block top-k expanded to tokens: (idx int32 [k], count)."""
    b = np.asarray(bscores)
    idx = np.zeros(k, np.int32)
    if b.dtype == np.float32:
        b = np.ascontiguousarray(b)
        c = lib().oracle_block_topk_f32(_p(b), n, block, k, _p(idx))
    else:
        b = _arr(b, np.float64)
        c = lib().oracle_block_topk(_p(b), n, block, k, _p(idx))
    return idx, c


# ----------------------------------------------------------------------------- batches

def build_index_batch(K, n, W: int, nthreads: int | None = None):
    """O0 over K bf16 [R][G][n_max][D] -> planes [R][G][D][4][W], kmin/kstep/kvar [R][G][D]."""
    K = _arr(K, np.uint16)
    R, G, n_max, D = K.shape
    n = _arr(n, np.int32)
    planes = np.zeros((R, G, D, 4, W), np.uint32)
    kmin, kstep, kvar = (np.zeros((R, G, D), np.float32) for _ in range(3))
    lib().oracle_build_index_batch(_p(K), _p(n), R, G, n_max, D, W, _p(planes), _p(kmin),
                                   _p(kstep), _p(kvar), nthreads or nthreads_default())
    return planes, kmin, kstep, kvar


def decode_batch(q, planes, kmin, kstep, kvar, n, B: int, k: int, slot_map, hotK, hotV, fullK,
                 fullV, scale: float, rows=None, nthreads: int | None = None,
                 want_scores: bool = False):
    """The Fathom decode step O1..O5 for rows u = r*G + g (all rows when None).

    Returns a dict with t, idx, slots, misses, out, lse (and scores) laid out
    over all R*G rows; rows that were not processed stay zero.
    """
    q = _arr(q, np.float32)
    R, G, H, D = q.shape
    planes = _arr(planes, np.uint32)
    W = planes.shape[-1]
    fullK = _arr(fullK, np.uint16)
    fullV = _arr(fullV, np.uint16)
    n_max = fullK.shape[2]
    n = _arr(n, np.int32)
    S = 0 if hotK is None else int(np.asarray(hotK.shape)[2])
    res = dict(t=np.zeros((R, G, D), np.uint8), idx=np.zeros((R, G, k), np.int32),
               slots=np.zeros((R, G, k), np.int32), misses=np.zeros((R, G), np.int32),
               out=np.zeros((R, G, H, D), np.float64), lse=np.zeros((R, G, H), np.float64))
    scores = np.zeros((R, G, n_max), np.float64) if want_scores else None
    rows_a = None if rows is None else _arr(rows, np.int32)
    rc = lib().oracle_decode_batch(
        _p(q), R, G, H, D, _p(planes), W, _p(_arr(kmin, np.float32)), _p(_arr(kstep, np.float32)),
        _p(_arr(kvar, np.float32)), _p(n), n_max, B, k,
        _p(None if slot_map is None else _arr(slot_map, np.int32)),
        _p(None if hotK is None else _arr(hotK, np.uint16)),
        _p(None if hotV is None else _arr(hotV, np.uint16)), S, _p(fullK), _p(fullV), scale,
        _p(rows_a), 0 if rows_a is None else rows_a.size, nthreads or nthreads_default(),
        _p(res["t"]), _p(res["idx"]), _p(res["slots"]), _p(res["misses"]), _p(res["out"]),
        _p(res["lse"]), _p(scores))
    if rc != 0:
        raise ValueError(f"bad bit budget B={B}")
    if want_scores:
        res["scores"] = scores
    return res


def lightning_batch(kidx, qidx, w, n, block: int, k: int, reqs=None, nthreads=None):
    """O6 selection for requests (all when None): (bscores fp64 [R][nb], idx int32 [R][k])."""
    kidx = _arr(kidx, np.uint8)
    qidx = _arr(qidx, np.uint16)
    R, n_max, Dl = kidx.shape
    Hi = qidx.shape[1]
    n = _arr(n, np.int32)
    nb = (n_max + block - 1) // block
    bs = np.zeros((R, nb), np.float64)
    idx = np.zeros((R, k), np.int32)
    reqs_a = None if reqs is None else _arr(reqs, np.int32)
    lib().oracle_lightning_batch(_p(kidx), _p(qidx), _p(_arr(w, np.float32)), R, Hi, Dl, _p(n),
                                 n_max, block, k, _p(reqs_a),
                                 0 if reqs_a is None else reqs_a.size,
                                 nthreads or nthreads_default(), _p(bs), _p(idx))
    return bs, idx


def shared_attention_batch(q, K, V, idx, scale: float, rows=None, nthreads=None):
    """O5 over a per-request selection shared by all KV heads: (out [R][G][H][D], lse [R][G][H])."""
    q = _arr(q, np.float32)
    R, G, H, D = q.shape
    K = _arr(K, np.uint16)
    V = _arr(V, np.uint16)
    n_max = K.shape[2]
    idx = _arr(idx, np.int32)
    k = idx.shape[-1]
    out = np.zeros((R, G, H, D), np.float64)
    lse = np.zeros((R, G, H), np.float64)
    rows_a = None if rows is None else _arr(rows, np.int32)
    lib().oracle_shared_attention_batch(_p(q), R, G, H, D, _p(K), _p(V), n_max, _p(idx), k, scale,
                                        _p(rows_a), 0 if rows_a is None else rows_a.size,
                                        nthreads or nthreads_default(), _p(out), _p(lse))
    return out, lse
