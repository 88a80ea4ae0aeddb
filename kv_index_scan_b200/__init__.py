"""Python binding of libkvscan.so: the B200 per-step top-k sparse-attention
decode path (Fathom bit-plane index scan, top-k, hot-buffer gather, sparse GQA
attention, and the lightning-indexer variant).

This module only marshals arguments: it allocates output tensors with torch,
passes raw device pointers and the current CUDA stream to the C ABI declared in
include/kvscan.h, and raises on a non-OK status. Every step runs in the CUDA
kernels of the library; there is no CPU fallback. Importing fails loudly when
the library has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvscan.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m kv_index_scan_b200.build` "
        "(nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

KVS_OK, KVS_EINVAL, KVS_EUNSUPPORTED, KVS_ECUDA, KVS_EWORKSPACE, KVS_ETIMEOUT, KVS_EBOUNDS = range(7)
KVS_F32, KVS_BF16 = 0, 1
KVS_SCAN_FATHOM, KVS_SCAN_LIGHTNING = 0, 1
STATUS_NAMES = {0: "KVS_OK", 1: "KVS_EINVAL", 2: "KVS_EUNSUPPORTED", 3: "KVS_ECUDA",
                4: "KVS_EWORKSPACE", 5: "KVS_ETIMEOUT", 6: "KVS_EBOUNDS"}

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
SZ = ctypes.c_size_t
F32 = ctypes.c_float


class FathomIndexC(ctypes.Structure):
    _fields_ = [("planes", P), ("kmin", P), ("kstep", P), ("kvar", P), ("R", I32), ("G", I32),
                ("D", I32), ("W", I32), ("host_mapped", I32)]


class PlanC(ctypes.Structure):
    _fields_ = [("t", P), ("plane_idx", P), ("plane_w", P), ("C", P), ("B", I32)]


class ScanArgsC(ctypes.Structure):
    _fields_ = [("kind", I32), ("R", I32), ("n_max", I32), ("n", P), ("ix", ctypes.POINTER(FathomIndexC)),
                ("plan", ctypes.POINTER(PlanC)), ("kidx", P), ("qidx", P), ("widx", P), ("Hi", I32),
                ("Dl", I32), ("block", I32)]


class DecodeArgsC(ctypes.Structure):
    _fields_ = [("q", P), ("q_dtype", I32), ("H", I32), ("ix", ctypes.POINTER(FathomIndexC)),
                ("plan", ctypes.POINTER(PlanC)), ("k", I32), ("n", P), ("n_max", I32),
                ("slot_map", P), ("hotK", P), ("hotV", P), ("S", I32), ("fullK", P), ("fullV", P),
                ("idx_in", P), ("idx_shared", I32), ("scale", F32), ("out", P), ("lse", P),
                ("idx", P), ("slots", P), ("misses", P)]


def _declare():
    L = _lib
    L.kvs_abi_version.restype = I32
    L.kvs_last_error.restype = ctypes.c_char_p
    L.kvs_build_fathom_index.argtypes = [P, P, I32, I32, I32, I32, I32, P, P, P, P, P, SZ, P, P]
    L.kvs_build_fathom_index.restype = I32
    L.kvs_build_index_workspace_size.argtypes = [I32, I32, I32]
    L.kvs_build_index_workspace_size.restype = SZ
    L.fathom_plan_bits.argtypes = [P, I32, ctypes.POINTER(FathomIndexC), I32, ctypes.POINTER(PlanC), P, P]
    L.fathom_plan_bits.restype = I32
    L.index_scan.argtypes = [ctypes.POINTER(ScanArgsC), P, P, P]
    L.index_scan.restype = I32
    L.topk_select.argtypes = [P, I64, P, I32, I32, I32, I32, P, P, P, SZ, P, P]
    L.topk_select.restype = I32
    L.kvs_topk_workspace_size.argtypes = [I32, I32, I32, I32, I32]
    L.kvs_topk_workspace_size.restype = SZ
    L.sparse_gather.argtypes = [P, I32, P, P, P, I32, P, P, P, I32, I32, I32, I32, P, P, P, P, P, P]
    L.sparse_gather.restype = I32
    L.sparse_decode_attn.argtypes = [P, I32, P, P, P, I32, I32, I32, I32, I32, F32, P, P, P, SZ, P, P]
    L.sparse_decode_attn.restype = I32
    L.kvs_attn_workspace_size.argtypes = [I32, I32, I32, I32]
    L.kvs_attn_workspace_size.restype = SZ
    L.sparse_decode_attn_noalloc.argtypes = [P, I32, P, P, P, I32, I32, I32, I32, I32, F32, P, P, P, P]
    L.sparse_decode_attn_noalloc.restype = I32
    L.decode_step.argtypes = [ctypes.POINTER(DecodeArgsC), P, SZ, P, P]
    L.decode_step.restype = I32
    L.kvs_decode_step_workspace_size.argtypes = [I32, I32, I32, I32, I32, I32]
    L.kvs_decode_step_workspace_size.restype = SZ
    L.kvs_decode_step_workspace_size_host.argtypes = [I32, I32, I32, I32, I32, I32]
    L.kvs_decode_step_workspace_size_host.restype = SZ
    L.decode_step_timed.argtypes = [ctypes.POINTER(DecodeArgsC), P, SZ, P, P, ctypes.POINTER(P), I32]
    L.decode_step_timed.restype = I32
    L.kvs_append_token.argtypes = [P, P, P, I32, I32, I32, I32, P, I32, P, P, P, P, P, P, P, P, P, I32,
                                   P, P]
    L.kvs_append_token.restype = I32
    L.kvs_selftest_scan_timeout.argtypes = [ctypes.POINTER(FathomIndexC), ctypes.POINTER(PlanC), P, I32,
                                            P, I64, P, P]
    L.kvs_selftest_scan_timeout.restype = I32


_declare()


class KvsError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.kvs_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status: int, where: str):
    if status != KVS_OK:
        raise KvsError(status, where)


def abi_version() -> int:
    return _lib.kvs_abi_version()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, MappedHostStore):
        return t.ptr
    return t.data_ptr()


def _stream(stream=None) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _u16(t):
    return t.view(torch.int16) if isinstance(t, torch.Tensor) and t.dtype == torch.bfloat16 else t


def plane_words(n_max: int) -> int:
    """Words per bit plane: ceil(n_max / 32) rounded up to a multiple of 4."""
    return ((n_max + 31) // 32 + 3) // 4 * 4


class FathomIndex:
    """The 4-bit channel-major bit-plane K index (tensors owned by torch).

    planes int32 [R][G][D][4][W] (u32 bit patterns), kmin/kstep/kvar f32 [R][G][D].
    `planes_ptr` overrides the planes address (a mapped pinned host alias).
    """

    def __init__(self, planes, kmin, kstep, kvar, planes_ptr: int | None = None,
                 host_mapped: bool = False):
        self.planes, self.kmin, self.kstep, self.kvar = planes, kmin, kstep, kvar
        self.R, self.G, self.D, _, self.W = planes.shape
        self.planes_ptr = planes_ptr
        self.host_mapped = host_mapped

    def c(self) -> FathomIndexC:
        pp = self.planes_ptr if self.planes_ptr is not None else self.planes.data_ptr()
        return FathomIndexC(pp, _ptr(self.kmin), _ptr(self.kstep), _ptr(self.kvar), self.R, self.G,
                            self.D, self.W, int(self.host_mapped))


class MappedHostIndex(FathomIndex):
    """A FathomIndex whose planes live in mapped pinned host memory
    (cudaHostAlloc with cudaHostAllocMapped); the scan reads them over the host
    link through the device alias from cudaHostGetDevicePointer. The host
    buffer is freed when this object is."""

    def __init__(self, index: FathomIndex):
        from cuda.bindings import runtime as rt
        self._rt = rt
        nbytes = index.planes.numel() * 4
        err, hptr = rt.cudaHostAlloc(nbytes, rt.cudaHostAllocMapped | rt.cudaHostAllocPortable)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostAlloc: {err}")
        self._hptr = hptr
        err, dptr = rt.cudaHostGetDevicePointer(hptr, 0)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostGetDevicePointer: {err}")
        torch.cuda.synchronize()
        err, = rt.cudaMemcpy(hptr, index.planes.data_ptr(), nbytes,
                             rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpy: {err}")
        super().__init__(index.planes, index.kmin, index.kstep, index.kvar, planes_ptr=int(dptr),
                         host_mapped=True)
        self.nbytes = nbytes

    def __del__(self):
        try:
            self._rt.cudaFreeHost(self._hptr)
        except Exception:
            pass


class MappedHostStore:
    """A full K or V store in mapped pinned host memory (cudaHostAlloc with
    cudaHostAllocMapped): the host tier of the pages' system. `ptr` is its
    device alias, which decode_step reads over the host link (only the missing
    selected rows). Built from a bf16 device tensor [R][G][n_max][D]; the host
    buffer is freed when this object is."""

    def __init__(self, t: torch.Tensor):
        from cuda.bindings import runtime as rt
        self._rt = rt
        self.shape = tuple(t.shape)
        self.nbytes = t.numel() * t.element_size()
        err, hptr = rt.cudaHostAlloc(self.nbytes, rt.cudaHostAllocMapped | rt.cudaHostAllocPortable)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostAlloc: {err}")
        self._hptr = hptr
        err, dptr = rt.cudaHostGetDevicePointer(hptr, 0)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostGetDevicePointer: {err}")
        torch.cuda.synchronize()
        err, = rt.cudaMemcpy(hptr, t.data_ptr(), self.nbytes, rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaMemcpy: {err}")
        self.ptr = int(dptr)

    def __del__(self):
        try:
            self._rt.cudaFreeHost(self._hptr)
        except Exception:
            pass


class Plan:
    """Per-(r, g) bit allocation: t u8 [R][G][D], plane_idx int16 [R][G][B]
    (u16 plane ids c*4+p), plane_w f32 [R][G][B], C f32 [R][G]."""

    def __init__(self, R: int, G: int, D: int, B: int, device):
        self.B = B
        self.t = torch.empty(R, G, D, dtype=torch.uint8, device=device)
        self.plane_idx = torch.empty(R, G, max(B, 1), dtype=torch.int16, device=device)
        self.plane_w = torch.empty(R, G, max(B, 1), dtype=torch.float32, device=device)
        self.C = torch.empty(R, G, dtype=torch.float32, device=device)

    def c(self) -> PlanC:
        return PlanC(_ptr(self.t), _ptr(self.plane_idx), _ptr(self.plane_w), _ptr(self.C), self.B)


def _n_tensor(n, R: int, device) -> torch.Tensor:
    if isinstance(n, torch.Tensor):
        return n.to(device=device, dtype=torch.int32).contiguous()
    if isinstance(n, int):
        n = [n] * R
    return torch.tensor(list(n), dtype=torch.int32, device=device)


def build_fathom_index(K: torch.Tensor, n, W: int | None = None, stream=None,
                       dev_status=None) -> FathomIndex:
    """a0: K bf16 [R][G][n_max][D] -> FathomIndex (kvs_build_fathom_index)."""
    R, G, n_max, D = K.shape
    W = plane_words(n_max) if W is None else W
    dev = K.device
    nt = _n_tensor(n, R, dev)
    planes = torch.empty(R, G, D, 4, W, dtype=torch.int32, device=dev)
    kmin = torch.empty(R, G, D, dtype=torch.float32, device=dev)
    kstep = torch.empty_like(kmin)
    kvar = torch.empty_like(kmin)
    wsb = _lib.kvs_build_index_workspace_size(R, G, D)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    st = _lib.kvs_build_fathom_index(_ptr(_u16(K)), _ptr(nt), R, G, n_max, D, W, _ptr(planes),
                                     _ptr(kmin), _ptr(kstep), _ptr(kvar), _ptr(ws), ws.numel(),
                                     _ptr(dev_status), _stream(stream))
    _check(st, "kvs_build_fathom_index")
    return FathomIndex(planes, kmin, kstep, kvar)


def fathom_plan_bits(q: torch.Tensor, index: FathomIndex, B: int, plan: Plan | None = None,
                     stream=None, dev_status=None) -> Plan:
    """a1: q f32 [R][G][H][D] -> Plan."""
    R, G, H, D = q.shape
    plan = plan or Plan(R, G, D, B, q.device)
    ix, pc = index.c(), plan.c()
    st = _lib.fathom_plan_bits(_ptr(q), H, ctypes.byref(ix), B, ctypes.byref(pc), _ptr(dev_status),
                               _stream(stream))
    _check(st, "fathom_plan_bits")
    return plan


def index_scan_fathom(index: FathomIndex, plan: Plan, n, n_max: int, scores=None, stream=None,
                      dev_status=None) -> torch.Tensor:
    """a2 (Fathom): scores f32 [R][G][n_max] (-inf past n[r])."""
    dev = index.kmin.device
    nt = _n_tensor(n, index.R, dev)
    if scores is None:
        scores = torch.empty(index.R, index.G, n_max, dtype=torch.float32, device=dev)
    ix, pc = index.c(), plan.c()
    a = ScanArgsC(KVS_SCAN_FATHOM, index.R, n_max, _ptr(nt), ctypes.pointer(ix), ctypes.pointer(pc),
                  None, None, None, 0, 0, 0)
    _check(_lib.index_scan(ctypes.byref(a), _ptr(scores), _ptr(dev_status), _stream(stream)),
           "index_scan(fathom)")
    return scores


def index_scan_lightning(kidx: torch.Tensor, qidx: torch.Tensor, w: torch.Tensor, n,
                         block: int = 64, scores=None, stream=None, dev_status=None) -> torch.Tensor:
    """a2 (lightning): kidx e4m3 codes u8 [R][n_max][Dl], qidx bf16 [R][Hi][Dl], w f32 [R][Hi]
    -> block scores f32 [R][ceil(n_max/block)] (token scores when block == 1)."""
    R, n_max, Dl = kidx.shape
    Hi = qidx.shape[1]
    nt = _n_tensor(n, R, kidx.device)
    nb = (n_max + block - 1) // block
    if scores is None:
        scores = torch.empty(R, nb, dtype=torch.float32, device=kidx.device)
    a = ScanArgsC(KVS_SCAN_LIGHTNING, R, n_max, _ptr(nt), None, None, _ptr(kidx), _ptr(_u16(qidx)),
                  _ptr(w), Hi, Dl, block)
    _check(_lib.index_scan(ctypes.byref(a), _ptr(scores), _ptr(dev_status), _stream(stream)),
           "index_scan(lightning)")
    return scores


def topk_select(scores: torch.Tensor, n, k: int, block: int = 1, want_vals: bool = False,
                idx=None, stream=None, dev_status=None):
    """a3: scores f32 [R][G][ld] (or [R][ld]) -> idx int32 [R][G][k] (and vals)."""
    s3 = scores if scores.dim() == 3 else scores.unsqueeze(1)
    R, G, ld = s3.shape
    nt = _n_tensor(n, R, scores.device)
    if idx is None:
        idx = torch.empty(R, G, k, dtype=torch.int32, device=scores.device)
    vals = torch.empty(R, G, k, dtype=torch.float32, device=scores.device) if want_vals else None
    wsb = _lib.kvs_topk_workspace_size(R, G, ld, k, block)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=scores.device)
    st = _lib.topk_select(_ptr(s3), ld, _ptr(nt), R, G, k, block, _ptr(idx), _ptr(vals), _ptr(ws),
                          ws.numel(), _ptr(dev_status), _stream(stream))
    _check(st, "topk_select")
    if scores.dim() == 2:
        idx = idx.squeeze(1)
        vals = vals.squeeze(1) if vals is not None else None
    return (idx, vals) if want_vals else idx


def sparse_gather(idx, slot_map, hotK, hotV, fullK, fullV, n, stream=None, dev_status=None):
    """a4: -> (gK, gV bf16 [R][G][k][D], slots int32 [R][G][k], misses int32 [R][G])."""
    R, G, k = idx.shape
    S = hotK.shape[2]
    n_max, D = fullK.shape[2], fullK.shape[3]
    dev = idx.device
    nt = _n_tensor(n, R, dev)
    gK = torch.empty(R, G, k, D, dtype=torch.bfloat16, device=dev)
    gV = torch.empty_like(gK)
    slots = torch.empty(R, G, k, dtype=torch.int32, device=dev)
    misses = torch.empty(R, G, dtype=torch.int32, device=dev)
    st = _lib.sparse_gather(_ptr(idx), k, _ptr(slot_map), _ptr(_u16(hotK)), _ptr(_u16(hotV)), S,
                            _ptr(_u16(fullK)), _ptr(_u16(fullV)), _ptr(nt), n_max, R, G, D,
                            _ptr(_u16(gK)), _ptr(_u16(gV)), _ptr(slots), _ptr(misses),
                            _ptr(dev_status), _stream(stream))
    _check(st, "sparse_gather")
    return gK, gV, slots, misses


def sparse_decode_attn(q, K, V, k_eff=None, scale: float | None = None, want_lse: bool = True,
                       stream=None, dev_status=None):
    """a5: q f32/bf16 [R][G][H][D], K/V bf16 [R][G][k][D] -> (out f32 [R][G][H][D], lse)."""
    R, G, H, D = q.shape
    k = K.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = torch.empty(R, G, H, D, dtype=torch.float32, device=q.device)
    lse = torch.empty(R, G, H, dtype=torch.float32, device=q.device) if want_lse else None
    wsb = _lib.kvs_attn_workspace_size(R, G, H, k)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    qd = KVS_BF16 if q.dtype == torch.bfloat16 else KVS_F32
    st = _lib.sparse_decode_attn(_ptr(_u16(q)), qd, _ptr(_u16(K)), _ptr(_u16(V)), _ptr(k_eff), R, G,
                                 H, D, k, scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                 _ptr(dev_status), _stream(stream))
    _check(st, "sparse_decode_attn")
    return out, lse


def _require(cond: bool, what: str):
    if not cond:
        raise ValueError(what)


def sparse_decode_attn_noalloc(q, K, V, out, lse=None, k_eff=None, scale: float | None = None,
                               stream=None, dev_status=None):
    """a5 without a workspace, into caller-provided out (and lse): the library
    keeps the split-K scratch in a fixed device array (see include/kvscan.h).
    out must be f32 [R][G][H][D] and lse f32 [R][G][H], contiguous, on q's
    device; k_eff (nullable) int32 [R][G]."""
    R, G, H, D = q.shape
    k = K.shape[2]
    for name, t, shape, dt in (("out", out, (R, G, H, D), torch.float32),
                               ("lse", lse, (R, G, H), torch.float32),
                               ("k_eff", k_eff, (R, G), torch.int32)):
        if t is None:
            _require(name != "out", "out is required")
            continue
        _require(t.dtype == dt, f"{name} must be {dt}, got {t.dtype}")
        _require(tuple(t.shape) == shape, f"{name} must have shape {shape}, got {tuple(t.shape)}")
        _require(t.is_contiguous(), f"{name} must be contiguous")
        _require(t.device == q.device, f"{name} must be on {q.device}")
    _require(tuple(K.shape) == (R, G, k, D) and tuple(V.shape) == (R, G, k, D),
             "K and V must be [R][G][k][D]")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qd = KVS_BF16 if q.dtype == torch.bfloat16 else KVS_F32
    st = _lib.sparse_decode_attn_noalloc(_ptr(_u16(q)), qd, _ptr(_u16(K)), _ptr(_u16(V)), _ptr(k_eff),
                                         R, G, H, D, k, scale, _ptr(out), _ptr(lse),
                                         _ptr(dev_status), _stream(stream))
    _check(st, "sparse_decode_attn_noalloc")
    return out, lse


def append_token(index: FathomIndex, Knew, Vnew, n: torch.Tensor, fullK, fullV, slot_map=None,
                 hot_slot=None, hot_tok=None, hotK=None, hotV=None, stream=None, dev_status=None):
    """Per-step write-back (kvs_append_token): the new token Knew/Vnew bf16
    [R][G][D] of every request joins its rows at position n[r] -- its 4-bit
    codes (the index's own quantiser) into the planes, its K/V rows into the
    full store, optionally a hot slot (hot_slot int32 [R][G], with hot_tok
    int32 [R][G][S] the token each slot holds) -- and n (device int32 [R]) is
    advanced in place."""
    R, G, D = Knew.shape
    n_max = fullK.shape[2]
    if n.dtype != torch.int32 or not n.is_contiguous() or n.device != Knew.device:
        raise ValueError("n must be a contiguous device int32 tensor on Knew's device")
    S = hotK.shape[2] if hotK is not None else 0
    st = _lib.kvs_append_token(_ptr(_u16(Knew)), _ptr(_u16(Vnew)), _ptr(n), R, G, D, n_max,
                               _ptr(index.planes), index.W, _ptr(index.kmin), _ptr(index.kstep),
                               _ptr(_u16(fullK)), _ptr(_u16(fullV)), _ptr(slot_map), _ptr(hot_slot),
                               _ptr(hot_tok), _ptr(_u16(hotK)), _ptr(_u16(hotV)), S,
                               _ptr(dev_status), _stream(stream))
    _check(st, "kvs_append_token")


def selftest_scan_timeout(index: FathomIndex, plan: Plan, n, n_max: int, wait_cycles: int,
                          dev_status: torch.Tensor, stream=None):
    """kvs_selftest_scan_timeout: the HBM scan with a withheld producer
    arrival, so that its bounded waits run out; dev_status (device int32)
    receives KVS_ETIMEOUT. For tests of the failure path."""
    nt = _n_tensor(n, index.R, index.kmin.device)
    scores = torch.empty(index.R, index.G, n_max, dtype=torch.float32, device=index.kmin.device)
    ix, pc = index.c(), plan.c()
    st = _lib.kvs_selftest_scan_timeout(ctypes.byref(ix), ctypes.byref(pc), _ptr(nt), n_max,
                                        _ptr(scores), wait_cycles, _ptr(dev_status), _stream(stream))
    _check(st, "kvs_selftest_scan_timeout")


def decode_step_workspace_size(R, G, H, n_max, k, B) -> int:
    return int(_lib.kvs_decode_step_workspace_size(R, G, H, n_max, k, B))


class DecodeStep:
    """a6 with persistent, caller-owned buffers (like a graph-captured decode
    layer): outputs and workspace are allocated once, each call only launches."""

    def __init__(self, index: FathomIndex, n, n_max: int, H: int, B: int, k: int, fullK, fullV,
                 slot_map=None, hotK=None, hotV=None, scale: float | None = None,
                 q_dtype=torch.float32, device=None):
        dev = device or index.kmin.device
        self.index, self.H, self.B, self.k, self.n_max = index, H, B, k, n_max
        R, G, D = index.R, index.G, index.D
        self.R, self.G, self.D = R, G, D
        self.n = _n_tensor(n, R, dev)
        self.fullK, self.fullV, self.slot_map, self.hotK, self.hotV = fullK, fullV, slot_map, hotK, hotV
        self.S = hotK.shape[2] if hotK is not None else 0
        self.scale = 1.0 / math.sqrt(D) if scale is None else scale
        self.plan = Plan(R, G, D, B, dev)
        self.out = torch.empty(R, G, H, D, dtype=torch.float32, device=dev)
        self.lse = torch.empty(R, G, H, dtype=torch.float32, device=dev)
        self.idx = torch.empty(R, G, k, dtype=torch.int32, device=dev)
        self.slots = torch.empty(R, G, k, dtype=torch.int32, device=dev)
        self.misses = torch.empty(R, G, dtype=torch.int32, device=dev)
        # a full store in host memory (MappedHostStore) needs the staging too
        self.full_on_host = isinstance(fullK, MappedHostStore)
        wsb = (int(_lib.kvs_decode_step_workspace_size_host(R, G, H, n_max, k, B)) if self.full_on_host
               else decode_step_workspace_size(R, G, H, n_max, k, B))
        self.ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
        self.q_dtype = KVS_BF16 if q_dtype == torch.bfloat16 else KVS_F32
        self._ix = index.c()
        self._plan = self.plan.c()

    def args(self, q, idx_in=None, idx_shared: bool = False, out=None) -> DecodeArgsC:
        return DecodeArgsC(
            _ptr(_u16(q)), self.q_dtype, self.H, ctypes.pointer(self._ix), ctypes.pointer(self._plan),
            self.k, _ptr(self.n), self.n_max, _ptr(self.slot_map), _ptr(_u16(self.hotK)),
            _ptr(_u16(self.hotV)), self.S, _ptr(_u16(self.fullK)), _ptr(_u16(self.fullV)),
            _ptr(idx_in), int(idx_shared), self.scale, _ptr(self.out if out is None else out),
            _ptr(self.lse), _ptr(self.idx), _ptr(self.slots), _ptr(self.misses))

    def __call__(self, q, idx_in=None, idx_shared: bool = False, stream=None, dev_status=None,
                 out=None):
        a = self.args(q, idx_in, idx_shared, out)
        st = _lib.decode_step(ctypes.byref(a), _ptr(self.ws), self.ws.numel(), _ptr(dev_status),
                              _stream(stream))
        _check(st, "decode_step")
        return self.out if out is None else out

    DECODE_STAGES = ("allocation", "scan", "selection", "attention")

    def timed(self, q, events, idx_in=None, idx_shared: bool = False, stream=None,
              dev_status=None, out=None):
        """decode_step_timed: as __call__, recording the 5 torch.cuda.Event(enable_timing=True)
        objects in `events` at the stage boundaries (see DECODE_STAGES)."""
        if len(events) != len(self.DECODE_STAGES) + 1:
            raise ValueError(f"{len(self.DECODE_STAGES) + 1} events needed")
        s = stream if stream is not None else torch.cuda.current_stream()
        for e in events:  # make sure each event exists (torch creates it lazily)
            e.record(s)
        evs = (P * len(events))(*[e.cuda_event for e in events])
        a = self.args(q, idx_in, idx_shared, out)
        st = _lib.decode_step_timed(ctypes.byref(a), _ptr(self.ws), self.ws.numel(),
                                    _ptr(dev_status), _stream(s), evs, len(events))
        _check(st, "decode_step_timed")
        return self.out if out is None else out


def decode_step(q, index: FathomIndex, n, B: int, k: int, fullK, fullV, slot_map=None, hotK=None,
                hotV=None, scale=None, idx_in=None, idx_shared=False, stream=None):
    """a6 one-shot: returns (out, lse, idx, slots, misses, plan)."""
    R, G, H, D = q.shape
    step = DecodeStep(index, n, fullK.shape[2], H, B, k, fullK, fullV, slot_map, hotK, hotV, scale,
                      q_dtype=q.dtype)
    step(q, idx_in=idx_in, idx_shared=idx_shared, stream=stream)
    return step.out, step.lse, step.idx, step.slots, step.misses, step.plan
