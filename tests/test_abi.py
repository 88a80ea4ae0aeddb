"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/kvscan.h declares, and rejects bad arguments on the host before
any launch (no CUDA call is reached on these paths)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvscan.h")).read()
    return sorted(set(re.findall(r"KVS_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def kvs():
    from kv_index_scan_b200 import build
    build.build()
    import kv_index_scan_b200
    return kv_index_scan_b200


def test_header_declares_the_boundary():
    names = _declared()
    for f in ["fathom_plan_bits", "index_scan", "topk_select", "sparse_gather",
              "sparse_decode_attn", "decode_step", "kvs_build_fathom_index", "kvs_abi_version",
              "kvs_last_error"]:
        assert f in names


def test_library_exports_every_declared_symbol(kvs):
    lib = ctypes.CDLL(kvs.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert kvs.abi_version() == 1


def test_host_argument_checks(kvs):
    L = kvs._lib
    # null index descriptor
    plan = kvs.PlanC(None, None, None, None, 92)
    st = L.fathom_plan_bits(ctypes.c_void_p(16), 4, None, 92, ctypes.byref(plan), None, None)
    assert st == kvs.KVS_EINVAL and b"index" in L.kvs_last_error()
    # unsupported head dim
    ix = kvs.FathomIndexC(16, 16, 16, 16, 1, 1, 64, 128, 0)
    st = L.fathom_plan_bits(ctypes.c_void_p(16), 4, ctypes.byref(ix), 92, ctypes.byref(plan), None, None)
    assert st == kvs.KVS_EUNSUPPORTED
    # budget beyond 4*D
    ix = kvs.FathomIndexC(16, 16, 16, 16, 1, 1, 128, 128, 0)
    plan = kvs.PlanC(16, 16, 16, 16, 513)
    st = L.fathom_plan_bits(ctypes.c_void_p(16), 4, ctypes.byref(ix), 513, ctypes.byref(plan), None, None)
    assert st == kvs.KVS_EINVAL
    # misaligned planes
    ix = kvs.FathomIndexC(20, 16, 16, 16, 1, 1, 128, 128, 0)
    plan = kvs.PlanC(16, 16, 16, 16, 92)
    st = L.fathom_plan_bits(ctypes.c_void_p(16), 4, ctypes.byref(ix), 92, ctypes.byref(plan), None, None)
    assert st == kvs.KVS_EINVAL and b"aligned" in L.kvs_last_error()
    # W not a multiple of 4
    ix = kvs.FathomIndexC(16, 16, 16, 16, 1, 1, 128, 126, 0)
    st = L.fathom_plan_bits(ctypes.c_void_p(16), 4, ctypes.byref(ix), 92, ctypes.byref(plan), None, None)
    assert st == kvs.KVS_EINVAL
    # top-k: block must divide k
    st = L.topk_select(16, 100, 16, 1, 1, 100, 64, 16, None, None, 0, None, None)
    assert st == kvs.KVS_EINVAL
    # attention: H out of range, D != 128
    st = L.sparse_decode_attn(16, 0, 16, 16, None, 1, 1, 9, 128, 8, 1.0, 16, None, None, 0, None, None)
    assert st == kvs.KVS_EINVAL
    st = L.sparse_decode_attn(16, 0, 16, 16, None, 1, 1, 4, 64, 8, 1.0, 16, None, None, 0, None, None)
    assert st == kvs.KVS_EUNSUPPORTED
    # decode step: workspace too small is reported before any launch
    ix = kvs.FathomIndexC(16, 16, 16, 16, 1, 1, 128, 128, 0)
    plan = kvs.PlanC(16, 16, 16, 16, 92)
    a = kvs.DecodeArgsC(16, 0, 4, ctypes.pointer(ix), ctypes.pointer(plan), 256, 16, 4096, None,
                        None, None, 0, 16, 16, None, 0, 0.1, 16, None, 16, None, None)
    st = L.decode_step(ctypes.byref(a), None, 0, None, None)
    assert st == kvs.KVS_EWORKSPACE
    assert L.kvs_decode_step_workspace_size(16, 8, 4, 131072, 2048, 92) > 0


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "kv_index_scan_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "oracle.cpp" not in text, f


def test_selftest_and_append_argument_checks(kvs):
    """The failure-path self-test and the write-back refuse bad arguments on
    the host, before any launch."""
    L = kvs._lib
    ix = kvs.FathomIndexC(16, 16, 16, 16, 1, 1, 128, 128, 0)
    plan = kvs.PlanC(16, 16, 16, 16, 92)
    # no status word, a wait bound out of range, an index in host memory
    assert L.kvs_selftest_scan_timeout(ctypes.byref(ix), ctypes.byref(plan), 16, 4096, 16, 2000000,
                                       None, None) == kvs.KVS_EINVAL
    assert L.kvs_selftest_scan_timeout(ctypes.byref(ix), ctypes.byref(plan), 16, 4096, 16, 10,
                                       16, None) == kvs.KVS_EINVAL
    ixh = kvs.FathomIndexC(16, 16, 16, 16, 1, 1, 128, 128, 1)
    assert L.kvs_selftest_scan_timeout(ctypes.byref(ixh), ctypes.byref(plan), 16, 4096, 16, 2000000,
                                       16, None) == kvs.KVS_EUNSUPPORTED
    # append: W too small for n_max, G out of range, a hot slot without a slot map
    args = [16, 16, 16, 1, 1, 128, 4096, 16, 128, 16, 16, 16, 16, None, None, None, None, None, 0, None, None]
    a = list(args); a[8] = 64
    assert L.kvs_append_token(*a) == kvs.KVS_EINVAL
    a = list(args); a[4] = 9
    assert L.kvs_append_token(*a) == kvs.KVS_EINVAL
    a = list(args); a[14] = 16
    assert L.kvs_append_token(*a) == kvs.KVS_EINVAL
    assert b"hot_slot" in L.kvs_last_error()
