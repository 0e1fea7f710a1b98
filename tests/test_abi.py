"""The C-ABI library: it loads, exports every symbol the header declares, and rejects bad
arguments on the host before touching the GPU (these calls need no device)."""
import ctypes
import os
import re

import pytest

from int4_routed_expert_gemv_b200 import binding as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "colimoe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(coli_\w+)\s*\(", src)))


def test_header_symbols_exported(colimoe):
    names = declared_functions()
    assert len(names) >= 12
    L = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(L, n), f"{n} declared in colimoe.h but not exported"
    assert sorted(B.EXPORTS) == names


def test_sizes(colimoe):
    assert B.coli_moe_blob_bytes(6144, 2048) == 20054016
    assert B.coli_moe_blob_bytes(1024, 512) == 835584
    d = B.make_dims(6144, 2048, 256, 8, 1)
    ws1 = B.coli_moe_workspace_bytes(d, 1)
    ws4 = B.coli_moe_workspace_bytes(d, 4)
    assert 0 < ws1 < ws4 and ws1 % 256 == 0
    for bad in [(6144, 2048, 256, 33, 1), (6100, 2048, 256, 8, 1), (6144, 2048, 2000, 8, 1),
                (6144, 2048, 4, 8, 1), (6144, 2048, 256, 8, 2), (0, 64, 4, 1, 0)]:
        assert B.coli_moe_workspace_bytes(B.make_dims(*bad), 1) == 0, bad
    assert B.coli_moe_workspace_bytes(d, -1) == 0


def test_status_strings(colimoe):
    assert B.status_string(B.COLI_OK) == "ok"
    assert "workspace" in B.status_string(B.COLI_ENOMEM)
    assert B.status_string(99) == "unknown status"


def test_host_side_rejections(colimoe):
    L = B.lib()
    d = B.make_dims(1024, 512, 64, 4, 1)
    bad = B.make_dims(1024, 512, 64, 65, 1)
    P = ctypes.c_void_p
    fake = P(0x10000)          # aligned non-null: never dereferenced on these paths
    mis = P(0x10004)           # misaligned
    big = 1 << 40
    r = L.coli_moe_route
    assert r(ctypes.byref(bad), fake, None, fake, 0, 1, fake, fake, None, fake, big, None) == B.COLI_EINVAL
    assert r(ctypes.byref(d), fake, None, fake, 0, -1, fake, fake, None, fake, big, None) == B.COLI_EINVAL
    assert r(ctypes.byref(d), fake, None, fake, 0, 0, fake, fake, None, fake, big, None) == B.COLI_OK
    assert r(ctypes.byref(d), None, None, fake, 0, 1, fake, fake, None, fake, big, None) == B.COLI_EINVAL
    assert r(ctypes.byref(d), fake, None, mis, 0, 1, fake, fake, None, fake, big, None) == B.COLI_EINVAL
    assert r(ctypes.byref(d), fake, None, fake, 7, 1, fake, fake, None, fake, big, None) == B.COLI_EINVAL
    assert r(ctypes.byref(d), fake, None, fake, 0, 1, fake, fake, None, fake, 16, None) == B.COLI_ENOMEM
    assert r(ctypes.byref(d), fake, None, fake, 0, 1, fake, fake, None, mis, big, None) == B.COLI_EINVAL
    w_bad_stride = B.Weights(fake, None, fake, fake, 835584 + 1)
    w_ok = B.Weights(fake, None, fake, fake, 835584 + 256 - 835584 % 256)
    f = L.coli_moe_forward
    args = lambda w, dt=0, T=1: (ctypes.byref(d), ctypes.byref(w), fake, dt, T, fake, fake, fake,
                                 fake, fake, fake, None, fake, fake, big, None)
    assert f(*args(w_bad_stride)) == B.COLI_EINVAL
    assert f(*args(w_ok, T=0)) == B.COLI_OK
    assert f(*args(w_ok, dt=3)) == B.COLI_EINVAL
    no_shared = B.Weights(fake, None, fake, None, 835840)
    assert f(*args(no_shared)) == B.COLI_EINVAL
    u = L.coli_moe_union
    assert u(ctypes.byref(d), None, 1, fake, fake, fake, fake, fake, big, None) == B.COLI_EINVAL
    assert L.coli_rmsnorm(0, 1, fake, fake, 1e-5, fake, None) == B.COLI_EINVAL
    assert L.coli_rmsnorm(64, 1, fake, fake, -1.0, fake, None) == B.COLI_EINVAL
    assert L.coli_moe_workspace_init(None, 256, None) == B.COLI_EINVAL
