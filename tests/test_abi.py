"""Host-side checks of the C ABI: the library builds and loads, exports every
symbol include/moba.h declares, and rejects bad arguments before launching
anything.  No call here reaches a kernel, so these run without a GPU."""
import ctypes
import os
import re

import pytest

import block_sparse_long_07_b200 as moba
from block_sparse_long_07_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moba.h")

INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return moba.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moba_[a-z_]+)\s*\(", text)))


def test_header_declares_the_prefill_calls():
    names = declared_functions()
    for n in ("moba_gate", "moba_forward", "moba_forward_varlen", "moba_full_causal",
              "moba_workspace_size", "moba_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(moba.EXPORTS) == set(declared_functions())


def test_no_oracle_in_product_library():
    so = open(moba.LIB_PATH, "rb").read()
    assert b"oracle_" not in so
    src_dir = os.path.join(ROOT, "block_sparse_long_07_b200")
    for dirpath, _, files in os.walk(src_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f


def test_status_strings(lib):
    for code, name in moba._STATUS.items():
        assert lib.moba_status_string(code).decode() == name
    assert lib.moba_status_string(99).decode() == "MOBA_ERR_UNKNOWN"
    assert lib.moba_version() >= 100


def _p(**kw):
    d = dict(batch=1, seqlen=2048, Hq=32, Hkv=8, d=128, block_size=256, top_k=4)
    d.update(kw)
    return moba.make_params(d["batch"], d["seqlen"], d["Hq"], d["Hkv"], d["d"], d["block_size"],
                            d["top_k"])


def test_workspace_size_grows_with_heads_per_pass(lib):
    p = _p()
    one = moba.workspace_size(p, 1)
    allh = moba.workspace_size(p, 0)
    assert 0 < one < allh
    assert moba.workspace_size(p, 8) == allh
    assert moba.workspace_size(p, 4) < allh
    # a bigger top_k needs more partial slots
    assert moba.workspace_size(_p(top_k=8), 1) > one
    assert moba.workspace_size_varlen(p, 2048, 1, 1) >= one
    assert moba.full_causal_workspace_size(2048, 1) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), UNSUPPORTED),
    (dict(block_size=100), UNSUPPORTED),
    (dict(block_size=0), INVALID),
    (dict(top_k=0), INVALID),
    (dict(Hq=30, Hkv=8), INVALID),
    (dict(Hkv=0), INVALID),
    (dict(batch=0), INVALID),
    (dict(seqlen=-1), INVALID),
    # T * Hq = 2^31 (q rows take an int32 index)
    (dict(seqlen=1 << 26, block_size=1 << 20), UNSUPPORTED),
])
def test_bad_params_rejected(lib, kw, code):
    p = _p(**kw)
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.moba_forward(fake, fake, fake, fake, fake, None, ctypes.byref(p), fake, 1 << 40, None)
    assert rc == code
    assert moba.workspace_size(p, 1) == 0


def test_null_and_misaligned_pointers_rejected(lib):
    p = _p()
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 24)
    big = moba.workspace_size(p, 0)
    assert lib.moba_forward(None, fake, fake, fake, fake, None, ctypes.byref(p), ws, big, None) == INVALID
    assert lib.moba_forward(ctypes.c_void_p((1 << 20) + 2), fake, fake, fake, fake, None,
                            ctypes.byref(p), ws, big, None) == INVALID
    assert lib.moba_gate(fake, fake, None, ctypes.byref(p), ws, big, None) == INVALID
    assert lib.moba_full_causal(fake, None, fake, fake, fake, ctypes.byref(p), ws, big, None) == INVALID
    assert lib.moba_forward_varlen(fake, fake, fake, None, 1, 2048, fake, fake, None,
                                   ctypes.byref(p), ws, big, None) == INVALID


def test_workspace_checks(lib):
    p = _p()
    fake = ctypes.c_void_p(1 << 20)
    need = moba.workspace_size(p, 1)
    # too small, null, misaligned
    assert lib.moba_forward(fake, fake, fake, fake, fake, None, ctypes.byref(p), fake, need - 1,
                            None) == WORKSPACE
    assert lib.moba_forward(fake, fake, fake, fake, fake, None, ctypes.byref(p), None, need,
                            None) == WORKSPACE
    assert lib.moba_forward(fake, fake, fake, fake, fake, None, ctypes.byref(p),
                            ctypes.c_void_p((1 << 20) + 16), need, None) == WORKSPACE
    assert lib.moba_gate(fake, fake, fake, ctypes.byref(p), fake, need - 1, None) == WORKSPACE
    dneed = moba.full_causal_workspace_size(2048, 1)
    assert lib.moba_full_causal(fake, fake, fake, fake, fake, ctypes.byref(p), fake, dneed - 1,
                                None) == WORKSPACE
    assert lib.moba_last_device_status(None, None) == WORKSPACE


def test_topk_limit(lib):
    # more than 64 ranked past blocks is outside the register top-k
    p = _p(seqlen=65536, block_size=128, top_k=70)
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.moba_forward(fake, fake, fake, fake, fake, None, ctypes.byref(p), fake, 1 << 45, None)
    assert rc == UNSUPPORTED
    # ... unless every block is taken anyway (k >= n)
    p2 = _p(seqlen=4096, block_size=128, top_k=70)
    assert moba.workspace_size(p2, 1) > 0


def test_binding_refuses_missing_library(tmp_path):
    with pytest.raises(OSError):
        moba.load_library(str(tmp_path / "nope.so"))


def test_selftest_argument_checks(lib):
    # the limit is checked first; a null ws would aim at the allocation-free
    # gate's status word, which needs a device
    assert lib.moba_selftest_wait_timeout(None, 4096, 0, None) == INVALID
    fake = ctypes.c_void_p(1 << 20)
    assert lib.moba_selftest_wait_timeout(ctypes.c_void_p(1 << 20 | 8), 4096, 1000, None) == WORKSPACE
    assert lib.moba_selftest_wait_timeout(fake, 4096, 0, None) == INVALID
    assert lib.moba_selftest_wait_timeout(fake, 4096, 10**12, None) == INVALID
    assert lib.moba_selftest_wait_timeout(fake, 16, 1000, None) == WORKSPACE


def _dp(**kw):
    d = dict(batch=2, cap=8192, Hq=8, Hkv=2, d=128, B=256, k=4)
    d.update(kw)
    return moba.make_decode_params(d["batch"], d["cap"], d["Hq"], d["Hkv"], d["d"], d["B"],
                                   d["k"])


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), UNSUPPORTED),
    (dict(B=100), UNSUPPORTED),
    (dict(k=66), UNSUPPORTED),
    (dict(k=0), INVALID),
    (dict(Hq=6, Hkv=4), INVALID),
    (dict(batch=0), INVALID),
    (dict(cap=0), INVALID),
    (dict(cap=256 * 8192 + 1), UNSUPPORTED),  # 8193 blocks of 256
])
def test_decode_bad_params_rejected(lib, kw, code):
    p = _dp(**kw)
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.moba_decode(fake, fake, fake, fake, fake, fake, fake, None, ctypes.byref(p), fake,
                         1 << 40, None)
    assert rc == code
    assert moba.decode_workspace_size(p) == 0 and moba.kbar_cache_size(p) == 0


def test_decode_pointer_and_workspace_checks(lib):
    p = _dp()
    fake = ctypes.c_void_p(1 << 20)
    need = moba.decode_workspace_size(p)
    assert need > 0
    assert moba.kbar_cache_size(p) == 4 * 2 * 2 * (8192 // 256) * 128
    args = [fake] * 8
    for bad in range(7):  # q, k, v, seqlens, kbar, o, lse may not be null
        a = list(args)
        a[bad] = None
        assert lib.moba_decode(*a, ctypes.byref(p), fake, need, None) == INVALID
    a = list(args)
    a[0] = ctypes.c_void_p((1 << 20) + 8)  # q not 16-byte aligned
    assert lib.moba_decode(*a, ctypes.byref(p), fake, need, None) == INVALID
    assert lib.moba_decode(*args, ctypes.byref(p), fake, need - 1, None) == WORKSPACE
    assert lib.moba_decode(*args, ctypes.byref(p), None, need, None) == WORKSPACE
    assert lib.moba_kbar_cache_update(fake, fake, fake, 0, ctypes.byref(p), fake, need - 1,
                                      None) == WORKSPACE
    assert lib.moba_kbar_cache_update(None, fake, fake, 0, ctypes.byref(p), fake, need,
                                      None) == INVALID


def test_backward_argument_checks(lib):
    p = _p()
    fake = ctypes.c_void_p(1 << 20)
    need = moba.backward_workspace_size(p, 1)
    assert need > 0 and moba.backward_workspace_size(p, 2) > need
    args = [fake] * 10  # q, k, v, o, lse, dO, sel, dq, dk, dv
    for bad in range(10):
        a = list(args)
        a[bad] = None
        assert lib.moba_backward(*a, ctypes.byref(p), fake, need, None) == INVALID
    a = list(args)
    a[5] = ctypes.c_void_p((1 << 20) + 8)  # dO not 16-byte aligned
    assert lib.moba_backward(*a, ctypes.byref(p), fake, need, None) == INVALID
    a = list(args)
    a[6] = ctypes.c_void_p((1 << 20) + 2)  # sel not 4-byte aligned
    assert lib.moba_backward(*a, ctypes.byref(p), fake, need, None) == INVALID
    assert lib.moba_backward(*args, ctypes.byref(p), fake, need - 1, None) == WORKSPACE
    assert lib.moba_backward(*args, ctypes.byref(p), None, need, None) == WORKSPACE
    bad = _p(d=96)
    assert lib.moba_backward(*args, ctypes.byref(bad), fake, 1 << 40, None) == UNSUPPORTED


def test_routing_variant_argument_checks(lib):
    p = _p()
    fake = ctypes.c_void_p(1 << 20)
    need = moba.workspace_size(p, 1)
    # static selections: a destination and one of the two modes
    assert lib.moba_static_selection(None, 0, ctypes.byref(p), None) == INVALID
    assert lib.moba_static_selection(ctypes.c_void_p((1 << 20) + 2), 0, ctypes.byref(p),
                                     None) == INVALID
    assert lib.moba_static_selection(fake, 7, ctypes.byref(p), None) == INVALID
    # min/max gate: q, k, sel, then the workspace
    assert lib.moba_gate_minmax(None, fake, fake, ctypes.byref(p), fake, need, None) == INVALID
    assert lib.moba_gate_minmax(fake, fake, None, ctypes.byref(p), fake, need, None) == INVALID
    assert lib.moba_gate_minmax(fake, fake, fake, ctypes.byref(p), fake, need - 1,
                                None) == WORKSPACE
    # forward over a given selection needs the selection
    assert lib.moba_forward_selected(fake, fake, fake, fake, fake, None, ctypes.byref(p), fake,
                                     need, None) == INVALID
    assert lib.moba_forward_minmax(None, fake, fake, fake, fake, None, ctypes.byref(p), fake,
                                   need, None) == INVALID


def test_forward_host_argument_checks(lib):
    p = _p()
    host = ctypes.c_void_p(1 << 20)
    dev = ctypes.c_void_p(1 << 24)  # kAlign-aligned
    need = moba.forward_host_buffer_size(p, 1)
    assert need > moba.workspace_size(p, 1)  # workspace plus the staging of one kv-head group
    for bad in range(5):  # q, k, v, o, lse
        a = [host] * 5
        a[bad] = None
        assert lib.moba_forward_host(*a, None, ctypes.byref(p), dev, need, None) == INVALID
    a = [host] * 5
    assert lib.moba_forward_host(*a, None, ctypes.byref(p), None, need, None) == WORKSPACE
    assert lib.moba_forward_host(*a, None, ctypes.byref(p), ctypes.c_void_p((1 << 24) + 16),
                                 need, None) == WORKSPACE
    assert lib.moba_forward_host(*a, None, ctypes.byref(p), dev, need - 1, None) == WORKSPACE
