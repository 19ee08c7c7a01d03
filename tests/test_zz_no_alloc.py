"""Allocation-free gate entry point, checked against the workspace gate and
the fp64 oracle.

moba_gate_noalloc is for callers that cannot allocate device memory or pass
a workspace (code inside a host framework that owns every device allocation,
or a latency-critical loop that must not call cudaMalloc).  It keeps its
scratch in one fixed array inside the library.  These tests call it through
the C ABI:
  * twice in a row, on two different shapes: the selection must equal
    moba_gate's exactly (integer data), and the oracle's on every row except
    flagged near-ties (the prefill's selection rule, parity_util);
  * with a shape too large for the fixed scratch and null pointers: it must
    refuse with MOBA_ERR_WORKSPACE, so nothing is ever launched on them;
  * with its status word made to latch a timeout (the bounded-wait self-test
    aimed at it): moba_gate_noalloc_status must report it once, clear it, and
    later calls must run and report no error.

The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import Oracle, bf16_bits
from parity_util import FLAG_REL

pytestmark = pytest.mark.gpu

MOBA_ERR_WORKSPACE = 3
MOBA_ERR_TIMEOUT = 5


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def moba():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as m
    return m


def _noalloc(moba, w, q4, k4, stream):
    lib = moba.load_library()
    b, N = len(w.lengths), w.lengths[0]
    got = torch.full((b, w.Hq, N, w.k), -9, dtype=torch.int32, device="cuda")
    p = moba.make_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
    rc = lib.moba_gate_noalloc(_ptr(q4), _ptr(k4), _ptr(got), ctypes.byref(p), stream)
    assert rc == 0, moba._STATUS.get(rc, rc)
    return got


def test_gate_noalloc_matches_gate_and_oracle_on_two_calls(moba):
    lib = moba.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        S.Workload("noalloc_a", [8192], 8, 2, 128, 256, 5, seed=901),
        S.Workload("noalloc_b", [3000, 3000], 4, 4, 64, 128, 3, seed=902),
    ]
    for w in cases:
        q, k, _ = S.make_qkv(w, "cuda", need_v=False)
        b, N = len(w.lengths), w.lengths[0]
        q4 = q.view(b, N, w.Hq, w.d)
        k4 = k.view(b, N, w.Hkv, w.d)
        ref = moba.gate(q4, k4, w.B, w.k)
        got = _noalloc(moba, w, q4, k4, stream)
        assert lib.moba_gate_noalloc_status(stream) == 0
        assert torch.equal(got, ref), w.name
        # against the oracle: every row, flagged near-ties exempt
        orc = Oracle(bf16_bits(q), bf16_bits(k), None, w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
        rows = np.arange(w.T, dtype=np.int64)
        osel, margin, maxabs = orc.select(rows)
        gsel = got.permute(0, 2, 1, 3).reshape(w.T, w.Hq, w.k).cpu().numpy()
        differ = np.any(gsel != osel, axis=2)
        flagged = margin < FLAG_REL * maxabs
        assert not (differ & ~flagged).any(), (w.name, int((differ & ~flagged).sum()))


def test_gate_noalloc_refuses_shapes_beyond_its_scratch(moba):
    lib = moba.load_library()
    # 8 kv heads x 8192 blocks x 128 dims x 4 B = 32 MiB of block means > 16 MiB;
    # the size is checked before the (null) pointers, so nothing can launch
    p = moba.make_params(4, 262144, 8, 8, 128, 128, 3)
    null = ctypes.c_void_p(None)
    assert lib.moba_gate_noalloc(null, null, null, ctypes.byref(p), None) == MOBA_ERR_WORKSPACE


def test_gate_noalloc_reports_a_latched_device_error_once(moba):
    lib = moba.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.moba_gate_noalloc_status(stream) == 0
    # a bounded wait on a barrier nothing arrives on, latching into the gate's word
    assert lib.moba_selftest_wait_timeout(None, 0, 20_000_000, stream) == 0
    assert lib.moba_gate_noalloc_status(stream) == MOBA_ERR_TIMEOUT
    assert lib.moba_gate_noalloc_status(stream) == 0  # reading cleared it
    w = S.Workload("noalloc_after", [4096], 4, 1, 128, 256, 4, seed=903)
    q, k, _ = S.make_qkv(w, "cuda", need_v=False)
    q4, k4 = q.view(1, 4096, 4, 128), k.view(1, 4096, 1, 128)
    got = _noalloc(moba, w, q4, k4, stream)
    assert lib.moba_gate_noalloc_status(stream) == 0
    assert torch.equal(got, moba.gate(q4, k4, w.B, w.k))
