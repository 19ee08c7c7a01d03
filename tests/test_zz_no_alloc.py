"""Allocation-free gate entry point, checked against the workspace gate.

moba_gate_noalloc is for callers that cannot allocate device memory or pass
a workspace (code inside a host framework that owns every device allocation,
or a latency-critical loop that must not call cudaMalloc).  It keeps its
scratch in one fixed array inside the library.  This test calls it through
the C ABI twice in a row, on two different shapes, and requires the same
selection as moba_gate (exactly: the selection is integer data).  It also
checks that a shape too large for the fixed scratch is refused.

The file name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu

MOBA_ERR_WORKSPACE = 3


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_gate_noalloc_matches_gate_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as moba
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
        got = torch.full_like(ref, -9)
        p = moba.make_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
        rc = lib.moba_gate_noalloc(_ptr(q4), _ptr(k4), _ptr(got), ctypes.byref(p), stream)
        assert rc == 0, moba._STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), w.name


def test_gate_noalloc_refuses_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_long_07_b200 as moba
    lib = moba.load_library()
    # 8 kv heads x 8192 blocks x 128 dims x 4 B = 32 MiB of block means > 16 MiB
    p = moba.make_params(4, 262144, 8, 8, 128, 128, 3)
    fake = ctypes.c_void_p(1 << 20)
    assert lib.moba_gate_noalloc(fake, fake, fake, ctypes.byref(p), None) == MOBA_ERR_WORKSPACE
