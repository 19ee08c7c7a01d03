"""Parity of the backward (moba_backward) with the fp64 backward oracle.

The backward is defined over a fixed selection (no gradient passes through
the hard gate), so both sides take the selection the GPU forward wrote; the
forward's own selection parity is tested in test_gpu_parity.py.  Every
element of dq, dk and dv is compared.

Tolerance, from the arithmetic: the outputs are rounded to bf16 and P and dS
enter the tensor-core products as bf16 (relative error up to 2^-8 each),
with fp32 accumulation; the error is therefore a small multiple of 2^-8 of
the gradients' scale.  Bound: max |err| <= 2e-2 * max |ref| and mean |err|
<= 2e-3 * max |ref|, per tensor.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import Oracle, bf16_bits

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 2e-2, 2e-3


@pytest.fixture(scope="module")
def moba():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as m
    return m


CASES = [
    # N, Hq, Hkv, d, B, k
    (1024, 2, 1, 128, 256, 3),
    (2048, 4, 2, 128, 256, 4),
    (1500, 4, 1, 64, 128, 3),     # ragged last block, d = 64, GQA 4
    (1024, 2, 2, 128, 128, 1),    # k = 1: own block only
    (1280, 2, 1, 128, 256, 9),    # k beyond the blocks
]


@pytest.mark.parametrize("case", CASES, ids=["%d_%d_%d_%d_%d_%d" % c for c in CASES])
def test_backward_matches_oracle(moba, case):
    N, Hq, Hkv, d, B, k = case
    w = S.Workload("bw", [N], Hq, Hkv, d, B, k, seed=1111)
    q, kk, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, N, x.shape[1], d) for x in (q, kk, v))
    sel = torch.empty(1, Hq, N, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward(q4, k4, v4, B, k, sel_out=sel)
    g = torch.Generator(device="cuda").manual_seed(77)
    dO = torch.randn(1, N, Hq, d, generator=g, device="cuda").to(torch.bfloat16)
    p = moba.make_params(1, N, Hq, Hkv, d, B, k)
    ws = moba.alloc_workspace(moba.backward_workspace_size(p, 0))
    dq, dk, dv = moba.backward(q4, k4, v4, o, lse, dO, sel, B, k, ws=ws)
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == 0
    orc = Oracle(bf16_bits(q), bf16_bits(kk), bf16_bits(v), w.cu, Hq, Hkv, d, B, k)
    rows = np.arange(N, dtype=np.int64)
    sel_rows = sel[0].permute(1, 0, 2).contiguous().cpu().numpy()
    rq, rk, rv = orc.attend_backward(rows, sel_rows, bf16_bits(dO[0]))
    for name, got, ref in (("dq", dq[0], rq), ("dk", dk[0], rk), ("dv", dv[0], rv)):
        got = got.float().cpu().numpy().astype(np.float64)
        scale = np.abs(ref).max()
        err = np.abs(got - ref)
        assert err.max() <= MAX_REL * scale, (name, err.max(), scale)
        assert err.mean() <= MEAN_REL * scale, (name, err.mean(), scale)


def test_backward_is_deterministic_up_to_atomic_order(moba):
    N, Hq, Hkv, d, B, k = 2048, 4, 2, 128, 256, 4
    w = S.Workload("bw2", [N], Hq, Hkv, d, B, k, seed=2222)
    q, kk, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, N, x.shape[1], d) for x in (q, kk, v))
    sel = torch.empty(1, Hq, N, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward(q4, k4, v4, B, k, sel_out=sel)
    dO = torch.randn_like(o.float()).to(torch.bfloat16)
    a = moba.backward(q4, k4, v4, o, lse, dO, sel, B, k)
    b = moba.backward(q4, k4, v4, o, lse, dO, sel, B, k)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        # fp32 atomic sums may add in a different order: equal to bf16 rounding
        assert torch.allclose(x.float(), y.float(), rtol=1e-2, atol=1e-3)


@pytest.mark.parametrize("lengths,Hq,Hkv,d,B,k", [
    ([700, 1, 1300, 0, 900], 4, 2, 128, 256, 3),
    ([1500, 600], 4, 1, 64, 128, 4),
])
def test_backward_varlen_matches_oracle(moba, lengths, Hq, Hkv, d, B, k):
    """The packed-sequence backward: every element of dq, dk, dv against the
    oracle, over the selection forward_varlen wrote (blocks counted from each
    sequence's start, no key or row crossing a sequence boundary)."""
    w = S.Workload("bw_varlen", lengths, Hq, Hkv, d, B, k, seed=1212, batch_mode=False)
    q, kk, v = S.make_qkv(w, "cuda")
    cu = torch.tensor(w.cu, dtype=torch.int32, device="cuda")
    sel = torch.empty(Hq, w.T, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward_varlen(q, kk, v, cu, B, k, sel_out=sel)
    g = torch.Generator(device="cuda").manual_seed(79)
    dO = torch.randn(w.T, Hq, d, generator=g, device="cuda").to(torch.bfloat16)
    p = moba.make_params(1, 0, Hq, Hkv, d, B, k)
    ws = moba.alloc_workspace(moba.backward_workspace_size_varlen(p, w.T, len(lengths), 0))
    dq, dk, dv = moba.backward_varlen(q, kk, v, o, lse, dO, sel, cu, B, k, ws=ws)
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == 0
    orc = Oracle(bf16_bits(q), bf16_bits(kk), bf16_bits(v), w.cu, Hq, Hkv, d, B, k)
    rows = np.arange(w.T, dtype=np.int64)
    sel_rows = sel.permute(1, 0, 2).contiguous().cpu().numpy()
    rq, rk, rv = orc.attend_backward(rows, sel_rows, bf16_bits(dO))
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        got = got.float().cpu().numpy().astype(np.float64)
        scale = np.abs(ref).max()
        err = np.abs(got - ref)
        assert err.max() <= MAX_REL * scale, (name, err.max(), scale)
        assert err.mean() <= MEAN_REL * scale, (name, err.mean(), scale)
