"""Parity of the routing variants (static window / sink selections, the
min/max-pooled gate, the forward over a given selection) with the oracle.

Selections are compared exactly (the min/max gate with the same near-tie
rule as the mean gate: a row may differ only where the oracle's margin is
below 1e-3 of its largest score); O and lse within the forward's tolerances,
against the oracle's attention over the selection each side used.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import Oracle, bf16_bits, local_block_info, static_selection
from parity_util import FLAG_REL, LSE_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, check_selection_invariants

pytestmark = pytest.mark.gpu


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
    (4096, 8, 2, 128, 256, 4),
    (3000, 4, 1, 64, 128, 3),     # ragged last block, d = 64, GQA 4
    (2048, 4, 2, 128, 256, 1),    # k = 1
    (1536, 4, 2, 128, 512, 9),    # k beyond the block count
    (8192, 4, 2, 128, 128, 12),   # many blocks
]
IDS = ["%d_%d_%d_%d_%d_%d" % c for c in CASES]


def _setup(case, seed):
    N, Hq, Hkv, d, B, k = case
    w = S.Workload("variant", [N], Hq, Hkv, d, B, k, seed=seed)
    q, kk, v = S.make_qkv(w, "cuda")
    orc = Oracle(bf16_bits(q), bf16_bits(kk), bf16_bits(v), w.cu, Hq, Hkv, d, B, k)
    shape4 = lambda x: x.view(1, N, x.shape[1], d)
    return w, shape4(q), shape4(kk), shape4(v), orc


def _gpu_rows(o, lse, sel, N):
    """o [1,N,H,d], lse [1,H,N], sel [1,H,N,k] -> [N,H,d], [N,H], [N,H,k]."""
    return (o[0].float().cpu().numpy(), lse[0].t().contiguous().cpu().numpy(),
            None if sel is None else sel[0].permute(1, 0, 2).contiguous().cpu().numpy())


def _check_attention(orc, rows, O, L, sel):
    Or, Lr, _ = orc.attend(rows, sel)
    err = np.abs(O.astype(np.float64) - Or)
    lerr = np.abs(L.astype(np.float64) - Lr)
    assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS and lerr.max() <= LSE_MAX_ABS, \
        (err.max(), err.mean(), lerr.max())


@pytest.mark.parametrize("mode", ["window", "sink"])
@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_static_selection_and_forward(moba, case, mode):
    N, Hq, Hkv, d, B, k = case
    w, q, kk, v, orc = _setup(case, seed=606)
    m = moba.ROUTE_WINDOW if mode == "window" else moba.ROUTE_SINK
    sel = moba.static_selection(1, N, Hq, B, k, m)
    o, lse = moba.forward_selected(q, kk, v, sel, B, k)
    torch.cuda.synchronize()
    rows = np.arange(N, dtype=np.int64)
    want = static_selection(w.cu, rows, B, k, mode)
    O, L, Sg = _gpu_rows(o, lse, sel, N)
    assert np.array_equal(Sg, np.broadcast_to(want[:, None, :], Sg.shape))
    _check_attention(orc, rows, O, L, Sg)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_minmax_gate_and_forward(moba, case):
    N, Hq, Hkv, d, B, k = case
    w, q, kk, v, orc = _setup(case, seed=707)
    sel = torch.full((1, Hq, N, k), -7, dtype=torch.int32, device="cuda")
    o, lse = moba.forward_minmax(q, kk, v, B, k, sel_out=sel)
    sel_g = moba.gate_minmax(q, kk, B, k)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_g)
    rows = np.arange(N, dtype=np.int64)
    O, L, Sg = _gpu_rows(o, lse, sel, N)
    _, _, own = local_block_info(w.cu, rows, B)
    check_selection_invariants(Sg, own, k)
    ref, margin, maxabs = orc.select_minmax(rows)
    differ = np.any(Sg != ref, axis=2)
    flagged = margin < FLAG_REL * maxabs
    assert not np.any(differ & ~flagged), np.argwhere(differ & ~flagged)[:3]
    _check_attention(orc, rows, O, L, Sg)


def test_forward_selected_with_the_gate_selection_equals_forward(moba):
    case = (4096, 8, 2, 128, 256, 5)
    N, Hq, Hkv, d, B, k = case
    _, q, kk, v, _ = _setup(case, seed=808)
    sel = torch.empty(1, Hq, N, k, dtype=torch.int32, device="cuda")
    o1, l1 = moba.forward(q, kk, v, B, k, sel_out=sel)
    o2, l2 = moba.forward_selected(q, kk, v, sel, B, k)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_forward_selected_flags_a_future_block(moba):
    case = (1024, 2, 1, 128, 256, 3)
    N, Hq, Hkv, d, B, k = case
    _, q, kk, v, _ = _setup(case, seed=909)
    sel = moba.static_selection(1, N, Hq, B, k, moba.ROUTE_WINDOW)
    sel[0, 0, 900, 0] = 3  # row 900 is in block 3: a past slot may not name it
    p = moba.make_params(1, N, Hq, Hkv, d, B, k)
    ws = moba.alloc_workspace(moba.workspace_size(p, 1))
    moba.forward_selected(q, kk, v, sel, B, k, ws=ws)
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == 6  # MOBA_ERR_DEVICE_CHECK


# ---------------------------------------------------------------- packed sequences
VARLEN_CASES = [
    # lengths, Hq, Hkv, d, B, k
    ([1500, 1, 0, 3000, 700], 4, 2, 128, 256, 4),
    ([300, 4100, 129], 4, 1, 64, 128, 3),
]
VIDS = ["v" + "_".join(map(str, c[0])) for c in VARLEN_CASES]


def _setup_varlen(case, seed):
    lengths, Hq, Hkv, d, B, k = case
    w = S.Workload("variant_v", lengths, Hq, Hkv, d, B, k, seed=seed, batch_mode=False)
    q, kk, v = S.make_qkv(w, "cuda")
    orc = Oracle(bf16_bits(q), bf16_bits(kk), bf16_bits(v), w.cu, Hq, Hkv, d, B, k)
    cu = torch.tensor(w.cu, dtype=torch.int32, device="cuda")
    return w, q, kk, v, cu, orc


def _gpu_rows_varlen(o, lse, sel):
    """o [T,H,d], lse [H,T], sel [H,T,k] -> [T,H,d], [T,H], [T,H,k]."""
    return (o.float().cpu().numpy(), lse.t().contiguous().cpu().numpy(),
            None if sel is None else sel.permute(1, 0, 2).contiguous().cpu().numpy())


@pytest.mark.parametrize("mode", ["window", "sink"])
@pytest.mark.parametrize("case", VARLEN_CASES, ids=VIDS)
def test_static_selection_and_forward_varlen(moba, case, mode):
    lengths, Hq, Hkv, d, B, k = case
    w, q, kk, v, cu, orc = _setup_varlen(case, seed=616)
    m = moba.ROUTE_WINDOW if mode == "window" else moba.ROUTE_SINK
    sel = moba.static_selection_varlen(cu, w.T, Hq, B, k, m)
    o, lse = moba.forward_selected_varlen(q, kk, v, cu, sel, B, k)
    torch.cuda.synchronize()
    rows = np.arange(w.T, dtype=np.int64)
    want = static_selection(w.cu, rows, B, k, mode)
    O, L, Sg = _gpu_rows_varlen(o, lse, sel)
    assert np.array_equal(Sg, np.broadcast_to(want[:, None, :], Sg.shape))
    _check_attention(orc, rows, O, L, Sg)


@pytest.mark.parametrize("case", VARLEN_CASES, ids=VIDS)
def test_minmax_gate_and_forward_varlen(moba, case):
    lengths, Hq, Hkv, d, B, k = case
    w, q, kk, v, cu, orc = _setup_varlen(case, seed=717)
    sel = torch.full((Hq, w.T, k), -7, dtype=torch.int32, device="cuda")
    o, lse = moba.forward_minmax_varlen(q, kk, v, cu, B, k, sel_out=sel)
    sel_g = moba.gate_minmax_varlen(q, kk, cu, B, k)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_g)
    rows = np.arange(w.T, dtype=np.int64)
    O, L, Sg = _gpu_rows_varlen(o, lse, sel)
    _, _, own = local_block_info(w.cu, rows, B)
    check_selection_invariants(Sg, own, k)
    ref, margin, maxabs = orc.select_minmax(rows)
    differ = np.any(Sg != ref, axis=2)
    flagged = margin < FLAG_REL * maxabs
    assert not np.any(differ & ~flagged), np.argwhere(differ & ~flagged)[:3]
    _check_attention(orc, rows, O, L, Sg)


def test_forward_selected_varlen_with_the_gate_selection_equals_forward_varlen(moba):
    case = ([2000, 900, 2500], 8, 2, 128, 256, 5)
    w, q, kk, v, cu, _ = _setup_varlen(case, seed=818)
    sel = torch.empty(8, w.T, 5, dtype=torch.int32, device="cuda")
    o1, l1 = moba.forward_varlen(q, kk, v, cu, 256, 5, sel_out=sel)
    o2, l2 = moba.forward_selected_varlen(q, kk, v, cu, sel, 256, 5)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
