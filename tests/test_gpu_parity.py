"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases compare every row; the five benchmark workloads compare the
seeded sample of query rows (all heads of each sampled row) in the launch
configuration the benchmark uses (binding defaults: workspace picked by
pick_heads_per_pass).  Tolerances and the flagged-row rule live in
parity_util.
"""
import os

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import Oracle, bf16_bits, local_block_info
from parity_util import (check_selection_invariants, compare, compare_dense,
                         gather_rows_packed)

pytestmark = pytest.mark.gpu

PARITY_ROWS = int(os.environ.get("MOBA_PARITY_ROWS", "4096"))


@pytest.fixture(scope="module")
def moba():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as m
    return m


def _run_forward(m, w, q, k, v):
    """Run the forward the way a user would; returns (o, lse, sel, ws)."""
    dev = q.device
    T = w.T
    varlen = not w.batch_mode or len(set(w.lengths)) > 1
    if varlen:
        cu = torch.tensor(w.cu, dtype=torch.int32, device=dev)
        p = m.make_params(1, 0, w.Hq, w.Hkv, w.d, w.B, w.k)
        hp = m.pick_heads_per_pass(lambda n: m.workspace_size_varlen(p, T, len(w.lengths), n),
                                   w.Hkv)
        ws = m.alloc_workspace(m.workspace_size_varlen(p, T, len(w.lengths), hp), dev)
        ws.zero_()
        sel = torch.full((w.Hq, T, w.k), -7, dtype=torch.int32, device=dev)
        o, lse = m.forward_varlen(q, k, v, cu, w.B, w.k, ws=ws, sel_out=sel)
    else:
        b, N = len(w.lengths), w.lengths[0]
        q4, k4, v4 = (x.view(b, N, x.shape[1], x.shape[2]) for x in (q, k, v))
        p = m.make_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
        hp = m.pick_heads_per_pass(lambda n: m.workspace_size(p, n), w.Hkv)
        ws = m.alloc_workspace(m.workspace_size(p, hp), dev)
        ws.zero_()
        sel = torch.full((b, w.Hq, N, w.k), -7, dtype=torch.int32, device=dev)
        o, lse = m.forward(q4, k4, v4, w.B, w.k, ws=ws, sel_out=sel)
    torch.cuda.synchronize()
    assert m.last_device_status(ws) == 0
    return o, lse, sel, varlen


def _check_forward(m, w, rows=None, label=""):
    q, k, v = S.make_qkv(w, "cuda")
    o, lse, sel, varlen = _run_forward(m, w, q, k, v)
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    if rows is None:
        rows = np.arange(w.T, dtype=np.int64)
    N = None if varlen else w.lengths[0]
    Og, Lg, Sg = gather_rows_packed(o, lse, sel, rows, w.Hq, varlen, N)
    _, _, own = local_block_info(w.cu, rows, w.B)
    check_selection_invariants(Sg, own, w.k)
    stats = compare(orc, rows, Og, Lg, Sg, label=label or w.name)
    return stats


SMALL = [
    # lengths, Hq, Hkv, d, B, k
    ([2048], 1, 1, 64, 256, 3),
    ([1000], 4, 1, 128, 128, 3),      # ragged N, GQA 4
    ([777], 8, 1, 64, 256, 2),        # GQA 8, d = 64, partial last block
    ([1536], 2, 2, 128, 512, 2),      # B = 512
    ([640], 4, 2, 128, 128, 1),       # k = 1: own block only
    ([900], 4, 2, 128, 128, 20),      # k > n: every block
    ([1280, 1280], 4, 2, 128, 256, 3),  # batch of 2
    ([129], 2, 1, 128, 128, 2),       # one row past the first block
    ([4096], 8, 2, 128, 128, 5),      # many blocks, top-k ranking
    ([32896], 2, 1, 128, 128, 6),     # 257 blocks: 256 past, the tensor-core gate's limit
    ([40000], 2, 1, 64, 128, 8),      # 313 blocks: beyond it, the SIMT gate
    ([4096], 4, 1, 128, 128, 17),     # k - 1 = 16: the last of the 256-block score tiles
    ([16384], 2, 1, 128, 128, 32),    # k - 1 = 31 of up to 127 past blocks (32-long lists)
    ([20000], 2, 1, 64, 128, 20),     # k - 1 = 19 beyond 128 past blocks: the SIMT gate's rows
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "x".join(map(str, c[0])) + "_%d_%d_%d_%d_%d" % c[1:])
def test_forward_small(moba, case):
    lengths, Hq, Hkv, d, B, k = case
    w = S.Workload("small", lengths, Hq, Hkv, d, B, k, seed=101)
    _check_forward(moba, w)


VARLEN_SMALL = [
    ([300, 1, 1024, 129, 640], 4, 2, 128, 128, 3),
    ([0, 513, 0, 1], 2, 1, 64, 256, 2),   # empty and one-token sequences
    ([2000, 700, 1500], 8, 2, 128, 256, 4),
    # one sequence of 258 blocks: its last tiles go to the SIMT gate, the rest
    # (and the other sequences) to the tensor-core gate, in one call
    ([300, 33024, 1000], 2, 1, 64, 128, 4),
]


@pytest.mark.parametrize("case", VARLEN_SMALL, ids=lambda c: "v" + "_".join(map(str, c[0])))
def test_forward_varlen_small(moba, case):
    lengths, Hq, Hkv, d, B, k = case
    w = S.Workload("varlen_small", lengths, Hq, Hkv, d, B, k, seed=202, batch_mode=False)
    _check_forward(moba, w)


DENSE_SMALL = [
    ([1], 1, 1, 64), ([127], 2, 1, 128), ([128], 1, 1, 128), ([300], 4, 2, 128),
    ([2000], 8, 2, 64), ([700, 700], 4, 1, 128),
]


@pytest.mark.parametrize("case", DENSE_SMALL, ids=lambda c: "d" + "_".join(map(str, c[0])) + "_%d_%d_%d" % c[1:])
def test_full_causal_small(moba, case):
    lengths, Hq, Hkv, d = case
    w = S.Workload("dense_small", lengths, Hq, Hkv, d, 128, 1, seed=303)
    q, k, v = S.make_qkv(w, "cuda")
    b, N = len(lengths), lengths[0]
    o, lse = moba.full_causal(*(x.view(b, N, x.shape[1], x.shape[2]) for x in (q, k, v)))
    torch.cuda.synchronize()
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, Hq, Hkv, d, 128, 1)
    rows = np.arange(w.T)
    Og, Lg, _ = gather_rows_packed(o, lse, None, rows, Hq, False, N)
    compare_dense(orc, rows, Og, Lg, label=str(case))


def test_full_causal_varlen_small(moba):
    w = S.Workload("dense_varlen", [5, 300, 1000, 0, 17], 4, 2, 128, 128, 1, seed=304,
                   batch_mode=False)
    q, k, v = S.make_qkv(w, "cuda")
    cu = torch.tensor(w.cu, dtype=torch.int32, device="cuda")
    o, lse = moba.full_causal_varlen(q, k, v, cu)
    torch.cuda.synchronize()
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, 4, 2, 128, 128, 1)
    rows = np.arange(w.T)
    Og, Lg, _ = gather_rows_packed(o, lse, None, rows, 4, True)
    compare_dense(orc, rows, Og, Lg, label="dense varlen")


def _half_ulp_bf16(x):
    """Half the spacing of bf16 numbers (8 significant bits) around |x|."""
    _, e = np.frexp(np.abs(x))
    return np.ldexp(1.0, e - 9)


@pytest.mark.parametrize("d", [128, 64])
def test_first_rows_of_a_block_round_once(moba, d):
    # Rows 0..63 of a block's first tile attend to 1..64 keys, too few for the
    # bf16 rounding of their softmax weights to average out.  The attention
    # gives them the residual weights as well, so their output is the exact
    # value rounded once to bf16: within half a bf16 step, plus 1e-4 for the
    # fp32 arithmetic.  Own block only (k = 1) and the dense kernel.
    N, Hq, Hkv, B = 2048, 4, 2, 256
    w = S.Workload("first_rows", [N], Hq, Hkv, d, B, 1, seed=707)
    q, k, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, N, x.shape[1], d) for x in (q, k, v))
    o1, _ = moba.forward(q4, k4, v4, B, 1)
    o2, _ = moba.full_causal(q4, k4, v4)
    torch.cuda.synchronize()
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, Hq, Hkv, d, B, 1)
    rows = np.array([t for t in range(N) if t % B < 64], dtype=np.int64)
    _, _, own = local_block_info(w.cu, rows, B)
    sel = np.ascontiguousarray(np.broadcast_to(own[:, None, None], (len(rows), Hq, 1)), np.int32)
    ref, _, _ = orc.attend(rows, sel)
    got = o1[0].float().cpu().numpy()[rows].astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= _half_ulp_bf16(ref) + 1e-4), err.max()
    dense_rows = rows[rows < 64]
    sel_all = np.zeros((len(dense_rows), Hq, 1), np.int32)  # block 0 holds every earlier key
    ref_d, _, _ = orc.attend(dense_rows, sel_all)
    got_d = o2[0].float().cpu().numpy()[dense_rows].astype(np.float64)
    err_d = np.abs(got_d - ref_d)
    assert np.all(err_d <= _half_ulp_bf16(ref_d) + 1e-4), err_d.max()


@pytest.mark.parametrize("scale", [65536.0, 1.0e6])
def test_routed_partials_beyond_fp16_range(moba, scale):
    """Routed partials are stored in fp16, scaled by a power of two derived
    from the largest |v| (1 below 2^15), so values past the fp16 maximum
    still give the exact attention.  Block 0's v is a constant `scale` (every
    row of block 1 routes there: its only past block), block 2's v is N(0,1)
    times `scale`; the other blocks are ordinary.  Bound per element: the
    prefill's 1e-2 plus 2^-7 of the largest |v| the row attends (the bf16
    weights, the fp16 partial and the bf16 output each round relative to it)."""
    N, Hq, Hkv, d, B, k = 2048, 2, 1, 128, 256, 3
    w = S.Workload("fp16_range", [N], Hq, Hkv, d, B, k, seed=111)
    q, kk, v = S.make_qkv(w, "cuda")
    v = v.clone()
    v[:B] = scale
    v[2 * B:3 * B] = (v[2 * B:3 * B].float() * scale).to(torch.bfloat16)
    q4, k4, v4 = (x.view(1, N, x.shape[1], d) for x in (q, kk, v))
    p = moba.make_params(1, N, Hq, Hkv, d, B, k)
    ws = moba.alloc_workspace(moba.workspace_size(p, 1))
    sel = torch.empty(1, Hq, N, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward(q4, k4, v4, B, k, ws=ws, sel_out=sel)
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == 0
    assert torch.isfinite(o.float()).all()
    orc = Oracle(bf16_bits(q), bf16_bits(kk), bf16_bits(v), w.cu, Hq, Hkv, d, B, k)
    rows = np.arange(N, dtype=np.int64)
    Og, Lg, Sg = gather_rows_packed(o, lse, sel, rows, Hq, False, N)
    ref, lref, _ = orc.attend(rows, Sg)
    vmax_blk = v.float().abs().view(N // B, B * Hkv * d).max(dim=1).values.cpu().numpy()
    m_row = np.where(Sg >= 0, vmax_blk[np.maximum(Sg, 0)], 0.0).max(axis=2)  # [R, H]
    err = np.abs(Og.astype(np.float64) - ref)
    bound = 1e-2 + 2.0 ** -7 * m_row[..., None]
    assert np.all(err <= bound), float((err / bound).max())
    assert np.abs(Lg - lref).max() <= 1e-3
    assert (Sg == 0).any()  # block 0 is routed to


def test_k_equal_n_matches_full_causal_kernel(moba):
    # the method with every block selected is full attention: both CUDA paths agree
    w = S.Workload("kn", [2048], 8, 2, 128, 256, 8, seed=404)
    q, k, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, 2048, x.shape[1], 128) for x in (q, k, v))
    o1, l1 = moba.forward(q4, k4, v4, 256, 8)
    o2, l2 = moba.full_causal(q4, k4, v4)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_heads_per_pass_does_not_change_results(moba):
    w = S.Workload("passes", [3000], 8, 4, 128, 256, 4, seed=505)
    q, k, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, 3000, x.shape[1], 128) for x in (q, k, v))
    p = moba.make_params(1, 3000, 8, 4, 128, 256, 4)
    outs = []
    for hp in (1, 3, 4):
        ws = moba.alloc_workspace(moba.workspace_size(p, hp))
        outs.append(moba.forward(q4, k4, v4, 256, 4, ws=ws))
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


def test_deterministic(moba):
    w = S.Workload("det", [4096], 8, 2, 128, 256, 4, seed=606)
    q, k, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, 4096, x.shape[1], 128) for x in (q, k, v))
    a = moba.forward(q4, k4, v4, 256, 4)
    b = moba.forward(q4, k4, v4, 256, 4)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_gate_only_matches_forward_selection(moba):
    w = S.Workload("gate", [4096], 8, 2, 128, 256, 5, seed=707)
    q, k, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, 4096, x.shape[1], 128) for x in (q, k, v))
    sel_f = torch.empty(1, 8, 4096, 5, dtype=torch.int32, device="cuda")
    moba.forward(q4, k4, v4, 256, 5, sel_out=sel_f)
    sel_g = moba.gate(q4, k4, 256, 5)
    torch.cuda.synchronize()
    assert torch.equal(sel_f, sel_g)


@pytest.mark.parametrize("mode,k", [("all_equal", 5), ("pairs_equal", 4)])
def test_gate_exact_ties(moba, mode, k):
    """Blocks with equal key means give exactly equal scores, so the tie rule
    (the lower block index wins) alone decides the kept set.  With every block
    equal, rows past 24 blocks take the many-ties path of the gate; with equal
    pairs, the cut falls inside a pair.  Checked exactly on every row against
    the oracle's selection, with no near-tie exemption."""
    N, Hq, Hkv, d, B = 4096, 4, 1, 128, 128
    w = S.Workload("ties", [N], Hq, Hkv, d, B, k, seed=909)
    q, kk, v = S.make_qkv(w, "cuda")
    kb = kk.view(N // B, B, Hkv, d)
    if mode == "all_equal":
        kb[1:] = kb[0:1].clone()
    else:
        kb[1::2] = kb[0::2].clone()
    sel = moba.gate(q.view(1, N, Hq, d), kk.view(1, N, Hkv, d), B, k)
    torch.cuda.synchronize()
    orc = Oracle(bf16_bits(q), bf16_bits(kk), bf16_bits(v), w.cu, Hq, Hkv, d, B, k)
    osel, _, _ = orc.select(np.arange(N, dtype=np.int64))
    gsel = sel[0].permute(1, 0, 2).cpu().numpy()
    assert np.array_equal(gsel, osel)


# ---------------------------------------------------------------- workloads
def test_workload_tiny_all_rows(moba):
    stats = _check_forward(moba, S.TINY)
    print("tiny", stats)


@pytest.mark.slow
@pytest.mark.timeout(3600)
@pytest.mark.parametrize("name", ["fine_32k", "long_128k", "long_128k_k32", "varlen_8seq",
                                  "prefill_1m"])
def test_workload_sampled_rows(moba, name):
    w = S.LONG_128K.with_k(32) if name == "long_128k_k32" else S.WORKLOADS[name]
    rows = S.sample_rows(w, PARITY_ROWS)
    stats = _check_forward(moba, w, rows=rows, label=name)
    print(name, stats)


@pytest.mark.slow
@pytest.mark.timeout(3600)
def test_workload_10m_shard_sampled_rows(moba):
    """One kv-head shard of the 10M-token setting (4 q heads, B = 40960), in
    the benchmark's launch configuration, on a seeded sample of rows."""
    w = S.PREFILL_10M_SHARD
    rows = S.sample_rows(w, max(64, PARITY_ROWS // 8))
    stats = _check_forward(moba, w, rows=rows, label=w.name)
    print(w.name, stats)


@pytest.mark.slow
@pytest.mark.timeout(3600)
@pytest.mark.parametrize("name", ["fine_32k", "long_128k"])
def test_workload_dense_sampled_rows(moba, name):
    w = S.WORKLOADS[name]
    q, k, v = S.make_qkv(w, "cuda")
    N = w.lengths[0]
    o, lse = moba.full_causal(*(x.view(1, N, x.shape[1], x.shape[2]) for x in (q, k, v)))
    torch.cuda.synchronize()
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    rows = S.sample_rows(w, 256, seed=99)
    Og, Lg, _ = gather_rows_packed(o, lse, None, rows, w.Hq, False, N)
    print(name, compare_dense(orc, rows, Og, Lg, label=name))


def test_forward_host_matches_forward(moba):
    """The host-buffer call (copies inside, pipelined by kv-head group) gives
    the device call's o, lse and selection bit for bit."""
    b, N, Hq, Hkv, d, B, k = 2, 4096, 8, 2, 128, 256, 4
    w = S.Workload("host", [N] * b, Hq, Hkv, d, B, k, seed=4242)
    q, kk, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(b, N, x.shape[1], d) for x in (q, kk, v))
    sel = torch.empty(b, Hq, N, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward(q4, k4, v4, B, k, sel_out=sel)
    pin = lambda x: x.cpu().pin_memory()
    qh, kh, vh = pin(q4), pin(k4), pin(v4)
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    sh = torch.empty(sel.shape, dtype=sel.dtype, pin_memory=True)
    p = moba.make_params(b, N, Hq, Hkv, d, B, k)
    buf = moba.alloc_workspace(moba.forward_host_buffer_size(p, 1))  # one kv head per pass
    moba.forward_host(qh, kh, vh, B, k, oh, lh, dev_buf=buf, sel_out=sh)
    torch.cuda.synchronize()
    assert moba.last_device_status(buf) == 0
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, lse.cpu()) and torch.equal(sh, sel.cpu())


def test_forward_host_varlen_matches_forward_varlen(moba):
    """The packed-sequence host-buffer call gives forward_varlen's o, lse and
    selection bit for bit (one kv head per pass, so the copies pipeline)."""
    lengths, Hq, Hkv, d, B, k = [3000, 1, 0, 2500, 700], 8, 2, 128, 256, 4
    w = S.Workload("host_varlen", lengths, Hq, Hkv, d, B, k, seed=4343, batch_mode=False)
    q, kk, v = S.make_qkv(w, "cuda")
    cu = torch.tensor(w.cu, dtype=torch.int32, device="cuda")
    sel = torch.empty(Hq, w.T, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward_varlen(q, kk, v, cu, B, k, sel_out=sel)
    pin = lambda x: x.cpu().pin_memory()
    qh, kh, vh = pin(q), pin(kk), pin(v)
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    sh = torch.empty(sel.shape, dtype=sel.dtype, pin_memory=True)
    p = moba.make_params(1, 0, Hq, Hkv, d, B, k)
    buf = moba.alloc_workspace(moba.forward_host_buffer_size_varlen(p, w.T, len(lengths), 1))
    moba.forward_host_varlen(qh, kh, vh, cu.cpu(), B, k, oh, lh, dev_buf=buf, sel_out=sh)
    torch.cuda.synchronize()
    assert moba.last_device_status(buf) == 0
    assert torch.equal(oh, o.cpu()) and torch.equal(lh, lse.cpu()) and torch.equal(sh, sel.cpu())
