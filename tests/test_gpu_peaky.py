"""Parity on peaky rows: inputs built so that the attention kernels' running
maximum jumps after the first key tile, which is the only place their output
accumulator is rescaled (the exact softmax over the selected set must hold
however the scores are spread: wispaper.ai blog, "The Change").

Two constructions:
  * planted keys (synthetic.make_peaky_qkv): in every block, two keys of
    tile 1 (and of tile 3 where the block has one) carry c * u with c = 24
    (48), and the even q heads carry 6 * u.  For d = 128 a planted key scores
    about 6 * 24 / sqrt(128) * log2(e) = 18 log2 units above an ordinary one
    (twice that for c = 48), against a spread of the ordinary scores of
    about 1.6 log2 units, so the jump exceeds the rescale threshold (8) in
    the routed span of every past block, in the own block of rows past its
    first plant and in the dense span past block 0's plants;
  * queries scaled by 16 (exact in bf16) on the ordinary inputs: scores
    spread over ~26 log2 units, so a later tile's maximum often clears the
    threshold.
tests/rescale_util.py replays the kernels' rescale rule in fp64 on the very
inputs of each test, and each test asserts the share of rows on which it
fires before comparing.  v is scaled by 1/4 (exactly) in both constructions:
near one-hot rows output nearly a single v row, and for |v| >= 4 the final
bf16 rounding alone (half a step, up to 2^-6) would exceed the 1e-2 bound.
The bounds are the prefill's (parity_util); the backward keeps its own.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import Oracle, bf16_bits, local_block_info
from parity_util import check_selection_invariants, compare, compare_dense, gather_rows_packed
from rescale_util import rescale_events

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moba():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as m
    return m


def _scaled_q_inputs(w):
    q, k, v = S.make_qkv(w, "cuda")
    return (q.float() * 16).to(torch.bfloat16), k, (v.float() * 0.25).to(torch.bfloat16)


def _inputs(w, kind, plants):
    if kind == "planted":
        return S.make_peaky_qkv(w, "cuda", plants=plants)
    return _scaled_q_inputs(w)


def _forward(m, w, q, k, v):
    T = w.T
    if not w.batch_mode:
        cu = torch.tensor(w.cu, dtype=torch.int32, device="cuda")
        sel = torch.full((w.Hq, T, w.k), -7, dtype=torch.int32, device="cuda")
        p = m.make_params(1, 0, w.Hq, w.Hkv, w.d, w.B, w.k)
        ws = m.alloc_workspace(m.workspace_size_varlen(p, T, len(w.lengths), 0))
        o, lse = m.forward_varlen(q, k, v, cu, w.B, w.k, ws=ws, sel_out=sel)
    else:
        b, N = len(w.lengths), w.lengths[0]
        q4, k4, v4 = (x.view(b, N, x.shape[1], w.d) for x in (q, k, v))
        sel = torch.full((b, w.Hq, N, w.k), -7, dtype=torch.int32, device="cuda")
        p = m.make_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
        ws = m.alloc_workspace(m.workspace_size(p, 0))
        o, lse = m.forward(q4, k4, v4, w.B, w.k, ws=ws, sel_out=sel)
    torch.cuda.synchronize()
    assert m.last_device_status(ws) == 0
    return o, lse, sel


FORWARD_CASES = [
    # name, lengths, Hq, Hkv, d, B, k, input kind, plants
    ("planted_b512", [4096], 4, 2, 128, 512, 3, "planted", ((1, 24.0), (3, 48.0))),
    ("planted_b256_d64", [2048], 4, 1, 64, 256, 4, "planted", ((1, 24.0),)),
    ("planted_varlen", [1500, 700, 2300], 4, 2, 128, 512, 3, "planted", ((1, 24.0), (3, 48.0))),
    ("q_x16_b512", [4096], 4, 2, 128, 512, 3, "scaled_q", None),
    ("q_x16_b256_d64", [2048], 4, 1, 64, 256, 4, "scaled_q", None),
]

# least share of (row, head) pairs on which the replayed rule must fire, per span
MIN_SHARE = {"planted": (0.3, 0.1, 0.3), "scaled_q": (0.2, 0.03, 0.3)}


@pytest.mark.parametrize("case", FORWARD_CASES, ids=[c[0] for c in FORWARD_CASES])
def test_peaky_forward_matches_oracle(moba, case):
    name, lengths, Hq, Hkv, d, B, k, kind, plants = case
    w = S.Workload(name, lengths, Hq, Hkv, d, B, k, seed=3131,
                   batch_mode=len(set(lengths)) == 1)
    q, kk, v = _inputs(w, kind, plants)
    o, lse, sel = _forward(moba, w, q, kk, v)
    qb, kb, vb = bf16_bits(q), bf16_bits(kk), bf16_bits(v)
    orc = Oracle(qb, kb, vb, w.cu, Hq, Hkv, d, B, k)
    rows = np.arange(w.T, dtype=np.int64)
    N = None if not w.batch_mode else lengths[0]
    Og, Lg, Sg = gather_rows_packed(o, lse, sel, rows, Hq, not w.batch_mode, N)
    _, _, own = local_block_info(w.cu, rows, B)
    check_selection_invariants(Sg, own, k)
    ev_routed, ev_own = rescale_events(qb, kb, w.cu, rows, Hq, Hkv, d, B, sel=Sg)
    lo_r, lo_o, _ = MIN_SHARE[kind]
    assert (ev_routed > 0).mean() >= lo_r, (ev_routed > 0).mean()
    assert (ev_own > 0).mean() >= lo_o, (ev_own > 0).mean()
    stats = compare(orc, rows, Og, Lg, Sg, label=name)
    print(name, stats, "rescaled rows: routed %.3f own %.3f" % ((ev_routed > 0).mean(),
                                                                (ev_own > 0).mean()))


DENSE_CASES = [
    ("planted_dense", [2048], 4, 2, 128, "planted"),
    ("planted_dense_varlen", [700, 1900], 4, 1, 64, "planted"),
    ("q_x16_dense", [2048], 4, 2, 128, "scaled_q"),
]


@pytest.mark.parametrize("case", DENSE_CASES, ids=[c[0] for c in DENSE_CASES])
def test_peaky_full_causal_matches_oracle(moba, case):
    name, lengths, Hq, Hkv, d, kind = case
    B = 512
    w = S.Workload(name, lengths, Hq, Hkv, d, B, 1, seed=3232,
                   batch_mode=len(set(lengths)) == 1)
    q, kk, v = _inputs(w, kind, ((1, 24.0), (3, 48.0)))
    if w.batch_mode:
        b, N = len(lengths), lengths[0]
        o, lse = moba.full_causal(*(x.view(b, N, x.shape[1], d) for x in (q, kk, v)))
    else:
        cu = torch.tensor(w.cu, dtype=torch.int32, device="cuda")
        o, lse = moba.full_causal_varlen(q, kk, v, cu)
    torch.cuda.synchronize()
    qb, kb, vb = bf16_bits(q), bf16_bits(kk), bf16_bits(v)
    rows = np.arange(w.T, dtype=np.int64)
    ev, _ = rescale_events(qb, kb, w.cu, rows, Hq, Hkv, d, B, dense=True)
    assert (ev > 0).mean() >= MIN_SHARE[kind][2], (ev > 0).mean()
    orc = Oracle(qb, kb, vb, w.cu, Hq, Hkv, d, B, 1)
    Og, Lg, _ = gather_rows_packed(o, lse, None, rows, Hq, not w.batch_mode,
                                   lengths[0] if w.batch_mode else None)
    print(name, compare_dense(orc, rows, Og, Lg, label=name), "rescaled rows %.3f" % (ev > 0).mean())


def test_peaky_decode_matches_oracle(moba):
    """The decode step's online softmax over planted keys: the new token's
    scores jump by far more than any threshold within its chosen blocks."""
    from test_gpu_decode import _caches
    w = S.Workload("peaky_decode", [4096, 3001, 700, 2048], 8, 2, 128, 512, 3, seed=3333,
                   batch_mode=False)
    q, k, v = S.make_peaky_qkv(w, "cuda")
    cap = max(w.lengths)
    qd, kc, vc, lens = _caches(w, q, k, v, cap)
    kbar = moba.alloc_kbar_cache(kc, w.B)
    p = moba.make_decode_params(len(w.lengths), cap, w.Hq, w.Hkv, w.d, w.B, w.k)
    ws = moba.alloc_workspace(moba.decode_workspace_size(p))
    moba.kbar_cache_update(kc, lens, kbar, w.B, ws=ws)
    sel = torch.full((len(w.lengths), w.Hq, w.k), -7, dtype=torch.int32, device="cuda")
    o, lse = moba.decode(qd, kc, vc, lens, kbar, w.B, w.k, ws=ws, sel_out=sel)
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == 0
    rows = np.array([w.cu[s] + L - 1 for s, L in enumerate(w.lengths)], dtype=np.int64)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    Sg = sel.cpu().numpy()
    ev_r, ev_o = rescale_events(qb, kb, w.cu, rows, w.Hq, w.Hkv, w.d, w.B, sel=Sg)
    assert ((ev_r + ev_o) > 0).mean() >= 0.3
    orc = Oracle(qb, kb, vb, w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    _, _, own = local_block_info(w.cu, rows, w.B)
    check_selection_invariants(Sg, own, w.k)
    print(compare(orc, rows, o.float().cpu().numpy(), lse.cpu().numpy(), Sg, label=w.name))


@pytest.mark.parametrize("kind", ["planted", "scaled_q"])
def test_peaky_backward_matches_oracle(moba, kind):
    """The backward recomputes P = 2^(z - lse2) from the forward's lse: on
    peaky rows lse is dominated by one planted key, and any error in it would
    scale every weight of the row."""
    from test_gpu_backward import MAX_REL, MEAN_REL
    N, Hq, Hkv, d, B, k = 2048, 4, 2, 128, 512, 3
    w = S.Workload("peaky_bw", [N], Hq, Hkv, d, B, k, seed=3434)
    q, kk, v = _inputs(w, kind, ((1, 24.0), (3, 48.0)))
    q4, k4, v4 = (x.view(1, N, x.shape[1], d) for x in (q, kk, v))
    sel = torch.empty(1, Hq, N, k, dtype=torch.int32, device="cuda")
    o, lse = moba.forward(q4, k4, v4, B, k, sel_out=sel)
    g = torch.Generator(device="cuda").manual_seed(78)
    dO = torch.randn(1, N, Hq, d, generator=g, device="cuda").to(torch.bfloat16)
    p = moba.make_params(1, N, Hq, Hkv, d, B, k)
    ws = moba.alloc_workspace(moba.backward_workspace_size(p, 0))
    dq, dk, dv = moba.backward(q4, k4, v4, o, lse, dO, sel, B, k, ws=ws)
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == 0
    qb, kb, vb = bf16_bits(q), bf16_bits(kk), bf16_bits(v)
    orc = Oracle(qb, kb, vb, w.cu, Hq, Hkv, d, B, k)
    rows = np.arange(N, dtype=np.int64)
    sel_rows = sel[0].permute(1, 0, 2).contiguous().cpu().numpy()
    ev_r, ev_o = rescale_events(qb, kb, w.cu, rows, Hq, Hkv, d, B, sel=sel_rows)
    assert ((ev_r + ev_o) > 0).mean() >= 0.2
    rq, rk, rv = orc.attend_backward(rows, sel_rows, bf16_bits(dO[0]))
    for name, got, ref in (("dq", dq[0], rq), ("dk", dk[0], rk), ("dv", dv[0], rv)):
        got = got.float().cpu().numpy().astype(np.float64)
        scale = np.abs(ref).max()
        err = np.abs(got - ref)
        assert err.max() <= MAX_REL * scale, (kind, name, err.max(), scale)
        assert err.mean() <= MEAN_REL * scale, (kind, name, err.mean(), scale)
