"""Parity of the decode step (moba_decode, moba_kbar_cache_update) with the
fp64 oracle.

A decode step for a sequence of length L is the prefill's row L-1: the same
routing and causality rules and the same attention over the chosen blocks,
computed against a KV cache.  So the oracle's forward on the last row of
each sequence is the expected result; every test compares every (sequence,
q head) it runs, with the same tolerances and near-tie rule as the prefill.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import Oracle, bf16_bits, local_block_info
from parity_util import check_selection_invariants, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moba():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as m
    return m


def _caches(w, q, k, v, cap):
    """Pad the packed sequences of `w` into [b, cap, H, d] caches; the decode
    query of each sequence is its last token's."""
    b = len(w.lengths)
    kc = torch.zeros(b, cap, k.shape[1], w.d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    qd = torch.empty(b, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    for s, L in enumerate(w.lengths):
        c0 = int(w.cu[s])
        kc[s, :L] = k[c0:c0 + L]
        vc[s, :L] = v[c0:c0 + L]
        qd[s] = q[c0 + L - 1]
    lens = torch.tensor(w.lengths, dtype=torch.int32, device="cuda")
    return qd, kc, vc, lens


def _check_decode(m, w, cap=None):
    q, k, v = S.make_qkv(w, "cuda")
    cap = cap or max(w.lengths)
    qd, kc, vc, lens = _caches(w, q, k, v, cap)
    kbar = m.alloc_kbar_cache(kc, w.B)
    p = m.make_decode_params(len(w.lengths), cap, w.Hq, w.Hkv, w.d, w.B, w.k)
    ws = m.alloc_workspace(m.decode_workspace_size(p))
    ws.zero_()
    m.kbar_cache_update(kc, lens, kbar, w.B, ws=ws)
    sel = torch.full((len(w.lengths), w.Hq, w.k), -7, dtype=torch.int32, device="cuda")
    o, lse = m.decode(qd, kc, vc, lens, kbar, w.B, w.k, ws=ws, sel_out=sel)
    torch.cuda.synchronize()
    assert m.last_device_status(ws) == 0
    rows = np.array([w.cu[s] + L - 1 for s, L in enumerate(w.lengths)], dtype=np.int64)
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    Sg = sel.cpu().numpy()
    _, _, own = local_block_info(w.cu, rows, w.B)
    check_selection_invariants(Sg, own, w.k)
    return compare(orc, rows, o.float().cpu().numpy(), lse.cpu().numpy(), Sg, label=w.name)


DECODE_CASES = [
    # lengths, Hq, Hkv, d, B, k
    ([4096], 8, 2, 128, 256, 4),                       # one sequence, block-aligned end
    ([4097, 1, 4095, 2048, 3000], 8, 2, 128, 256, 3),  # ragged: new block, 1 token, ...
    ([1000, 129, 640], 4, 1, 64, 128, 2),              # d = 64, GQA 4
    ([5000, 700], 4, 2, 128, 512, 20),                 # k beyond the blocks: all kept
    ([3000, 2500], 4, 2, 128, 256, 1),                 # k = 1: own block only
    ([40000], 8, 2, 128, 128, 12),                     # many blocks ranked
]


@pytest.mark.parametrize("case", DECODE_CASES,
                         ids=lambda c: "x".join(map(str, c[0])) + "_%d_%d_%d_%d_%d" % c[1:])
def test_decode_small(moba, case):
    lengths, Hq, Hkv, d, B, k = case
    w = S.Workload("decode", lengths, Hq, Hkv, d, B, k, seed=303, batch_mode=False)
    stats = _check_decode(moba, w)
    print(case, stats)


def test_decode_cache_capacity_beyond_lengths(moba):
    w = S.Workload("decode_cap", [2000, 1500], 4, 2, 128, 256, 3, seed=304, batch_mode=False)
    _check_decode(moba, w, cap=4096)


def test_kbar_cache_matches_block_means(moba):
    w = S.Workload("kbar", [3000, 1024, 77], 4, 2, 128, 256, 3, seed=305, batch_mode=False)
    q, k, v = S.make_qkv(w, "cuda")
    cap = 3072
    _, kc, _, lens = _caches(w, q, k, v, cap)
    kbar = moba.alloc_kbar_cache(kc, w.B)
    moba.kbar_cache_update(kc, lens, kbar, w.B)
    torch.cuda.synchronize()
    orc = Oracle(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    ref = orc.block_means()  # [Hkv][global block][d], blocks numbered sequence by sequence
    got = kbar.cpu().numpy()
    J0 = 0
    for s, L in enumerate(w.lengths):
        nb = (L + w.B - 1) // w.B
        for j in range(L // w.B):  # complete blocks only
            np.testing.assert_allclose(got[s, :, j, :], ref[:, J0 + j, :], rtol=0, atol=1e-5)
        for j in range(L // w.B, got.shape[2]):  # never written
            assert not np.any(got[s, :, j, :])
        J0 += nb


def test_kbar_only_last_equals_full_rebuild(moba):
    B = 256
    w = S.Workload("kbar_last", [2 * B, 3 * B + 5], 4, 2, 128, B, 3, seed=306, batch_mode=False)
    q, k, v = S.make_qkv(w, "cuda")
    _, kc, _, lens = _caches(w, q, k, v, 4 * B)
    full = moba.alloc_kbar_cache(kc, B)
    moba.kbar_cache_update(kc, lens, full, B)
    inc = moba.alloc_kbar_cache(kc, B)
    # grow each cache token by token from 1 and update the completed block only
    for L in range(1, max(w.lengths) + 1):
        cur = torch.tensor([min(L, n) for n in w.lengths], dtype=torch.int32, device="cuda")
        moba.kbar_cache_update(kc, cur, inc, B, only_last=True)
    torch.cuda.synchronize()
    assert torch.equal(full, inc)


@pytest.mark.slow
@pytest.mark.timeout(1800)
def test_decode_prefill_1m(moba):
    """The decode step at the 1M-token configuration the benchmark times."""
    w = S.MILLION
    stats = _check_decode(moba, w)
    print("decode 1m", stats)
