"""Pins for the gate variants of the oracle: the min/max-pooled gate
(oracle_select_minmax) and the static window / sink routings
(static_selection).

The pages name Quest as MoBA with smaller blocks and min/max pooling
(elamur summary card, "Key points"); the block score is Quest's bound
s_j = sum_c max(q_c max_t k_tc, q_c min_t k_tc), the largest value of q . x
over the box spanned by block j's keys.  The tests tie the oracle to:
  * exhaustive subset search with exact rational scores (bruteforce.py),
    including integer inputs with many exact ties;
  * the bound itself: s_j >= q . k_t for every key t of block j, exactly;
  * one-token blocks, where the box is a point and the min/max gate must
    choose exactly what the mean gate chooses.
The static routings are tied to the pages' statement that sliding window
and sink attention are gates that always pick recent (and initial) blocks:
on keys built so that the mean gate must make exactly those choices, the
static rules and the gate agree on every row.
"""
from fractions import Fraction

import numpy as np
import pytest

import torch

from oracle import Oracle, bf16_bits, cu_from_lengths, static_selection
from oracle import bruteforce as bf
from test_oracle_pins import SMALL_CASES, _problem


@pytest.mark.parametrize("case", SMALL_CASES)
def test_minmax_selection_matches_bruteforce(case):
    lengths, Hq, Hkv, d, B, k = case
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=17)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    T = int(cu[-1])
    sel, _, _ = orc.select_minmax(np.arange(T))
    ref = bf.brute_select_minmax(bf.to_fractions(q), bf.to_fractions(kb), cu, Hq, Hkv, B, k)
    for t in range(T):
        for h in range(Hq):
            assert tuple(int(x) for x in sel[t, h] if x >= 0) == ref[t][h], (t, h)


def test_minmax_exact_ties_match_bruteforce():
    lengths, Hq, Hkv, d, B, k = [48], 2, 1, 3, 4, 4
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=5, ints=True)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    sel, margin, _ = orc.select_minmax(np.arange(48))
    ref = bf.brute_select_minmax(bf.to_fractions(q), bf.to_fractions(kb), cu, Hq, Hkv, B, k)
    for t in range(48):
        for h in range(Hq):
            assert tuple(int(x) for x in sel[t, h] if x >= 0) == ref[t][h]
    assert np.sum(margin == 0.0) > 5  # ties really occur


def test_minmax_score_bounds_every_key_exactly():
    lengths, Hq, Hkv, d, B, k = [24], 2, 1, 4, 6, 2
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=9)
    qf, kf = bf.to_fractions(q), bf.to_fractions(kb)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    kx, kn = orc.block_minmax()
    for j in range(4):
        for c in range(d):  # the oracle's pooled values are the exact extremes
            col = [kf[t, 0, c] for t in range(j * B, (j + 1) * B)]
            assert Fraction(kx[0, j, c]) == max(col) and Fraction(kn[0, j, c]) == min(col)
        for t in range(24):
            for h in range(Hq):
                s = sum(max(qf[t, h, c] * max(kf[u, 0, c] for u in range(j * B, (j + 1) * B)),
                            qf[t, h, c] * min(kf[u, 0, c] for u in range(j * B, (j + 1) * B)))
                        for c in range(d))
                for u in range(j * B, (j + 1) * B):
                    assert s >= sum(qf[t, h, c] * kf[u, 0, c] for c in range(d))


def test_one_token_blocks_minmax_equals_mean_gate():
    lengths, Hq, Hkv, d, B, k = [40], 2, 1, 4, 1, 5
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=23)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    rows = np.arange(40)
    a, ma, xa = orc.select(rows)
    b, mb, xb = orc.select_minmax(rows)
    assert np.array_equal(a, b)
    np.testing.assert_allclose(mb, ma, rtol=0, atol=1e-12)


def test_minmax_score_is_a_dot_product_of_sign_split_queries():
    # max(q_c M_c, q_c m_c) = max(q_c, 0) M_c + min(q_c, 0) m_c since M_c >= m_c:
    # the min/max score is q+ . M + q- . m, two plain matrix products.  The
    # oracle's selection must be the top-(k-1) of those scores (ties to the
    # lower block) on every row whose (k-1)-th / k-th gap is not a rounding
    # tie, at a size brute force cannot reach.
    lengths, Hq, Hkv, d, B, k = [4096], 4, 2, 32, 64, 6
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=31)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    kx, kn = orc.block_minmax()
    qf = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double().numpy()  # exact
    rows = np.arange(0, 4096, 7)
    sel, _, _ = orc.select_minmax(rows)
    G = Hq // Hkv
    checked = 0
    for a, t in enumerate(rows):
        i = t // B
        if i == 0:
            continue
        for h in range(Hq):
            g = h // G
            qp, qn = np.maximum(qf[t, h], 0.0), np.minimum(qf[t, h], 0.0)
            s = kx[g, :i] @ qp + kn[g, :i] @ qn
            order = sorted(range(i), key=lambda j: (-s[j], j))
            npast = min(k - 1, i)
            if npast < i and abs(s[order[npast - 1]] - s[order[npast]]) < 1e-9 * np.abs(s).max():
                continue
            want = sorted(order[:npast]) + [i]
            got = [int(x) for x in sel[a, h] if x >= 0]
            assert got == want, (t, h)
            checked += 1
    assert checked > 1500


def _tb(a):
    return bf16_bits(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))


def test_window_rule_is_the_gate_on_recency_ordered_blocks():
    # block means j * u grow along u and every query points along u: the mean
    # gate must pick the most recent blocks
    B, d, k, nblk = 8, 4, 3, 10
    T = B * nblk
    gen = torch.Generator().manual_seed(21)
    u = np.array([1.0, 0.0, 0.0, 0.0])
    kk = np.zeros((T, 1, d))
    for j in range(nblk):
        w = torch.randint(-2, 3, (B // 2, d), generator=gen).numpy().astype(np.float64)
        w[:, 0] = 0
        kk[j * B:(j + 1) * B, 0] = np.concatenate([w, -w]) + j * u
    q = (torch.randint(1, 4, (T, 1, 1), generator=gen).numpy() * u).astype(np.float32)
    cu = cu_from_lengths([T])
    orc = Oracle(_tb(q), _tb(kk), _tb(kk), cu, 1, 1, d, B, k)
    rows = np.arange(T)
    sel, _, _ = orc.select(rows)
    assert np.array_equal(sel[:, 0], static_selection(cu, rows, B, k, "window"))


def test_sink_rule_is_the_gate_on_a_dominant_first_block():
    B, d, k, nblk = 4, 2, 4, 9
    T = B * nblk
    kk = np.zeros((T, 1, d), dtype=np.float32)
    for j in range(nblk):
        kk[j * B:(j + 1) * B, 0, 0] = 100.0 if j == 0 else float(j)
    q = np.tile(np.array([1.0, 0.0], dtype=np.float32), (T, 1, 1))
    cu = cu_from_lengths([T])
    orc = Oracle(_tb(q), _tb(kk), _tb(kk), cu, 1, 1, d, B, k)
    rows = np.arange(T)
    sel, _, _ = orc.select(rows)
    assert np.array_equal(sel[:, 0], static_selection(cu, rows, B, k, "sink"))


def test_static_rules_keep_all_blocks_when_few_and_respect_sequences():
    cu = cu_from_lengths([10, 3, 17])
    rows = np.arange(30)
    for mode in ("window", "sink"):
        sel = static_selection(cu, rows, 4, 3, mode)
        for r, t in enumerate(rows):
            s = int(np.searchsorted(cu, t, side="right") - 1)
            i = (t - cu[s]) // 4
            got = [x for x in sel[r] if x >= 0]
            assert got[-1] == i and len(got) == min(3, i + 1) and got == sorted(set(got))
            if i + 1 <= 3:
                assert got == list(range(i + 1))
