"""Pins of the fp64 oracle against what the pages and the mathematics fix.

CPU only.  Each test would fail for a plausible slip in the oracle: a dropped
own block, a future block let through, a wrong tie rule, a missing scale, an
off-by-one in the causal bound, a transposed operand or a wrong merge.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import Oracle, bf16_bits, cu_from_lengths, local_block_info, online_softmax_merge
from oracle import bruteforce as bf
from oracle.oracle import bits_to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_bits(shape, gen, scale=1.0, ints=False):
    if ints:
        x = torch.randint(-3, 4, shape, generator=gen).to(torch.float32)
    else:
        x = torch.randn(shape, generator=gen) * scale
    return bf16_bits(x.to(torch.bfloat16))


def _problem(lengths, Hq, Hkv, d, B, k, seed, ints=False, block_offset=0.5):
    gen = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    q = _rand_bits((T, Hq, d), gen, ints=ints)
    kk = torch.randn((T, Hkv, d), generator=gen) if not ints else \
        torch.randint(-3, 4, (T, Hkv, d), generator=gen).to(torch.float32)
    # per-block offset so that block means differ
    cu = cu_from_lengths(lengths)
    _, _, blk = local_block_info(cu, np.arange(T), B)
    seq, _, _ = local_block_info(cu, np.arange(T), B)
    key = seq * 100000 + blk
    uniq, inv = np.unique(key, return_inverse=True)
    if not ints:
        offs = torch.randn((len(uniq), Hkv, d), generator=gen) * block_offset
        kk = kk + offs[torch.from_numpy(inv)]
    k_bits = bf16_bits(kk.to(torch.bfloat16))
    v = _rand_bits((T, Hkv, d), gen)
    return q, k_bits, v, cu


SMALL_CASES = [
    # lengths, Hq, Hkv, d, B, k
    ([32], 1, 1, 4, 4, 3),
    ([29], 2, 1, 3, 4, 2),       # partial last block, GQA 2
    ([40], 4, 2, 4, 8, 3),       # GQA 2, two kv heads
    ([17, 23], 2, 2, 4, 4, 4),   # varlen, partial blocks
    ([24], 1, 1, 5, 4, 1),       # k = 1
    ([20], 1, 1, 4, 4, 9),       # k > n: every block
    ([1, 9, 4], 2, 1, 3, 4, 2),  # one-token sequence
]


@pytest.mark.parametrize("case", SMALL_CASES)
def test_selection_matches_bruteforce(case):
    lengths, Hq, Hkv, d, B, k = case
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=11)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    T = int(cu[-1])
    rows = np.arange(T)
    sel, margin, maxabs = orc.select(rows)
    ref = bf.brute_select(bf.to_fractions(q), bf.to_fractions(kb), cu, Hq, Hkv, B, k)
    for t in range(T):
        for h in range(Hq):
            got = tuple(int(x) for x in sel[t, h] if x >= 0)
            assert got == ref[t][h], (t, h, got, ref[t][h])


def test_exact_ties_go_to_lower_index():
    # Integer-valued inputs give exactly equal block scores; the oracle must
    # break them toward the lower block index, as brute force does exactly.
    lengths, Hq, Hkv, d, B, k = [64], 2, 1, 2, 4, 4
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=3, ints=True)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    rows = np.arange(64)
    sel, _, _ = orc.select(rows)
    ref = bf.brute_select(bf.to_fractions(q), bf.to_fractions(kb), cu, Hq, Hkv, B, k)
    n_tied = 0
    kbar = orc.block_means()
    for t in rows:
        i = t // B
        for h in range(Hq):
            got = tuple(int(x) for x in sel[t, h] if x >= 0)
            assert got == ref[t][h]
            s = bits_to_f64(q[t, h]) @ kbar[0, :i].T if i else np.zeros(0)
            n_tied += int(len(s) != len(np.unique(s)))
    assert n_tied > 10  # the case really exercises ties


def test_constructed_tie_prefers_lower_block():
    # Two identical past blocks and one weaker one, k = 2: block 0 must win.
    B, d = 4, 2
    T = 4 * B
    kk = np.zeros((T, 1, d), dtype=np.float32)
    kk[0:4, 0] = [1, 0]
    kk[4:8, 0] = [1, 0]
    kk[8:12, 0] = [0.5, 0]
    q = np.tile(np.array([1, 0], dtype=np.float32), (T, 1, 1))
    tb = lambda a: bf16_bits(torch.from_numpy(a).to(torch.bfloat16))
    orc = Oracle(tb(q), tb(kk), tb(kk), cu_from_lengths([T]), 1, 1, d, B, 2)
    sel, margin, _ = orc.select(np.array([13]))
    assert list(sel[0, 0]) == [0, 3]
    assert margin[0, 0] == 0.0  # the tie sits exactly at the selection boundary


@pytest.mark.parametrize("case", SMALL_CASES)
def test_attention_matches_explicit_mask(case):
    lengths, Hq, Hkv, d, B, k = case
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=5)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    T = int(cu[-1])
    rows = np.arange(T)
    O, lse, sel, _, _ = orc.forward(rows)
    ref_sel = bf.brute_select(bf.to_fractions(q), bf.to_fractions(kb), cu, Hq, Hkv, B, k)
    G = Hq // Hkv
    qf, kf, vf = bits_to_f64(q), bits_to_f64(kb), bits_to_f64(v)
    for h in range(Hq):
        M = bf.mask_from_selection([ref_sel[t][h] for t in range(T)], cu, B, T)
        Oref, lref = bf.masked_attention(qf[:, h], kf[:, h // G], vf[:, h // G], M,
                                         1.0 / math.sqrt(d))
        np.testing.assert_allclose(O[:, h], Oref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], lref, rtol=1e-12, atol=1e-12)


def _sdpa(qf, kf, vf, mask, scale):
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (qf, kf, vf))
    O = torch.nn.functional.scaled_dot_product_attention(
        qt[None, None], kt[None, None], vt[None, None], attn_mask=torch.from_numpy(mask)[None, None],
        scale=scale)[0, 0].numpy()
    z = np.where(mask, (qf @ kf.T) * scale, -np.inf)
    return O, logsumexp(z, axis=1)


@pytest.mark.parametrize("lengths,B", [([96], 16), ([70, 33], 16)])
def test_k_equal_n_is_full_causal_attention(lengths, B):
    Hq, Hkv, d = 4, 2, 8
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, 1, seed=7)
    T = int(cu[-1])
    nmax = max((L + B - 1) // B for L in lengths)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, nmax)
    rows = np.arange(T)
    O, lse, sel, _, _ = orc.forward(rows)
    Od, lsed = orc.dense(rows)
    np.testing.assert_allclose(O, Od, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lsed, rtol=1e-12, atol=1e-13)
    # and against torch's SDPA with a plain causal (per-sequence) mask
    seq, _, _ = local_block_info(cu, rows, B)
    mask = (rows[:, None] >= rows[None, :]) & (seq[:, None] == seq[None, :])
    qf, kf, vf = bits_to_f64(q), bits_to_f64(kb), bits_to_f64(v)
    for h in range(Hq):
        Oref, lref = _sdpa(qf[:, h], kf[:, h // 2], vf[:, h // 2], mask, 1 / math.sqrt(d))
        np.testing.assert_allclose(O[:, h], Oref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], lref, rtol=1e-12, atol=1e-12)


def test_k_one_is_block_diagonal_causal():
    lengths, Hq, Hkv, d, B = [100], 2, 1, 8, 16
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, 1, seed=9)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, 1)
    rows = np.arange(100)
    O, lse, sel, margin, _ = orc.forward(rows)
    assert np.all(sel[:, :, 0] == (rows // B)[:, None])
    assert np.all(np.isinf(margin))
    blk = rows // B
    mask = (rows[:, None] >= rows[None, :]) & (blk[:, None] == blk[None, :])
    qf, kf, vf = bits_to_f64(q), bits_to_f64(kb), bits_to_f64(v)
    for h in range(Hq):
        Oref, lref = _sdpa(qf[:, h], kf[:, 0], vf[:, 0], mask, 1 / math.sqrt(d))
        np.testing.assert_allclose(O[:, h], Oref, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], lref, rtol=1e-12, atol=1e-12)


def test_sliding_window_special_case():
    # Block means c*j*u grow along u and every query points along u, so the
    # gate must pick the most recent blocks: a sliding window of k blocks.
    B, d, k, nblk = 8, 4, 3, 10
    T = B * nblk
    gen = torch.Generator().manual_seed(21)
    u = np.array([1.0, 0.0, 0.0, 0.0])
    kk = np.zeros((T, 1, d))
    for j in range(nblk):
        # zero-mean pairs inside each block keep the block mean at j*u exactly
        w = torch.randint(-2, 3, (B // 2, d), generator=gen).numpy().astype(np.float64)
        w[:, 0] = 0
        kk[j * B:(j + 1) * B, 0] = np.concatenate([w, -w]) + j * u
    q = (torch.randint(1, 4, (T, 1, 1), generator=gen).numpy() * u).astype(np.float32)
    v = torch.randn(T, 1, d, generator=gen).to(torch.bfloat16)
    tb = lambda a: bf16_bits(torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16))
    orc = Oracle(tb(q), tb(kk), bf16_bits(v), cu_from_lengths([T]), 1, 1, d, B, k)
    rows = np.arange(T)
    O, lse, sel, _, _ = orc.forward(rows)
    for t in rows:
        i = t // B
        want = list(range(max(0, i - k + 1), i + 1))
        assert [x for x in sel[t, 0] if x >= 0] == want
    lo = np.maximum(0, (rows // B) - k + 1) * B
    mask = (rows[None, :] <= rows[:, None]) & (rows[None, :] >= lo[:, None])
    Oref, lref = _sdpa(bits_to_f64(tb(q))[:, 0], bits_to_f64(tb(kk))[:, 0],
                       bits_to_f64(bf16_bits(v))[:, 0], mask, 0.5)
    np.testing.assert_allclose(O[:, 0], Oref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[:, 0], lref, rtol=1e-12, atol=1e-12)


def test_sink_special_case():
    # A dominant first block plus recency-ordered others: the gate must pick
    # the sink block 0, the most recent past blocks and the own block.
    B, d, k, nblk = 4, 2, 4, 9
    T = B * nblk
    kk = np.zeros((T, 1, d), dtype=np.float32)
    for j in range(nblk):
        kk[j * B:(j + 1) * B, 0, 0] = 100.0 if j == 0 else float(j)
    q = np.tile(np.array([1.0, 0.0], dtype=np.float32), (T, 1, 1))
    tb = lambda a: bf16_bits(torch.from_numpy(a).to(torch.bfloat16))
    orc = Oracle(tb(q), tb(kk), tb(kk), cu_from_lengths([T]), 1, 1, d, B, k)
    sel, _, _ = orc.select(np.arange(T))
    for t in range(T):
        i = t // B
        got = [x for x in sel[t, 0] if x >= 0]
        if i + 1 <= k:
            assert got == list(range(i + 1))
        else:
            assert got == [0] + list(range(i - k + 2, i + 1))


def test_selection_invariants_every_row():
    lengths, Hq, Hkv, d, B, k = [700, 300, 1], 8, 2, 16, 32, 5
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=13)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    rows = np.arange(int(cu[-1]))
    sel, margin, maxabs = orc.select(rows)
    _, _, own = local_block_info(cu, rows, B)
    for r in rows:
        for h in range(Hq):
            s = [int(x) for x in sel[r, h] if x >= 0]
            assert own[r] in s                         # own block always chosen
            assert max(s) == own[r]                    # never a future block
            assert len(s) == min(k, own[r] + 1)        # exactly min(k, i+1) blocks
            assert s == sorted(set(s))                 # ascending, unique
            assert all(x == -1 for x in sel[r, h][len(s):])
    assert np.all(margin[own >= k] >= 0)
    assert np.all(np.isinf(margin[own < k]))
    assert np.all(maxabs >= 0)


def test_margin_and_maxabs_definition():
    lengths, Hq, Hkv, d, B, k = [48], 2, 1, 3, 4, 3
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=17)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    rows = np.arange(48)
    _, margin, maxabs = orc.select(rows)
    qf, kf = bf.to_fractions(q), bf.to_fractions(kb)
    for t in rows:
        i = t // B
        for h in range(Hq):
            means = [[sum(kf[u, 0, c] for u in range(j * B, j * B + B)) / B for c in range(d)]
                     for j in range(i)]
            sc = sorted((sum(qf[t, h, c] * means[j][c] for c in range(d)) for j in range(i)),
                        reverse=True)
            if i < k:
                assert math.isinf(margin[t, h])
            else:
                assert margin[t, h] == pytest.approx(float(sc[k - 2] - sc[k - 1]), abs=1e-12)
            want = max((abs(float(x)) for x in sc), default=0.0)
            assert maxabs[t, h] == pytest.approx(want, abs=1e-12)


def test_varlen_equals_each_sequence_alone():
    lengths, Hq, Hkv, d, B, k = [37, 64, 5, 50], 4, 2, 8, 8, 3
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=19)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    rows = np.arange(int(cu[-1]))
    O, lse, sel, _, _ = orc.forward(rows)
    for s in range(len(lengths)):
        a, e = int(cu[s]), int(cu[s + 1])
        one = Oracle(q[a:e], kb[a:e], v[a:e], cu_from_lengths([e - a]), Hq, Hkv, d, B, k)
        O1, l1, s1, _, _ = one.forward(np.arange(e - a))
        np.testing.assert_array_equal(sel[a:e], s1)
        np.testing.assert_array_equal(O[a:e], O1)
        np.testing.assert_array_equal(lse[a:e], l1)


def test_online_softmax_merge_is_exact():
    # Any partition of a key set, merged by the online-softmax rule, equals
    # the direct softmax over the whole set.
    rng = np.random.default_rng(0)
    d, n = 8, 50
    q = rng.standard_normal(d)
    K = rng.standard_normal((n, d)) * 2
    V = rng.standard_normal((n, d))
    z = K @ q
    full_lse = logsumexp(z)
    full_O = np.exp(z - full_lse) @ V
    for parts in (3, 7, 50):
        cuts = np.sort(rng.choice(np.arange(1, n), size=parts - 1, replace=False))
        groups = np.split(rng.permutation(n), cuts)
        Os, ls = [], []
        for gidx in groups:
            lz = logsumexp(z[gidx])
            Os.append(np.exp(z[gidx] - lz) @ V[gidx])
            ls.append(lz)
        O, lse = online_softmax_merge(np.array(Os), np.array(ls))
        np.testing.assert_allclose(O, full_O, rtol=1e-12, atol=1e-14)
        assert lse == pytest.approx(full_lse, abs=1e-12)


def _golden(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            cols = line.rstrip("\n").split("\t")
            out.append(cols)
    return out


@pytest.mark.parametrize("row", _golden("sparsity.txt"))
def test_printed_sparsity(row):
    # The pages' sparsity figures follow from the gate choosing exactly k whole
    # blocks of B keys for every query whose sequence has at least k blocks
    # before it: check the oracle's selection size against each printed value.
    N, B, k, pct = int(row[0]), int(row[1]), int(row[2]), float(row[3])
    d = 2
    gen = torch.Generator().manual_seed(N % 1000 + k)
    q = bf16_bits(torch.randn(N, 1, d, generator=gen).to(torch.bfloat16))
    kb = bf16_bits(torch.randn(N, 1, d, generator=gen).to(torch.bfloat16))
    orc = Oracle(q, kb, None, cu_from_lengths([N]), 1, 1, d, B, k)
    rows = np.arange(N - 64, N)  # the last block: at least k blocks precede... or equal
    sel, _, _ = orc.select(rows)
    positions = (sel >= 0).sum(axis=2) * B
    assert np.all(positions == k * B)
    sparsity = 100.0 * (1.0 - positions.mean() / N)
    assert round(sparsity, 2) == pytest.approx(pct, abs=0.005)


def test_printed_attended_positions():
    for row in _golden("attended_positions.txt"):
        N, B, k, pos = (int(x) for x in row[:4])
        gen = torch.Generator().manual_seed(5)
        q = bf16_bits(torch.randn(N, 1, 2, generator=gen).to(torch.bfloat16))
        kb = bf16_bits(torch.randn(N, 1, 2, generator=gen).to(torch.bfloat16))
        orc = Oracle(q, kb, None, cu_from_lengths([N]), 1, 1, 2, B, k)
        sel, _, _ = orc.select(np.array([N - 1]))
        assert int((sel >= 0).sum()) * B == pos


def test_selected_key_count_closed_form():
    # |I| per row = (min(k, i+1) - 1) * B + (t - i*B + 1) for full past blocks;
    # the benchmark's FLOP count rests on this.
    lengths, Hq, Hkv, d, B, k = [203], 2, 1, 4, 16, 4
    q, kb, v, cu = _problem(lengths, Hq, Hkv, d, B, k, seed=23)
    orc = Oracle(q, kb, v, cu, Hq, Hkv, d, B, k)
    rows = np.arange(203)
    sel, _, _ = orc.select(rows)
    _, _, nk = orc.attend(rows, sel)
    i = rows // B
    want = (np.minimum(k, i + 1) - 1) * B + (rows - i * B + 1)
    assert np.all(nk == want[:, None])
