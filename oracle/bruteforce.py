"""Brute-force MoBA for tiny inputs, written independently of the C oracle.

TEST INFRASTRUCTURE ONLY.  It pins the C oracle:
  * the gate is found by enumerating every admissible block subset (own block
    present, no future block, size min(k, i+1)) and keeping the one with the
    largest total past score, ties to the lexicographically smallest subset;
    scores are exact rationals (fractions.Fraction), so ties are exact;
  * attention builds the explicit token-level mask M~ (globaladvisors.biz,
    "Mathematical and complexity implications") and applies a dense masked
    softmax in float64.

Maximising the summed score over admissible subsets and breaking ties
lexicographically picks exactly the top-(k-1) past blocks by (score desc,
index asc) plus the own block, which is the pages' top-k rule (wispaper.ai
blog, "The Change"; sherconan.github.io, steps 3-4) with the lower-index
tie rule.
"""
import itertools
from fractions import Fraction

import numpy as np


def _bits_to_fraction(b):
    u = np.uint32(int(b) << 16)
    f = np.array([u], dtype=np.uint32).view(np.float32)[0]
    return Fraction(float(f))


def to_fractions(bits):
    flat = [_bits_to_fraction(b) for b in np.asarray(bits).reshape(-1)]
    return np.array(flat, dtype=object).reshape(np.asarray(bits).shape)


def blocks_of_sequence(start, end, B):
    """List of (first token, end token) of each block of one sequence."""
    out = []
    a = start
    while a < end:
        out.append((a, min(a + B, end)))
        a += B
    return out


def _best_subset(score, i, k):
    """Admissible subset (own block i plus min(k, i+1) - 1 past blocks) of
    largest total past score, ties to the lexicographically smallest."""
    size = min(k, i + 1)
    best = None
    for sub in itertools.combinations(range(i), size - 1):
        tot = sum((score[j] for j in sub), Fraction(0))
        cand = tuple(sorted(sub + (i,)))
        if best is None or tot > best[0] or (tot == best[0] and cand < best[1]):
            best = (tot, cand)
    return best[1]


def _brute_select_by(block_score, qf, kf, cu, Hq, Hkv, B, k):
    T = int(cu[-1])
    G = Hq // Hkv
    sel = [[None] * Hq for _ in range(T)]
    for s in range(len(cu) - 1):
        blocks = blocks_of_sequence(int(cu[s]), int(cu[s + 1]), B)
        for t in range(int(cu[s]), int(cu[s + 1])):
            i = (t - int(cu[s])) // B
            for h in range(Hq):
                g = h // G
                score = {j: block_score(qf[t, h], kf, g, blocks[j]) for j in range(i)}
                sel[t][h] = _best_subset(score, i, k)
    return sel


def _mean_score(qv, kf, g, blk):
    a, e = blk
    d = kf.shape[2]
    return sum(qv[c] * sum(kf[t, g, c] for t in range(a, e)) / (e - a) for c in range(d))


def _minmax_score(qv, kf, g, blk):
    a, e = blk
    d = kf.shape[2]
    tot = Fraction(0)
    for c in range(d):
        col = [kf[t, g, c] for t in range(a, e)]
        tot += max(qv[c] * max(col), qv[c] * min(col))
    return tot


def brute_select(qf, kf, cu, Hq, Hkv, B, k):
    """sel[t][h] = sorted tuple of local block ids, for every token t (mean
    pooling: s_j = q . mean of block j's keys, exact rationals)."""
    return _brute_select_by(_mean_score, qf, kf, cu, Hq, Hkv, B, k)


def brute_select_minmax(qf, kf, cu, Hq, Hkv, B, k):
    """The same with min/max pooling: s_j = sum_c max(q_c max_t k_tc,
    q_c min_t k_tc) over block j's keys, exact rationals."""
    return _brute_select_by(_minmax_score, qf, kf, cu, Hq, Hkv, B, k)


def mask_from_selection(sel_t_h, cu, B, T):
    """Token-level mask M~[t, u] for one head: u in a selected block, u <= t."""
    M = np.zeros((T, T), dtype=bool)
    for s in range(len(cu) - 1):
        a0, e0 = int(cu[s]), int(cu[s + 1])
        for t in range(a0, e0):
            for j in sel_t_h[t]:
                a = a0 + j * B
                e = min(a + B, e0)
                for u in range(a, e):
                    if u <= t:
                        M[t, u] = True
    return M


def masked_attention(q, k, v, M, scale):
    """Softmax attention restricted to M, float64, by library routines.

    torch's scaled_dot_product_attention computes O and scipy's logsumexp the
    log-normaliser; neither shares code with the C oracle.  q [T,d], k,v [T,d].
    """
    import torch
    from scipy.special import logsumexp
    qt = torch.from_numpy(np.ascontiguousarray(q, dtype=np.float64))[None, None]
    kt = torch.from_numpy(np.ascontiguousarray(k, dtype=np.float64))[None, None]
    vt = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64))[None, None]
    mt = torch.from_numpy(M)[None, None]
    O = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt,
                                                         scale=scale)[0, 0].numpy()
    z = np.where(M, (q @ k.T) * scale, -np.inf)
    return O, logsumexp(z, axis=1)
