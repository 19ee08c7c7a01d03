"""Where the attention kernels' running-maximum rescale must run.

The tensor-core attention streams a row's keys in 128-key tiles, starting at
the first key of the span it attends (a routed past block, the own block, or
the sequence start for the dense kernel).  It keeps a running maximum m of
the row's log2-domain scores z = (q . k) * scale * log2(e) and rescales its
output accumulator only when a later tile's maximum exceeds m by more than
RESCALE_LOG2 (then m takes the new maximum).  This module replays that rule
in fp64 on the test inputs, so a test can show that its inputs drive the
rescale branch (and on how many rows), independently of the kernel.
"""
import math

import numpy as np

from oracle.oracle import bits_to_f64, local_block_info

RESCALE_LOG2 = 8.0
TILE = 128
LOG2E = 1.4426950408889634


def _events_on_span(tmax, t0, t1):
    """Rescale events of the rule above over tiles t0 .. t1 - 1 of one row."""
    if t1 - t0 <= 1:
        return 0
    m = tmax[t0]
    n = 0
    for j in range(t0 + 1, t1):
        if tmax[j] > m + RESCALE_LOG2:
            m = tmax[j]
            n += 1
    return n


def rescale_events(q_bits, k_bits, cu, rows, Hq, Hkv, d, B, sel=None, dense=False):
    """Per (row, head) counts of rescale events, split as (routed, own) or,
    with dense=True, (dense, None).

    q_bits [T][Hq][d], k_bits [T][Hkv][d] bf16 bit patterns; rows are global
    token indices; sel [R][Hq][k] local block ids (-1 padded) of each row, the
    own block last among the valid entries."""
    cu = np.asarray(cu, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    s_of, p_of, own_of = local_block_info(cu, rows, B)
    G = Hq // Hkv
    c = LOG2E / math.sqrt(d)
    R = len(rows)
    ev_a = np.zeros((R, Hq), dtype=np.int64)
    ev_b = np.zeros((R, Hq), dtype=np.int64)
    q = bits_to_f64(q_bits)
    k = bits_to_f64(k_bits)
    for s in np.unique(s_of):
        c0, c1 = int(cu[s]), int(cu[s + 1])
        L = c1 - c0
        nt = (L + TILE - 1) // TILE
        ridx = np.nonzero(s_of == s)[0]
        p = p_of[ridx]
        for h in range(Hq):
            g = h // G
            Z = (q[c0 + p, h, :] @ k[c0:c1, g, :].T) * c  # [r, L]
            keys = np.arange(L)
            Z = np.where(keys[None, :] <= p[:, None], Z, -np.inf)
            pad = nt * TILE - L
            Zp = np.pad(Z, ((0, 0), (0, pad)), constant_values=-np.inf)
            tmax = Zp.reshape(len(ridx), nt, TILE).max(axis=2)
            for n, r in enumerate(ridx):
                tl = int(p[n]) // TILE
                if dense:
                    ev_a[r, h] = _events_on_span(tmax[n], 0, tl + 1)
                    continue
                ob = int(own_of[r])
                ev_b[r, h] = _events_on_span(tmax[n], ob * B // TILE, tl + 1)
                if sel is None:
                    continue
                tot = 0
                for J in sel[r, h]:
                    if J < 0 or J == ob:
                        continue
                    tot += _events_on_span(tmax[n], J * B // TILE, (J + 1) * B // TILE)
                ev_a[r, h] = tot
    return ev_a, (None if dense else ev_b)
