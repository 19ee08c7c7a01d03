"""ctypes front end of the fp64 C oracle, plus the merge rule in numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Arrays are numpy.  bf16 tensors enter as their raw 16-bit patterns
(``bf16_bits``), packed [T][H][d]; sequences are given by int64 cumulative
lengths ``cu`` (a batch of b sequences of length N is cu = 0, N, ..., bN).

Passages followed (MoBA: Mixture of Block Attention for Long-Context LLMs):
  wispaper.ai blog, "The Change" (partition, affinity, top-k routing,
  causality rules) and "Efficiency and Implementation" (online-softmax
  combination); globaladvisors.biz, "Underlying computational mechanism";
  sherconan.github.io, steps 1-5.
"""
import ctypes
import math
import os

import numpy as np

from .build_oracle import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build()
        lib = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i32 = ctypes.c_int
        i64 = ctypes.c_int64
        dbl = ctypes.c_double
        lib.oracle_num_threads.restype = i32
        lib.oracle_num_threads.argtypes = []
        lib.oracle_total_blocks.restype = i64
        lib.oracle_total_blocks.argtypes = [p, i32, i32]
        lib.oracle_block_means.restype = i32
        lib.oracle_block_means.argtypes = [p, p, i32, i32, i32, i32, p]
        lib.oracle_select.restype = i32
        lib.oracle_select.argtypes = [p, p, p, i32, i32, i32, i32, i32, i32, p, i64,
                                      p, p, p]
        lib.oracle_block_minmax.restype = i32
        lib.oracle_block_minmax.argtypes = [p, p, i32, i32, i32, i32, p, p]
        lib.oracle_select_minmax.restype = i32
        lib.oracle_select_minmax.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, p, i64,
                                             p, p, p]
        lib.oracle_attend.restype = i32
        lib.oracle_attend.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, dbl,
                                      p, i64, p, p, p, p]
        lib.oracle_attend_backward.restype = i32
        lib.oracle_attend_backward.argtypes = [p, p, p, p, i32, i32, i32, i32, i32, i32, dbl,
                                               p, i64, p, p, p, p, p]
        lib.oracle_dense_causal.restype = i32
        lib.oracle_dense_causal.argtypes = [p, p, p, p, i32, i32, i32, i32, dbl, p, i64,
                                            p, p]
        _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def bf16_bits(t):
    """Raw bf16 bit patterns of a torch bf16 tensor, as a numpy uint16 array."""
    import torch
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits):
    """Exact widening of bf16 bit patterns to float64."""
    u = bits.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def cu_from_lengths(lengths):
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def local_block_info(cu, rows, B):
    """(sequence, position within sequence, own block) of each global row."""
    cu = np.asarray(cu, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    s = np.searchsorted(cu, rows, side="right") - 1
    p = rows - cu[s]
    return s, p, p // B


def online_softmax_merge(parts_O, parts_lse):
    """Combine partial attention results over disjoint key sets.

    Each part s holds O_s (normalised over its own keys) and lse_s.  The
    combination (Milakov & Gimelshein's online normaliser, the merge the
    wispaper.ai blog names under "Efficiency and Implementation") is
        m   = max_s lse_s
        w_s = exp(lse_s - m)
        O   = sum_s w_s O_s / sum_s w_s
        lse = m + log(sum_s w_s).
    parts_O: [S, ..., d]; parts_lse: [S, ...].
    """
    lse = np.asarray(parts_lse, dtype=np.float64)
    O = np.asarray(parts_O, dtype=np.float64)
    m = lse.max(axis=0)
    w = np.exp(lse - m)
    den = w.sum(axis=0)
    out = (w[..., None] * O).sum(axis=0) / den[..., None]
    return out, m + np.log(den)


def static_selection(cu, rows, B, k, mode):
    """Static routings the pages describe as fixed corners of the MoBA gate
    (wispaper.ai blog, "Why the Change Is Plausible"): "window" keeps the
    own block and the k-1 most recent past blocks; "sink" keeps block 0, the
    k-2 most recent past blocks and the own block.  With fewer than k blocks
    every block is kept, as the gate does.  Returns sel [R][k] (local block
    ids ascending, -1 padded); the same for every head."""
    cu = np.asarray(cu, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.full((len(rows), k), -1, dtype=np.int32)
    for r, t in enumerate(rows):
        s = int(np.searchsorted(cu, t, side="right") - 1)
        i = int((t - cu[s]) // B)
        npast = min(k - 1, i)
        if mode == "window" or npast == i or npast == 0:
            past = list(range(i - npast, i))
        elif mode == "sink":
            past = [0] + list(range(i - npast + 1, i))
        else:
            raise ValueError(mode)
        blocks = past + [i]
        out[r, :len(blocks)] = blocks
    return out


class Oracle:
    """fp64 reference for one problem (one set of q, k, v and parameters)."""

    def __init__(self, q_bits, k_bits, v_bits, cu, Hq, Hkv, d, B, k, scale=None):
        self.lib = _load()
        self.q = np.ascontiguousarray(q_bits, dtype=np.uint16)
        self.k = np.ascontiguousarray(k_bits, dtype=np.uint16)
        self.v = None if v_bits is None else np.ascontiguousarray(v_bits, dtype=np.uint16)
        self.cu = np.ascontiguousarray(cu, dtype=np.int64)
        self.nseq = len(self.cu) - 1
        self.Hq, self.Hkv, self.d, self.B, self.topk = Hq, Hkv, d, B, k
        self.scale = (1.0 / math.sqrt(d)) if (scale is None or scale <= 0) else float(scale)
        T = int(self.cu[-1])
        assert self.q.shape == (T, Hq, d), self.q.shape
        assert self.k.shape == (T, Hkv, d), self.k.shape
        self._kbar = None

    @staticmethod
    def num_threads():
        return _load().oracle_num_threads()

    @property
    def total_blocks(self):
        return int(self.lib.oracle_total_blocks(_ptr(self.cu), self.nseq, self.B))

    def block_means(self):
        """Kbar [Hkv][NB][d], blocks numbered sequence by sequence."""
        if self._kbar is None:
            kb = np.zeros((self.Hkv, self.total_blocks, self.d), dtype=np.float64)
            rc = self.lib.oracle_block_means(_ptr(self.k), _ptr(self.cu), self.nseq,
                                             self.Hkv, self.d, self.B, _ptr(kb))
            if rc:
                raise RuntimeError("oracle_block_means failed: %d" % rc)
            self._kbar = kb
        return self._kbar

    def select(self, rows):
        """sel [R][Hq][k] (local block ids, ascending, -1 padded), margin, maxabs."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = len(rows)
        kb = self.block_means()
        sel = np.zeros((R, self.Hq, self.topk), dtype=np.int32)
        margin = np.zeros((R, self.Hq), dtype=np.float64)
        maxabs = np.zeros((R, self.Hq), dtype=np.float64)
        rc = self.lib.oracle_select(_ptr(self.q), _ptr(kb), _ptr(self.cu), self.nseq,
                                    self.Hq, self.Hkv, self.d, self.B, self.topk,
                                    _ptr(rows), R, _ptr(sel), _ptr(margin), _ptr(maxabs))
        if rc:
            raise RuntimeError("oracle_select failed: %d" % rc)
        return sel, margin, maxabs

    def block_minmax(self):
        """(Kmax, Kmin) [Hkv][NB][d]: elementwise max / min of each block's keys."""
        if getattr(self, "_kminmax", None) is None:
            kx = np.zeros((self.Hkv, self.total_blocks, self.d), dtype=np.float64)
            kn = np.zeros_like(kx)
            rc = self.lib.oracle_block_minmax(_ptr(self.k), _ptr(self.cu), self.nseq, self.Hkv,
                                              self.d, self.B, _ptr(kx), _ptr(kn))
            if rc:
                raise RuntimeError("oracle_block_minmax failed: %d" % rc)
            self._kminmax = (kx, kn)
        return self._kminmax

    def select_minmax(self, rows):
        """The gate with min/max-pooled blocks (score sum_c max(q_c Kmax_c, q_c Kmin_c)):
        sel, margin, maxabs as select()."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = len(rows)
        kx, kn = self.block_minmax()
        sel = np.zeros((R, self.Hq, self.topk), dtype=np.int32)
        margin = np.zeros((R, self.Hq), dtype=np.float64)
        maxabs = np.zeros((R, self.Hq), dtype=np.float64)
        rc = self.lib.oracle_select_minmax(_ptr(self.q), _ptr(kx), _ptr(kn), _ptr(self.cu),
                                           self.nseq, self.Hq, self.Hkv, self.d, self.B,
                                           self.topk, _ptr(rows), R, _ptr(sel), _ptr(margin),
                                           _ptr(maxabs))
        if rc:
            raise RuntimeError("oracle_select_minmax failed: %d" % rc)
        return sel, margin, maxabs

    def attend(self, rows, sel):
        """Attention over the key set each row's selection names."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        R = len(rows)
        assert sel.shape[0] == R and sel.shape[1] == self.Hq
        kk = sel.shape[2]
        O = np.zeros((R, self.Hq, self.d), dtype=np.float64)
        lse = np.zeros((R, self.Hq), dtype=np.float64)
        nk = np.zeros((R, self.Hq), dtype=np.int64)
        rc = self.lib.oracle_attend(_ptr(self.q), _ptr(self.k), _ptr(self.v), _ptr(self.cu),
                                    self.nseq, self.Hq, self.Hkv, self.d, self.B, kk,
                                    self.scale, _ptr(rows), R, _ptr(sel), _ptr(O), _ptr(lse),
                                    _ptr(nk))
        if rc:
            raise RuntimeError("oracle_attend failed: %d" % rc)
        return O, lse, nk

    def attend_backward(self, rows, sel, dO_bits):
        """Gradients of the attention over a fixed selection (the gate passes
        none): dQ [R][Hq][d] for the listed rows, and dK, dV [T][Hkv][d]
        summed over the listed rows.  dO_bits: bf16 bits [R][Hq][d]."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        dO_bits = np.ascontiguousarray(dO_bits, dtype=np.uint16)
        R = len(rows)
        assert sel.shape[:2] == (R, self.Hq) and dO_bits.shape == (R, self.Hq, self.d)
        T = int(self.cu[-1])
        dQ = np.zeros((R, self.Hq, self.d), dtype=np.float64)
        dK = np.zeros((T, self.Hkv, self.d), dtype=np.float64)
        dV = np.zeros((T, self.Hkv, self.d), dtype=np.float64)
        rc = self.lib.oracle_attend_backward(_ptr(self.q), _ptr(self.k), _ptr(self.v),
                                             _ptr(self.cu), self.nseq, self.Hq, self.Hkv,
                                             self.d, self.B, sel.shape[2], self.scale,
                                             _ptr(rows), R, _ptr(sel), _ptr(dO_bits), _ptr(dQ),
                                             _ptr(dK), _ptr(dV))
        if rc:
            raise RuntimeError("oracle_attend_backward failed: %d" % rc)
        return dQ, dK, dV

    def forward(self, rows):
        """Gate then attention: O [R][Hq][d], lse [R][Hq], sel, margin, maxabs."""
        sel, margin, maxabs = self.select(rows)
        O, lse, _ = self.attend(rows, sel)
        return O, lse, sel, margin, maxabs

    def dense(self, rows):
        """Full causal attention (every earlier token of the row's sequence)."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R = len(rows)
        O = np.zeros((R, self.Hq, self.d), dtype=np.float64)
        lse = np.zeros((R, self.Hq), dtype=np.float64)
        rc = self.lib.oracle_dense_causal(_ptr(self.q), _ptr(self.k), _ptr(self.v),
                                          _ptr(self.cu), self.nseq, self.Hq, self.Hkv,
                                          self.d, self.scale, _ptr(rows), R, _ptr(O),
                                          _ptr(lse))
        if rc:
            raise RuntimeError("oracle_dense_causal failed: %d" % rc)
        return O, lse
