"""Seeded synthetic inputs for the MoBA prefill workloads.

This module is shared by the fp64 oracle's tests and by the CUDA path's
tests and benchmark, and holds none of the method's arithmetic: it only
draws numbers.

Recipe (the same for every workload):
  * q, k, v are bf16 roundings of standard normal draws, packed [T][H][d];
  * every (sequence, block, kv head) gets an offset vector with i.i.d.
    N(0, 0.5^2) entries, added to the keys of that block in fp32 before the
    rounding, so that block means differ;
  * draws come from one torch.Generator seeded with the workload's seed, on
    the device the tensors are made on, in this order: offsets, q, k, v, each
    in chunks of CHUNK tokens (so the numbers depend on the device, the seed
    and nothing else).
Varlen lengths come from numpy.random.default_rng(seed): uniform integers in
[lo, hi], rounded down to a multiple of `round_to`.
"""
import dataclasses
from typing import List, Optional

import numpy as np
import torch

CHUNK = 65536


@dataclasses.dataclass
class Workload:
    name: str
    lengths: List[int]          # tokens of each sequence (batch = equal lengths)
    Hq: int
    Hkv: int
    d: int
    B: int                      # block size
    k: int                      # top-k, counting the own block
    seed: int
    batch_mode: bool = True     # equal lengths passed as a [b, N, H, d] batch
    note: str = ""

    @property
    def T(self) -> int:
        return int(sum(self.lengths))

    @property
    def cu(self) -> np.ndarray:
        cu = np.zeros(len(self.lengths) + 1, dtype=np.int64)
        cu[1:] = np.cumsum(np.asarray(self.lengths, dtype=np.int64))
        return cu

    def with_k(self, k: int) -> "Workload":
        return dataclasses.replace(self, k=k, name="%s_k%d" % (self.name, k))


def varlen_lengths(seed: int, n: int, lo: int, hi: int, round_to: int) -> List[int]:
    rng = np.random.default_rng(seed)
    raw = rng.integers(lo, hi, size=n, endpoint=True)
    return [int(max(round_to, (x // round_to) * round_to)) for x in raw]


# The five benchmark workloads.
TINY = Workload("tiny_2k", [2048], 1, 1, 64, 256, 3, seed=0,
                note="batch 1, 1 head, d=64, N=2048, B=256 (n=8), k=3")
FINE_32K = Workload("fine_32k", [32768], 32, 8, 128, 256, 32, seed=1,
                    note="32 q / 8 kv heads, d=128, N=32768, B=256 (128 blocks), k=32")
LONG_128K = Workload("long_128k", [131072], 32, 8, 128, 4096, 12, seed=2,
                     note="32 q / 8 kv heads, d=128, N=131072, B=4096 (32 blocks), k=12")
MILLION = Workload("prefill_1m", [1048576], 32, 8, 128, 4096, 12, seed=3,
                   note="32 q / 8 kv heads, d=128, N=1048576, B=4096 (256 blocks), k=12")
VARLEN = Workload("varlen_8seq", varlen_lengths(4, 8, 4096, 65536, 256), 32, 8, 128, 512, 8,
                  seed=4, batch_mode=False,
                  note="8 packed sequences, lengths U[4096,65536] rounded to 256, B=512, k=8")

# The 10M-token setting (wispaper.ai blog, "Efficiency and Implementation":
# n = 256 blocks and k fixed, B grown to 10M / 256 = 40960) does not fit one
# GPU at 32 q heads; sharded by kv-head group across 8 GPUs, each GPU holds
# one kv head and its 4 q heads.  This is that per-GPU shard.
PREFILL_10M_SHARD = Workload("prefill_10m_shard", [10485760], 4, 1, 128, 40960, 12, seed=5,
                             note="one kv-head group (4 q / 1 kv head) of the 32 q / 8 kv "
                                  "model at N=10485760, B=40960 (256 blocks), k=12")

# long_128k's shape with a quarter of the heads (same N, B, k and per-head
# bucket sizes): a case small enough on the device for multi-pass kernel
# captures, with q (268 MB) still larger than L2.
LONG_128K_H8 = Workload("long_128k_h8", [131072], 8, 2, 128, 4096, 12, seed=2,
                        note="8 q / 2 kv heads, d=128, N=131072, B=4096 (32 blocks), k=12")

# fine_32k's shape with a quarter of the heads (same N, B, k): the small
# case for multi-pass captures of the short-block kernels.
FINE_32K_H8 = Workload("fine_32k_h8", [32768], 8, 2, 128, 256, 32, seed=1,
                       note="8 q / 2 kv heads, d=128, N=32768, B=256 (128 blocks), k=32")

WORKLOADS = {w.name: w for w in (TINY, FINE_32K, LONG_128K, MILLION, VARLEN, PREFILL_10M_SHARD,
                                 LONG_128K_H8, FINE_32K_H8)}


def block_ids(lengths: List[int], B: int) -> np.ndarray:
    """Global block id (sequence by sequence) of every token."""
    out = []
    base = 0
    for L in lengths:
        j = np.arange(L, dtype=np.int64) // B
        out.append(j + base)
        base += (L + B - 1) // B
    return np.concatenate(out) if out else np.zeros(0, dtype=np.int64)


def make_qkv(w: Workload, device="cpu", seed: Optional[int] = None, need_v: bool = True):
    """q [T,Hq,d], k [T,Hkv,d], v [T,Hkv,d] as bf16 tensors on `device`."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed if seed is None else seed)
    T = w.T
    bid = block_ids(w.lengths, w.B)
    nb = int(bid[-1]) + 1 if T else 0
    offs = torch.randn(nb, w.Hkv, w.d, generator=g, device=dev, dtype=torch.float32) * 0.5
    bid_t = torch.from_numpy(bid).to(dev)

    def draw(H, offsets=None):
        out = torch.empty(T, H, w.d, device=dev, dtype=torch.bfloat16)
        for a in range(0, T, CHUNK):
            e = min(T, a + CHUNK)
            x = torch.randn(e - a, H, w.d, generator=g, device=dev, dtype=torch.float32)
            if offsets is not None:
                x += offsets[bid_t[a:e]]
            out[a:e] = x.to(torch.bfloat16)
            del x
        return out

    q = draw(w.Hq)
    k = draw(w.Hkv, offs)
    v = draw(w.Hkv) if need_v else None
    return q, k, v


def sample_rows(w: Workload, per_head_rows: int, seed: int = 1234) -> np.ndarray:
    """Seeded sample of distinct global query rows, sorted (all rows if fewer)."""
    T = w.T
    if per_head_rows >= T:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=per_head_rows, replace=False)).astype(np.int64)


# Inputs whose attention rows are peaky: keys planted late in every block
# that outscore everything before them by far, and queries aligned with them.
# They exist so that the running maximum of a row's scores jumps, after the
# first 128-key tile of the keys it attends, by many powers of two (the
# attention kernels rescale their accumulators only on such a jump).
#
# Recipe, on top of make_qkv's draws:
#   * one unit direction u_g per kv head (N(0, I) normalised), drawn from a
#     generator seeded with seed + 7919;
#   * q heads with an even index get a * u_g added (their kv head's u);
#   * in every block, for each (tile, c) of `plants`, the keys at positions
#     tile * 128 + 37 and tile * 128 + 91 of the block (where they exist) get
#     c * u_g added;
#   * v is multiplied by v_scale (a power of two, so exactly).
# The additions happen in fp32 on the bf16 draws and are rounded once more.
PEAKY_PLANTS = ((1, 24.0), (3, 48.0))


def make_peaky_qkv(w: Workload, device="cpu", a: float = 6.0, plants=PEAKY_PLANTS,
                   v_scale: float = 0.25, seed: Optional[int] = None):
    dev = torch.device(device)
    q, k, v = make_qkv(w, dev, seed=seed)
    g = torch.Generator(device=dev)
    g.manual_seed((w.seed if seed is None else seed) + 7919)
    u = torch.randn(w.Hkv, w.d, generator=g, device=dev, dtype=torch.float32)
    u = u / u.norm(dim=1, keepdim=True)
    G = w.Hq // w.Hkv
    qf = q.float()
    for h in range(0, w.Hq, 2):
        qf[:, h] += a * u[h // G]
    kf = k.float()
    pos = []
    base = 0
    for L in w.lengths:
        for b0 in range(0, L, w.B):
            for tile, c in plants:
                for off in (37, 91):
                    p = b0 + tile * 128 + off
                    if p < min(L, b0 + w.B):
                        pos.append((base + p, c))
        base += L
    if pos:
        idx = torch.tensor([p for p, _ in pos], device=dev, dtype=torch.long)
        cs = torch.tensor([c for _, c in pos], device=dev, dtype=torch.float32)
        kf[idx] += cs[:, None, None] * u[None, :, :]
    return qf.to(torch.bfloat16), kf.to(torch.bfloat16), (v.float() * v_scale).to(torch.bfloat16)
