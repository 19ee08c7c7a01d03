"""The seeded input recipe the tests and the benchmark share (synthetic.py):
its stated shapes and properties, checked on the CPU."""
import numpy as np
import torch

import synthetic as S


def test_varlen_workload_lengths():
    w = S.VARLEN
    assert len(w.lengths) == 8 and w.T == 402176
    assert all(4096 <= n <= 65536 and n % 256 == 0 for n in w.lengths)
    assert list(w.cu) == [0] + list(np.cumsum(w.lengths))


def test_workload_shapes():
    assert (S.MILLION.T, S.MILLION.Hq, S.MILLION.Hkv, S.MILLION.d, S.MILLION.B, S.MILLION.k) == \
        (1048576, 32, 8, 128, 4096, 12)
    assert (S.LONG_128K_H8.T, S.LONG_128K_H8.B, S.LONG_128K_H8.k) == (131072, 4096, 12)
    assert S.PREFILL_10M_SHARD.T // S.PREFILL_10M_SHARD.B == 256
    for name, w in S.WORKLOADS.items():
        assert name == w.name and w.Hq % w.Hkv == 0


def test_inputs_are_seeded_and_bf16():
    w = S.Workload("t", [3000, 700], 4, 2, 64, 256, 3, seed=11, batch_mode=False)
    a = S.make_qkv(w, "cpu")
    b = S.make_qkv(w, "cpu")
    c = S.make_qkv(w, "cpu", seed=12)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    assert a[0].shape == (3700, 4, 64) and a[1].shape == (3700, 2, 64)


def test_block_offsets_make_block_means_differ():
    # keys get one N(0, 0.5^2) offset vector per (block, kv head): the spread
    # of block means across blocks is about 0.5, far above the ~1/sqrt(B)
    # spread of the unit-variance keys' own means
    w = S.Workload("t", [256 * 64], 1, 1, 128, 256, 3, seed=3)
    _, k, _ = S.make_qkv(w, "cpu")
    means = k.float().view(64, 256, 128).mean(dim=1)
    assert 0.4 < float(means.std()) < 0.6
    q, _, _ = S.make_qkv(w, "cpu")
    assert abs(float(q.float().std()) - 1.0) < 0.02  # queries carry no offset


def test_block_ids_restart_with_each_sequence():
    ids = S.block_ids([300, 5, 256], 256)
    assert list(ids[:300:100]) == [0, 0, 0] and ids[256] == 1
    assert ids[300] == 2 and ids[305] == 3 and ids[-1] == 3


def test_peaky_inputs_force_the_rescale_rule():
    """The planted-key recipe makes a row's running score maximum jump past
    the attention kernels' rescale threshold after the first key tile: in
    the routed span of past blocks, in the own block and in the dense span
    (replayed in fp64 on CPU-drawn inputs of the recipe)."""
    import sys, os
    sys.path.insert(0, os.path.dirname(__file__))
    from oracle import Oracle, bf16_bits
    from rescale_util import rescale_events
    w = S.Workload("peaky", [4096], 4, 2, 128, 512, 3, seed=3131)
    q, k, v = S.make_peaky_qkv(w, "cpu")
    assert torch.equal(v.float() * 4, S.make_qkv(w, "cpu")[2].float())  # v scaled exactly
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    rows = np.arange(w.T, dtype=np.int64)
    sel, _, _ = Oracle(qb, kb, vb, w.cu, 4, 2, 128, 512, 3).select(rows)
    ev_r, ev_o = rescale_events(qb, kb, w.cu, rows, 4, 2, 128, 512, sel=sel)
    ev_d, _ = rescale_events(qb, kb, w.cu, rows, 4, 2, 128, 512, dense=True)
    # the peaked (even) heads: every row with a past block rescales there
    assert (ev_r[:, 0::2] > 0).mean() >= 0.85
    assert (ev_o[:, 0::2] > 0).mean() >= 0.5
    assert (ev_d[:, 0::2] > 0).mean() >= 0.9
    assert (ev_r[:, 0::2] > 1).mean() >= 0.5 * (ev_r[:, 0::2] > 0).mean()  # tile 3 again
