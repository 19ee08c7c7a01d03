"""One problem split across ranks by kv-head group (block_sparse_long_07_b200
.shard), run as two (or three) gloo ranks on the CPU.

Each rank slices its kv heads and their q heads out of the shared inputs,
computes its slice with the fp64 oracle standing in for the library's
forward (the split itself does no arithmetic), and the pieces are gathered
along the head axis.  Rank 0 then requires the gathered o, lse and selection
to equal the oracle run on all heads at once, bit for bit: every head's
result depends only on its own q head and kv head, which is what makes the
split exact (wispaper.ai blog, "Efficiency and Implementation": tensor
parallelism extended to the query heads at 10M tokens).
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RANK_SCRIPT = r"""
import datetime, json, os, sys
import numpy as np, torch, torch.distributed as dist
root = sys.argv[1]
sys.path.insert(0, root)
import synthetic as S
from oracle import Oracle, bf16_bits
from block_sparse_long_07_b200 import shard

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
lengths, Hq, Hkv, d, B, k, packed = json.loads(sys.argv[2])
w = S.Workload("split", lengths, Hq, Hkv, d, B, k, seed=515, batch_mode=not packed)
q, kk, v = S.make_qkv(w, "cpu")                       # packed [T, H, d]
b, N = len(lengths), lengths[0]
if not packed:
    q, kk, v = (x.view(b, N, x.shape[1], d) for x in (q, kk, v))

def oracle_forward(qr, kr, vr):
    # stand-in for the library forward on this rank's heads
    hq, hkv = qr.shape[-2], kr.shape[-2]
    flat = lambda x: x.reshape(-1, x.shape[-2], d)
    orc = Oracle(bf16_bits(flat(qr)), bf16_bits(flat(kr)), bf16_bits(flat(vr)), w.cu, hq, hkv,
                 d, B, k)
    rows = np.arange(w.T, dtype=np.int64)
    O, lse, sel, _, _ = orc.forward(rows)             # [T, h, d], [T, h], [T, h, k]
    O, lse, sel = torch.from_numpy(O), torch.from_numpy(lse), torch.from_numpy(sel)
    if packed:
        return O, lse.t().contiguous(), sel.permute(1, 0, 2).contiguous()
    return (O.view(b, N, hq, d), lse.view(b, N, hq).permute(0, 2, 1).contiguous(),
            sel.view(b, N, hq, k).permute(0, 2, 1, 3).contiguous())

g0, g1 = shard.kv_head_range(rank, world, Hkv)
o, lse, sel = shard.forward_sharded(oracle_forward, q, kk, v, rank, world, dist,
                                    batch_layout=not packed)
res = {"rank": rank, "g": [g0, g1]}
if rank == 0:
    O1, L1, S1 = oracle_forward(q, kk, v)             # all heads in one call
    res["o_equal"] = bool(torch.equal(o, O1))
    res["lse_equal"] = bool(torch.equal(lse, L1))
    res["sel_equal"] = bool(torch.equal(sel, S1))
    res["shape"] = list(o.shape)
dist.barrier()
dist.destroy_process_group()
print(json.dumps(res))
"""


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(tmp_path, world, case):
    script = tmp_path / "rank.py"
    script.write_text(_RANK_SCRIPT)
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   LOCAL_RANK=str(r), WORLD_SIZE=str(world), OMP_NUM_THREADS="2")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT, json.dumps(case)],
                                      env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err[-3000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    return outs


@pytest.mark.parametrize("world,case", [
    (2, ([1024], 8, 4, 64, 128, 3, False)),          # 2 kv heads per rank, GQA 2
    (2, ([600, 600], 6, 3, 64, 128, 2, False)),      # uneven: 1 and 2 kv heads, batch of 2
    (3, ([300, 1000, 77], 8, 4, 64, 128, 3, True)),  # packed varlen, 3 ranks (1, 1, 2 heads)
])
def test_split_by_kv_head_equals_the_whole_problem(tmp_path, world, case):
    outs = _run(tmp_path, world, case)
    Hkv = case[2]
    ranges = sorted(o["g"] for o in outs)
    # the ranges tile [0, Hkv) with no gap and no overlap
    assert ranges[0][0] == 0 and ranges[-1][1] == Hkv
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    assert all(g1 > g0 for g0, g1 in ranges)
    r0 = [o for o in outs if o["rank"] == 0][0]
    assert r0["o_equal"] and r0["lse_equal"] and r0["sel_equal"], r0


def test_head_ranges():
    sys.path.insert(0, ROOT)
    from block_sparse_long_07_b200 import shard
    assert [shard.kv_head_range(r, 8, 8) for r in range(8)] == [(r, r + 1) for r in range(8)]
    assert [shard.kv_head_range(r, 3, 8) for r in range(3)] == [(0, 2), (2, 5), (5, 8)]
    assert shard.q_head_range(1, 3, 32, 8) == (8, 20)
    with pytest.raises(ValueError):
        shard.kv_head_range(0, 9, 8)   # a rank would own no kv head
    with pytest.raises(ValueError):
        shard.q_head_range(0, 2, 30, 8)
