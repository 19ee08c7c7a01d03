"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that
ties the committed DRAM-traffic record to the code it was measured on."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_code_hash_ignores_comments_and_blank_lines():
    b = _bench()
    src = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    assert b.code_sha1(src) == b.code_sha1("// header\n\nint f(int x) {\n  return x + 1;\n}\n")
    assert b.code_sha1(src) == b.code_sha1("/* block\n comment */int f(int x) {\n  return x + 1;\n}\n")


def test_code_hash_sees_code_changes():
    b = _bench()
    assert b.code_sha1("int f(int x) { return x + 1; }") != b.code_sha1("int f(int x) { return x + 2; }")


def test_traffic_record_is_dropped_when_the_code_differs(tmp_path, monkeypatch):
    b = _bench()
    ent = {"source_file": "k.cuh", "source_code_sha1": b.code_sha1("int a;"), "bytes_per_entry": 2.0}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text('{"k": %s}' % __import__("json").dumps(ent))
    (tmp_path / "k.cuh").write_text("int a;  // the measured code\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.load_traffic("k", 10) == 20.0
    (tmp_path / "k.cuh").write_text("int b;\n")
    assert b.load_traffic("k", 10) is None


_RANK_SCRIPT = r"""
import importlib.util, json, os, sys, datetime
import torch, torch.distributed as dist
root = sys.argv[1]
sys.path.insert(0, root)
spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
b = importlib.util.module_from_spec(spec); spec.loader.exec_module(b)
import synthetic as S
world, rank, _ = b.dist_setup()
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
ranks = b.RankGroup(dist, "cpu")
ranks.barrier()
ms = ranks.max(10.0 + rank)          # the slowest rank's step time
rate = b.whole_job_rate(world, 1000.0, ms)
w = S.Workload("ranks", [256], 2, 1, 64, 128, 2, seed=7)
q, _, _ = S.make_qkv(w, "cpu", seed=b.rank_seed(w, rank), need_v=False)
ranks.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "world": world, "ms": ms, "rate": rate,
                  "q0": float(q.float()[0, 0, 0])}))
"""


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_take_the_slowest_step_and_sum_the_work(tmp_path):
    # The multi-GPU bench runs one independent copy of the workload per rank:
    # each step is timed by the slowest rank and the work of all ranks adds.
    import json
    import subprocess
    import sys
    script = tmp_path / "rank.py"
    script.write_text(_RANK_SCRIPT)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   LOCAL_RANK=str(r), WORLD_SIZE="2")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2 and o["ms"] == 11.0
        assert abs(o["rate"] - 2 * 1000.0 / 0.011) < 1e-6
    assert outs[0]["q0"] != outs[1]["q0"]  # each rank draws its own inputs
