"""Benchmark of the MoBA causal prefill forward on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle, bounded sample
    python bench.py --mode decode ...        # one decode step against the workload as a cache

A step is one full MoBA prefill forward (pool, gate, bucketing, routed and
own-block attention, merge) over the workload's synthetic input, through the
library's public call with inputs already resident in HBM.  Inputs are far
larger than L2 (1M tokens: 12.9 GB of q/k/v), so no flush is needed between
steps.  With N > 1 every rank runs its own copy of the workload (independent
problems, no collective on the data path: weak scaling); the step time is the
maximum over ranks.

Reported (one JSON line on rank 0):
  value      effective TFLOP/s: 4*d FLOPs per selected (query, key) pair, own
             block counted causally, summed over all ranks / step time;
  e2e        the same metric with pinned host inputs copied in and O / lse
             copied out inside the timed region;
  roofline   the routed-attention kernel (the dominant launch) against the
             measured dense bf16 tensor peak;
  cpu_baseline  the oracle on a bounded row sample, on this host's cores;
  dense_ms / speedup_vs_dense  the dense causal kernel (k = n) at the same N.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoBA prefill ms & effective TFLOP/s at 1M tokens; % bf16 tensor peak; x vs dense"
DECODE_METRIC = "MoBA decode steps/s (one new token per sequence) against a 1M-token KV cache"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- work model
def selected_pairs(w):
    """(total selected (query, key) pairs per q head, routed part) for a workload."""
    tot = 0
    routed = 0
    for L in w.lengths:
        p = np.arange(L, dtype=np.int64)
        i = p // w.B
        past = (np.minimum(w.k, i + 1) - 1) * w.B
        own = p - i * w.B + 1
        tot += int((past + own).sum())
        routed += int(past.sum())
    return tot, routed


def dense_pairs(w):
    return sum(L * (L + 1) // 2 for L in w.lengths)


def flops_of_pairs(pairs, w):
    return 4.0 * w.d * pairs * w.Hq


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            cols = [c.strip() for c in line.split(",")]
            if len(cols) < 9:
                continue
            try:
                sm.append(float(cols[1]))
                mx = float(cols[2])
            except ValueError:
                continue
            for n, c in zip(names, cols[5:9]):
                if c.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def code_sha1(text):
    """sha1 of C++ source with comments and blank lines removed: the counters
    of a kernel stay valid across edits that touch only its comments."""
    import hashlib
    import re
    t = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    t = re.sub(r"//[^\n]*", "", t)
    lines = [ln.rstrip() for ln in t.splitlines() if ln.strip()]
    return hashlib.sha1("\n".join(lines).encode()).hexdigest()


def load_traffic(name, entries_per_launch):
    """DRAM bytes per launch of a kernel from the committed ncu summary, scaled
    to this workload by work entries, or None when the kernel's code changed
    since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            ent = json.load(f).get(name)
        with open(os.path.join(ROOT, ent["source_file"])) as f:
            sha = code_sha1(f.read())
    except (OSError, ValueError, KeyError, TypeError):
        return None
    if sha != ent.get("source_code_sha1"):
        return None
    return float(ent["bytes_per_entry"]) * entries_per_launch


class RankGroup:
    """The processes of a multi-GPU run, one per GPU: a barrier and the max of
    a scalar (the step time) over ranks through the given torch.distributed
    module (NCCL here; any backend works), or no-ops for a single process."""

    def __init__(self, pg=None, device="cpu"):
        self.pg, self.device = pg, device

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x):
        if self.pg is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())


def rank_seed(w, rank):
    """Each rank draws its own copy of the workload (independent problems)."""
    return w.seed + 1000 * rank


def whole_job_rate(world, units_per_rank_step, ms_max):
    """Units per second over all ranks, each step timed by the slowest rank."""
    return world * units_per_rank_step / (ms_max / 1e3)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_baseline(w, q_rows_fn, k_bits, v_bits, budget_s=15.0, seed=4321):
    """Time the oracle on a bounded sample of query rows of the workload."""
    from oracle import Oracle
    T = w.T
    q_bits = np.zeros((T, w.Hq, w.d), dtype=np.uint16)  # lazily backed; only sampled rows set
    orc = Oracle(q_bits, k_bits, v_bits, w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    t0 = time.perf_counter()
    orc.block_means()
    pool_s = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    # probe with a few rows, then size the sample to the time budget
    n_probe = 4
    rows = np.sort(rng.choice(T, size=n_probe, replace=False)).astype(np.int64)
    q_bits[rows] = q_rows_fn(rows)
    t0 = time.perf_counter()
    orc.forward(rows)
    probe_s = max(time.perf_counter() - t0, 1e-3)
    n = int(min(T, max(n_probe, n_probe * (budget_s / probe_s))))
    rows = np.sort(rng.choice(T, size=n, replace=False)).astype(np.int64)
    q_bits[rows] = q_rows_fn(rows)
    t0 = time.perf_counter()
    orc.forward(rows)
    run_s = time.perf_counter() - t0
    # selected pairs of exactly these rows (same closed form as the GPU count)
    pos = rows - w.cu[np.searchsorted(w.cu, rows, side="right") - 1]
    i = pos // w.B
    pairs = int(((np.minimum(w.k, i + 1) - 1) * w.B + (pos - i * w.B + 1)).sum())
    flops = 4.0 * w.d * pairs * w.Hq
    secs = run_s + pool_s * (n / T)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": Oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d query rows x %d heads of %s (%.1f s forward + block-mean pooling "
                      "prorated %.3f of %.1f s)" % (n, w.Hq, w.name, run_s, n / T, pool_s),
            "seconds": secs}


# ----------------------------------------------------------------- arms
def run_reference(args, w):
    """The oracle as it stands, each step a bounded sample of the workload (CPU)."""
    import torch
    import synthetic as S
    from oracle import bf16_bits
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    q, k, v = S.make_qkv(w, "cpu")
    kb, vb = bf16_bits(k), bf16_bits(v)
    qb_full = bf16_bits(q)
    del q, k, v
    qfn = lambda rows: qb_full[rows]
    for _ in range(args.warmup):
        cpu_baseline(w, qfn, kb, vb, budget_s=2.0)
    res = []
    for s in range(args.steps):
        res.append(cpu_baseline(w, qfn, kb, vb, budget_s=args.ref_step_seconds, seed=100 + s))
    secs = sum(r["seconds"] for r in res)
    value = float(np.mean([r["value"] for r in res]))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "tokens": w.T, "q_heads": w.Hq, "kv_heads": w.Hkv,
                       "head_dim": w.d, "block_size": w.B, "top_k": w.k},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res[0]["cores"],
                             "kind": "oracle", "sample": res[0]["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_moba(args, w):
    import torch
    import block_sparse_long_07_b200 as moba
    import synthetic as S

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=dev)
        pg = dist

    ranks = RankGroup(pg, dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    q, k, v = S.make_qkv(w, dev, seed=rank_seed(w, rank))
    T = w.T
    varlen = not w.batch_mode
    if varlen:
        cu = torch.tensor(w.cu, dtype=torch.int32, device=dev)
        p = moba.make_params(1, 0, w.Hq, w.Hkv, w.d, w.B, w.k)
        size_fn = lambda n: moba.workspace_size_varlen(p, T, len(w.lengths), n)
    else:
        b, N = len(w.lengths), w.lengths[0]
        q, k, v = (x.view(b, N, x.shape[1], x.shape[2]) for x in (q, k, v))
        p = moba.make_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
        size_fn = lambda n: moba.workspace_size(p, n)
    budget = (moba.DEFAULT_WS_BUDGET if args.ws_budget_gb is None
              else int(args.ws_budget_gb * (1 << 30)))
    hp = moba.pick_heads_per_pass(size_fn, w.Hkv, budget)
    ws = moba.alloc_workspace(size_fn(hp), dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.Hq, T) if varlen else (len(w.lengths), w.Hq, w.lengths[0]),
                      dtype=torch.float32, device=dev)

    route = getattr(args, "route", "gate")
    if route != "gate" and varlen:
        raise SystemExit("--route other than gate takes a batch workload")
    rsel = None
    if route != "gate":
        rsel = torch.empty(len(w.lengths), w.Hq, w.lengths[0], w.k, dtype=torch.int32,
                           device=dev)

    def step():
        if varlen:
            moba.forward_varlen(q, k, v, cu, w.B, w.k, ws=ws, out=o, lse=lse)
        elif route == "gate":
            moba.forward(q, k, v, w.B, w.k, ws=ws, out=o, lse=lse)
        elif route == "minmax":
            moba.forward_minmax(q, k, v, w.B, w.k, ws=ws, out=o, lse=lse, sel_out=rsel)
        else:  # window / sink: the static selection is part of the step
            moba.static_selection(len(w.lengths), w.lengths[0], w.Hq, w.B, w.k,
                                  moba.ROUTE_WINDOW if route == "window" else moba.ROUTE_SINK,
                                  sel=rsel)
            moba.forward_selected(q, k, v, rsel, w.B, w.k, ws=ws, out=o, lse=lse)

    pairs, routed_pairs = selected_pairs(w)
    flops = flops_of_pairs(pairs, w)
    routed_flops = flops_of_pairs(routed_pairs, w)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = moba.last_device_status(ws)
    if status != 0:
        raise RuntimeError("device status %d after warm-up" % status)

    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    moba.profile_enable(True)
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    kern = moba.profile_read()
    moba.profile_enable(False)
    status = moba.last_device_status(ws)  # the timed steps' device checks
    if status != 0:
        print("device status %d after the timed steps" % status, file=sys.stderr)
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local)
    value = whole_job_rate(world, flops, ms) / 1e12

    peaks, peak_src = load_peaks()
    peak_tf = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    r_launch, r_ms = kern.get("attn_routed", (0, 0.0))
    rl = None
    if r_launch:
        achieved = routed_flops * args.steps / (r_ms / 1e3) / 1e12
        entries_per_launch = routed_pairs * w.Hq / w.B * args.steps / r_launch
        traffic = load_traffic("attn_routed", entries_per_launch)
        rl = {"bound": "tensor", "kernel": "attn_routed", "achieved": achieved,
              "peak": peak_tf, "unit": "TFLOP/s", "frac": achieved / peak_tf,
              "peak_source": "%s bf16_tflops_sustained (kernel runs inside a long step)" % peak_src,
              "traffic": traffic, "launches_per_step": r_launch / args.steps,
              "ms_per_launch": r_ms / r_launch,
              "flops_per_launch": routed_flops * args.steps / r_launch}
    launches = int(sum(n for n, _ in kern.values()))
    kernels_ms = {name: round(t / args.steps, 4) for name, (n, t) in kern.items() if n}

    # ---- dense causal comparator (k = n), same N
    dense_ms = None
    if not args.no_dense:
        dws = moba.alloc_workspace(moba.full_causal_workspace_size(T, len(w.lengths)), dev)

        def dstep():
            if varlen:
                moba.full_causal_varlen(q, k, v, cu, ws=dws, out=o, lse=lse)
            else:
                moba.full_causal(q, k, v, ws=dws, out=o, lse=lse)

        for _ in range(args.dense_warmup):
            dstep()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(args.dense_steps):
            dstep()
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = max_over_ranks(e0.elapsed_time(e1) / args.dense_steps)
        del dws

    # ---- end to end: pinned host inputs in, O / lse out, every step
    e2e = None
    if not args.no_e2e:
        try:
            qh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
            kh = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
            vh = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
            oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
            lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
            qh.copy_(q)
            kh.copy_(k)
            vh.copy_(v)
            h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
            d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

            if not varlen and route == "gate":
                # the library's host-buffer call: copies inside, overlapped with the work
                hbuf = moba.alloc_workspace(moba.forward_host_buffer_size(p, hp), dev)

                def estep():
                    moba.forward_host(qh, kh, vh, w.B, w.k, oh, lh, dev_buf=hbuf)
            else:
                def estep():
                    q.copy_(qh, non_blocking=True)
                    k.copy_(kh, non_blocking=True)
                    v.copy_(vh, non_blocking=True)
                    step()
                    oh.copy_(o, non_blocking=True)
                    lh.copy_(lse, non_blocking=True)

            estep()
            torch.cuda.synchronize()
            barrier()
            n_e = args.steps  # the same number of timed steps as the device-resident value
            e0.record(stream)
            for _ in range(n_e):
                estep()
            e1.record(stream)
            torch.cuda.synchronize()
            ems = max_over_ranks(e0.elapsed_time(e1) / n_e)
            e2e = {"value": whole_job_rate(world, flops, ems) / 1e12, "unit": "TFLOP/s",
                   "ms_per_step": ems, "steps": n_e, "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h,
                   "call": ("moba_forward_host (copies inside the call)"
                            if not varlen and route == "gate" else
                            "host copies + moba_forward")}
            e2e_status = moba.last_device_status(hbuf) if (not varlen and route == "gate") else 0
            if e2e_status != 0:
                e2e["device_status"] = e2e_status
            del qh, kh, vh, oh, lh
        except RuntimeError as exc:  # pinned allocation refused
            e2e = {"value": None, "unit": "TFLOP/s", "error": str(exc)[:200]}

    # ---- CPU baseline (oracle), rank 0, single GPU only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        from oracle import bf16_bits
        kb = bf16_bits(k.reshape(T, w.Hkv, w.d))
        vb = bf16_bits(v.reshape(T, w.Hkv, w.d))
        qflat = q.reshape(T, w.Hq, w.d)

        def qfn(rows):
            r = torch.as_tensor(rows, device=dev)
            return bf16_bits(qflat[r])

        cpu = cpu_baseline(w, qfn, kb, vb, budget_s=args.cpu_seconds)
        cpu.pop("seconds", None)

    status = moba.last_device_status(ws)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "tokens": T, "sequences": len(w.lengths),
                       "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
                       "block_size": w.B, "top_k": w.k, "heads_per_pass": hp,
                       **({} if route == "gate" else {"route": route}),
                       "l2": "inputs larger than L2 (no flush)",
                       "parallelism": "replicas x%d (independent problems)" % world},
            "moba_ms": ms, "dense_ms": dense_ms,
            "speedup_vs_dense": (dense_ms / ms) if dense_ms else None,
            "pct_bf16_peak": 100.0 * (value / world) / peak_tf,
            "flops_per_step": flops, "dense_flops": flops_of_pairs(dense_pairs(w), w),
            "roofline": rl, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "kernels_ms_per_step": kernels_ms, "clocks": clk, "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0 if status == 0 else 1


# ----------------------------------------------------------------- decode
def decode_bytes(sel, N, B, Hkv, G, d):
    """Algorithmic HBM bytes of one decode step of a batch of sequences of N
    tokens: K and V of the union of the blocks the q heads of each kv head
    chose (a block shared by several heads is read once), the block means the
    gate scores, and the new token's q / o / lse."""
    b, Hq, k = sel.shape
    i = (N - 1) // B
    keys = 0
    for s in range(b):
        for g in range(Hkv):
            for j in set(sel[s, g * G:(g + 1) * G].ravel().tolist()) - {-1}:
                keys += min(N, (j + 1) * B) - j * B
    kv = keys * d * 2 * 2
    kbar = b * Hkv * i * d * 4
    io = b * Hq * (d * 2 * 2 + 4)
    return kv, kv + kbar + io


def run_decode(args, w):
    """One decode step per sequence: the workload's K / V are the cache, the
    new token is each sequence's last, the block-mean cache is built before
    timing (a prefill leaves it) and updated for the completed block inside
    every step."""
    import torch
    import block_sparse_long_07_b200 as moba
    import synthetic as S

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=dev)
        pg = dist
    if not w.batch_mode:
        raise SystemExit("decode mode takes a batch workload")
    b, N = len(w.lengths), w.lengths[0]
    G = w.Hq // w.Hkv
    q, k, v = S.make_qkv(w, dev, seed=rank_seed(w, rank))
    kc = k.view(b, N, w.Hkv, w.d)
    vc = v.view(b, N, w.Hkv, w.d)
    qd = q.view(b, N, w.Hq, w.d)[:, N - 1].contiguous()
    del q
    lens = torch.full((b,), N, dtype=torch.int32, device=dev)
    p = moba.make_decode_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
    ws = moba.alloc_workspace(moba.decode_workspace_size(p), dev)
    kbar = moba.alloc_kbar_cache(kc, w.B)
    moba.kbar_cache_update(kc, lens, kbar, w.B, ws=ws)
    o = torch.empty_like(qd)
    lse = torch.empty(b, w.Hq, dtype=torch.float32, device=dev)
    sel = torch.empty(b, w.Hq, w.k, dtype=torch.int32, device=dev)

    def step(qin=qd):
        moba.kbar_cache_update(kc, lens, kbar, w.B, only_last=True, ws=ws)
        moba.decode(qin, kc, vc, lens, kbar, w.B, w.k, ws=ws, out=o, lse=lse, sel_out=sel)

    ranks = RankGroup(pg, dev)
    barrier, max_over_ranks = ranks.barrier, ranks.max

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = moba.last_device_status(ws)
    if status != 0:
        raise RuntimeError("device status %d after warm-up" % status)
    kv_bytes, algo_bytes = decode_bytes(sel.cpu().numpy(), N, w.B, w.Hkv, G, w.d)

    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    moba.profile_enable(True)
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    kern = moba.profile_read()
    moba.profile_enable(False)
    status = moba.last_device_status(ws)  # the timed steps' device checks
    if status != 0:
        print("device status %d after the timed steps" % status, file=sys.stderr)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    value = whole_job_rate(world, b, ms)

    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    a_launch, a_ms = kern.get("decode_attn", (0, 0.0))
    rl = None
    if a_launch:
        achieved = kv_bytes * args.steps / a_launch / (a_ms / a_launch / 1e3) / 1e9
        rl = {"bound": "hbm", "kernel": "decode_attn", "achieved": achieved, "peak": hbm,
              "unit": "GB/s", "frac": achieved / hbm,
              "peak_source": "%s hbm_gbs (copy bandwidth)" % peak_src, "traffic": None,
              "bytes_per_launch": kv_bytes, "ms_per_launch": a_ms / a_launch}
    launches = int(sum(n for n, _ in kern.values()))
    kernels_ms = {name: round(t / args.steps, 5) for name, (n, t) in kern.items() if n}

    # ---- end to end: the new token's q from pinned host memory, o and lse back
    e2e = None
    if not args.no_e2e:
        qh = qd.cpu().pin_memory()
        oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        qdev = torch.empty_like(qd)

        def estep():
            qdev.copy_(qh, non_blocking=True)
            step(qdev)
            oh.copy_(o, non_blocking=True)
            lh.copy_(lse, non_blocking=True)

        for _ in range(args.warmup):
            estep()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            estep()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1) / args.steps)
        e2e = {"value": whole_job_rate(world, b, ems), "unit": "steps/s", "ms_per_step": ems,
               "h2d_bytes_per_step": qh.numel() * qh.element_size(),
               "d2h_bytes_per_step": oh.numel() * oh.element_size() +
               lh.numel() * lh.element_size()}

    cpu = None
    if rank == 0 and not args.no_cpu:
        from oracle import bf16_bits
        cpu = cpu_decode_baseline(w, bf16_bits(qd.view(b, 1, w.Hq, w.d)), bf16_bits(k),
                                  bf16_bits(v), budget_s=args.cpu_seconds)
    if rank == 0:
        line = {"metric": DECODE_METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "us_per_step": 1e3 * ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "decode_" + w.name, "context_tokens": N, "sequences": b,
                           "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
                           "block_size": w.B, "top_k": w.k,
                           "l2": "chosen blocks' K / V ({:.0f} MB) exceed L2; no flush".format(
                               kv_bytes / 1e6),
                           "parallelism": "replicas x%d (independent problems)" % world},
                "algorithmic_bytes_per_step": algo_bytes,
                "roofline": rl, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "kernels_ms_per_step": kernels_ms, "clocks": clk, "device_status": status}
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0 if status == 0 else 1


BACKWARD_METRIC = "MoBA backward (dq, dk, dv over the forward's selection) ms & TFLOP/s at 1M tokens"


def run_backward(args, w):
    """The backward of the prefill's attention: one forward (untimed) gives
    o, lse and the selection; each timed step is one moba_backward.  FLOPs:
    2.5x the forward's 4*d per selected pair (S, dP, dQ, dK, dV against S, PV),
    recomputation not counted."""
    import torch
    import block_sparse_long_07_b200 as moba
    import synthetic as S

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        raise SystemExit("backward mode runs on one GPU")
    if not w.batch_mode:
        raise SystemExit("backward mode takes a batch workload")
    b, N = len(w.lengths), w.lengths[0]
    q, k, v = S.make_qkv(w, dev)
    q, k, v = (x.view(b, N, x.shape[1], x.shape[2]) for x in (q, k, v))
    sel = torch.empty(b, w.Hq, N, w.k, dtype=torch.int32, device=dev)
    o, lse = moba.forward(q, k, v, w.B, w.k, sel_out=sel)
    g = torch.Generator(device=dev).manual_seed(99)
    dO = torch.randn(o.shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    p = moba.make_params(b, N, w.Hq, w.Hkv, w.d, w.B, w.k)
    hp = moba.pick_heads_per_pass(lambda n: moba.backward_workspace_size(p, n), w.Hkv)
    ws = moba.alloc_workspace(moba.backward_workspace_size(p, hp), dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def step():
        moba.backward(q, k, v, o, lse, dO, sel, w.B, w.k, ws=ws, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = moba.last_device_status(ws)
    if status != 0:
        raise RuntimeError("device status %d after warm-up" % status)
    pairs, _ = selected_pairs(w)
    flops = 2.5 * flops_of_pairs(pairs, w)
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    clocks.start()
    moba.profile_enable(True)
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    kern = moba.profile_read()
    moba.profile_enable(False)
    status = moba.last_device_status(ws)
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_src = load_peaks()
    peak_tf = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    value = flops / (ms / 1e3) / 1e12
    line = {"metric": BACKWARD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "backward_" + w.name, "tokens": w.T, "q_heads": w.Hq,
                       "kv_heads": w.Hkv, "head_dim": w.d, "block_size": w.B, "top_k": w.k,
                       "heads_per_pass": hp, "l2": "inputs larger than L2 (no flush)"},
            "flops_per_step": flops,
            "roofline": {"bound": "tensor", "kernel": "whole backward", "achieved": value,
                         "peak": peak_tf, "unit": "TFLOP/s", "frac": value / peak_tf,
                         "peak_source": "%s bf16_tflops_sustained" % peak_src, "traffic": None},
            "gpu_launches": int(sum(n for n, _ in kern.values())),
            "kernels_ms_per_step": {nm: round(t / args.steps, 4) for nm, (n, t) in kern.items()
                                    if n},
            "clocks": clk, "device_status": status}
    print(json.dumps(line), flush=True)
    return 0 if status == 0 else 1


def cpu_decode_baseline(w, qdec_bits, k_bits, v_bits, budget_s=15.0):
    """The oracle on the decode rows (every sequence's last token, all heads),
    repeated for about budget_s seconds; the block means are computed once
    beforehand, as the GPU path keeps them in its cache."""
    from oracle import Oracle
    b, N = len(w.lengths), w.lengths[0]
    q_bits = np.zeros((w.T, w.Hq, w.d), dtype=np.uint16)  # lazily backed; decode rows set
    rows = np.array([s * N + N - 1 for s in range(b)], dtype=np.int64)
    q_bits[rows] = qdec_bits.reshape(b, w.Hq, w.d)
    orc = Oracle(q_bits, k_bits, v_bits, w.cu, w.Hq, w.Hkv, w.d, w.B, w.k)
    orc.block_means()
    n, t0 = 0, time.perf_counter()
    while True:
        orc.forward(rows)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    secs = (time.perf_counter() - t0) / n
    return {"value": b / secs, "unit": "steps/s", "cores": Oracle.num_threads(),
            "kind": "oracle", "seconds": secs,
            "sample": "%d decode steps of %d sequence(s) x %d heads at %d context tokens "
                      "(block means precomputed)" % (n, b, w.Hq, N)}


def run_decode_reference(args, w):
    import synthetic as S
    from oracle import bf16_bits
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    b, N = len(w.lengths), w.lengths[0]
    q, k, v = S.make_qkv(w, "cpu")
    qd = q.view(b, N, w.Hq, w.d)[:, N - 1].contiguous()
    qb, kb, vb = bf16_bits(qd), bf16_bits(k), bf16_bits(v)
    del q, k, v
    for _ in range(args.warmup):
        cpu_decode_baseline(w, qb, kb, vb, budget_s=0.5)
    res = [cpu_decode_baseline(w, qb, kb, vb, budget_s=args.ref_step_seconds / 4)
           for _ in range(args.steps)]
    secs = float(np.mean([r["seconds"] for r in res]))
    value = b / secs
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * secs, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode_" + w.name, "context_tokens": N, "sequences": b,
                       "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
                       "block_size": w.B, "top_k": w.k},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": res[0]["cores"],
                             "kind": "oracle", "sample": res[0]["sample"]},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="moba", choices=["moba", "reference"])
    ap.add_argument("--workload", default="prefill_1m")
    ap.add_argument("--dense-steps", type=int, default=1)
    ap.add_argument("--dense-warmup", type=int, default=1)
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ws-budget-gb", type=float, default=None,
                    help="workspace budget (default: the binding's, 32 GiB)")
    ap.add_argument("--ref-step-seconds", type=float, default=20.0)
    ap.add_argument("--mode", default="prefill", choices=["prefill", "decode", "backward"])
    ap.add_argument("--route", default="gate", choices=["gate", "minmax", "window", "sink"],
                    help="prefill selection: the mean-pooled gate (the method), or a variant")
    args = ap.parse_args()
    import synthetic as S
    if args.workload.endswith("_k32"):
        w = S.WORKLOADS[args.workload[:-4]].with_k(32)
    else:
        w = S.WORKLOADS[args.workload]
    if args.mode == "backward":
        return run_backward(args, w)
    if args.mode == "decode":
        if args.impl == "reference":
            return run_decode_reference(args, w)
        return run_decode(args, w)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_moba(args, w)


if __name__ == "__main__":
    sys.exit(main())
