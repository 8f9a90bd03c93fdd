#!/usr/bin/env python
"""Benchmark of the PIVOT-Refine indexer at L=131072 on B200.

One step = one PIVOT-Refine call (proxy build, tcgen05 prefix scan with fused
filter, exact candidate select, per-member refine) over the long-context
prefill workload: L=131072, H=16, d=128, g=16, top_k=2048, Kc=4096, bf16,
seeded synthetic inputs (heavy-tailed keys, AR(1) queries).  The metric is
indexed query-heads per second (L*H per step), aggregated over all GPUs.  On N
GPUs the heads of the one layer are split: rank r indexes heads
[r*H/N, (r+1)*H/N) (strong scaling; heads are independent, so there is no
collective on the data path, only the barriers and the max over ranks of the
timing).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  `--impl reference` times the CPU oracle
(the plain fp64 restatement of the method) on a bounded sample of the same
workload on the host cores.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "PIVOT-Refine indexed queries/s at L=131072; fraction of tensor/HBM roofline"
UNIT = "query-heads/s"
WORKLOAD = "C3"
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, nominal


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sust=float(p["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


def workload_config(c, world=1):
    return {"workload": f"{WORKLOAD} long-context prefill L={c['L']} H={c['H']} d={c['d']} g={c['g']} "
                        f"top_k={c['top_k']} Kc={c['Kc']} PIVOT-Refine",
            "generator": f"keys N(0,1) with {c['heavy_frac']*100:g}% positions x{c['heavy_scale']:g}; "
                         f"queries AR(1) rho={c['rho']}; seed {c['seed']}",
            "l2": "inputs 1.07 GB and outputs 17.2 GB per step exceed the 126 MB L2; no flush needed",
            "parallelism": (f"heads split across {world} GPUs (rank r: heads [r*H/N, (r+1)*H/N)), "
                            "no collective on the data path")}


def algorithmic(c):
    """Method's own work per step, by kernel (flops or bytes)."""
    L, H, d, g, k, Kc = c["L"], c["H"], c["d"], c["g"], c["top_k"], c["Kc"]
    G = (L + g - 1) // g
    i = np.arange(G, dtype=np.int64)
    last = np.minimum(i * g + g, L) - 1
    scan_flops = 2.0 * d * H * float(last.sum())
    nC = np.minimum(Kc, last)
    return {
        "scan_filter": ("tensor", scan_flops),
        # a select must at least read Kc (key, index) pairs and write Kc indices per row
        "finalize": ("hbm", float(H * nC.sum() * (8 + 4))),
        # output rows + candidate rows + member queries + every key once
        "refine": ("hbm", float(L * H * k * 4 + H * nC.sum() * 4 + 2 * L * H * d * 2)),
        "proxy": ("hbm", float(L * H * d * 2 + G * H * d * 2)),
        "fallback": ("hbm", 0.0),
        "refine_fallback": ("hbm", 0.0),
    }


def config_work(c):
    """The method's own work per call on a prefill workload: compulsory HBM
    bytes (q and k read once, the index rows written once, and for Refine the
    candidate rows written and read once) and the scan's tensor-core flops
    (Refine scans j < last of each group, Reuse j < group start, dense j < pos)."""
    L, H, d, g, k, Kc = c["L"], c["H"], c["d"], c["g"], c["top_k"], c["Kc"]
    G = (L + g - 1) // g
    s = np.arange(G, dtype=np.int64) * g
    last = np.minimum(s + g, L) - 1
    qk = 2 * L * H * d * 2
    out = L * H * k * 4
    nC = np.minimum(Kc, last)
    return {
        "refine": {"bytes": float(qk + out + 2 * H * nC.sum() * 4), "flops": 2.0 * d * H * float(last.sum())},
        "reuse": {"bytes": float(qk + out), "flops": 2.0 * d * H * float(s.sum())},
        "dense": {"bytes": float(qk + out), "flops": 2.0 * d * H * float(np.arange(L, dtype=np.int64).sum())},
    }


def roofline_ms(work, pk):
    """The slower of the HBM and the tensor-core bound, in ms (measured peaks)."""
    return max(work["bytes"] / (pk["hbm"] * 1e9), work["flops"] / (pk["bf16"] * 1e12)) * 1e3


def config_records(qg, torch, stream, pk, steps, names=("C0", "C1", "C2"), member_names=("C0", "C1")):
    """Refine, Reuse and dense on the smaller prefill workloads: ms per call,
    query-heads/s, the fraction of each call's roofline, PIVOT's speedup over
    the dense indexer and Recall@k against it (on a seeded sample of rows).
    On `member_names` also the per-member-scan variant of Refine (each member's
    own top-Kc candidates over its prefix), whose recall change is the point
    of that variant."""
    recs = {}
    for name in names:
        c = synthetic.CONFIGS[name]
        q_np, k_np = synthetic.make_prefill(name)
        q = torch.from_numpy(q_np.view(np.int16)).cuda().view(torch.bfloat16)
        k = torch.from_numpy(k_np.view(np.int16)).cuda().view(torch.bfloat16)
        L, H, d, g, top_k, Kc = c["L"], c["H"], c["d"], c["g"], c["top_k"], c["Kc"]
        outs, ms = {}, {}
        calls = {"refine": lambda o: qg.pivot_index(q, k, g, top_k, Kc, qg.REFINE, out=o),
                 "reuse": lambda o: qg.pivot_index(q, k, g, top_k, Kc, qg.REUSE, out=o),
                 "dense": lambda o: qg.dense_index(q, k, top_k, out=o)}
        if name in member_names:
            calls["refine_member_scan"] = lambda o: qg.pivot_index(q, k, g, top_k, Kc, qg.REFINE, out=o,
                                                                   scan="member")
        for mode, fn in calls.items():
            o = torch.empty((L, H, top_k), dtype=torch.int32, device="cuda")
            for _ in range(2):
                fn(o)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn(o)
            e1.record(stream)
            torch.cuda.synchronize()
            ms[mode] = e0.elapsed_time(e1) / steps
            outs[mode] = o
        qg.sync_status()
        rng = np.random.default_rng(11)
        n = max(256, L * H // 100)
        rows = torch.from_numpy(rng.integers(1, L, size=n)).cuda()
        heads = torch.from_numpy(rng.integers(0, H, size=n)).cuda()
        dn = outs["dense"][rows, heads].cpu().numpy()
        rec = {}
        for mode in [m for m in outs if m != "dense"]:
            pv = outs[mode][rows, heads].cpu().numpy()
            rec[mode] = float(np.mean([np.intersect1d(a[a >= 0], b[b >= 0]).size / max(1, (b >= 0).sum())
                                       for a, b in zip(pv, dn)]))
        work = config_work(c)
        recs[name] = {
            "shape": f"L={L} H={H} d={d} g={g} top_k={top_k} Kc={Kc}",
            "ms": ms,
            "query_heads_per_s": {m: L * H / (v / 1000.0) for m, v in ms.items()},
            "roofline_ms": {m: roofline_ms(work[m], pk) for m in ms if m in work},
            "roofline_frac": {m: roofline_ms(work[m], pk) / ms[m] for m in ms if m in work},
            "speedup_vs_dense": {m: ms["dense"] / v for m, v in ms.items() if m != "dense"},
            "recall_at_k_vs_dense": rec, "recall_rows": int(n)}
        del outs, q, k
        torch.cuda.empty_cache()
    return recs


def measured_traffic(kernel, heads):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, scaled
    from its one-head capture to `heads` (the traffic grows with the heads);
    None when there is no capture or the kernel's source changed since."""
    if kernel != "refine":
        return None
    prof = os.path.join(ROOT, "profiles", "refine_c3_one_head.md")
    src = os.path.join(ROOT, "query_group_top_b200", "csrc", "refine.cuh")
    try:
        fields = dict(line.split(": ", 1) for line in open(prof).read().splitlines() if ": " in line)
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if fields.get("source_sha256_16", "").strip() != digest:
            return None
        return float(fields["traffic_bytes_per_head_launch"]) * heads
    except (OSError, KeyError, ValueError):
        return None


class RankGroup:
    """One process per GPU (or per CPU rank in tests): the barrier and the
    max-over-ranks reduction of the bench's timings.  Every rank takes the same
    collective steps in the same order; rank 0 alone reports."""

    def __init__(self, backend, device):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.device = device
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, x):
        if self.world == 1:
            return x
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()


def job_value(L, H, ms_max):
    """Whole-job throughput: the ranks together index the layer's L x H
    query-heads, and the job takes as long as its slowest rank."""
    return L * H / (ms_max / 1000.0)


def split(n, rank, world):
    """Items [a, b) of n (the decode batch's sequences) that rank `rank` of
    `world` takes: contiguous, in rank order, sizes differing by at most one."""
    return rank * n // world, (rank + 1) * n // world


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_sample(c, q, k, budget_s, threads, seed):
    """The oracle, as it stands, on seeded random (group, head) units of the
    workload, one stream of units per host thread (the oracle is plain C called
    through ctypes, which releases the GIL), until budget_s has passed.
    Returns (query-heads indexed, units, wall seconds, summed per-unit seconds)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    L, H, g = c["L"], c["H"], c["g"]
    G = (L + g - 1) // g

    def worker(w):
        rng = np.random.default_rng([seed, w])
        t0 = time.perf_counter()
        nq = nu = 0
        busy = 0.0
        while time.perf_counter() - t0 < budget_s:
            gi = rng.integers(0, G, size=1).astype(np.int32)
            hi = rng.integers(0, H, size=1).astype(np.int32)
            a = time.perf_counter()
            oracle.prefill_units(q, k, g, c["top_k"], c["Kc"], oracle.REFINE, gi, hi)
            busy += time.perf_counter() - a
            nq += min(int(gi[0]) * g + g, L) - int(gi[0]) * g
            nu += 1
        return nq, nu, busy

    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(worker, range(threads)))
    wall = time.perf_counter() - t0
    return sum(r[0] for r in res), sum(r[1] for r in res), wall, sum(r[2] for r in res)


def cpu_baseline(c, q, k, budget_s=12.0, seed=0):
    """The oracle on all host cores, on a bounded sample of the workload, with
    the full-workload time it implies (extrapolated: units are drawn uniformly,
    so the mean unit time estimates the mean over all units)."""
    cores = host_cores()
    nq, nu, wall, busy = oracle_sample(c, q, k, budget_s, cores, seed)
    L, H, g = c["L"], c["H"], c["g"]
    units = ((L + g - 1) // g) * H
    full_s = busy / max(nu, 1) * units / cores
    return {"value": nq / wall, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{nu} random (group, head) units of {WORKLOAD} ({nq} query-heads) on {cores} threads, "
                      f"single-threaded C oracle per unit, {wall:.1f} s",
            "single_thread_value": nq / busy if busy > 0 else None,
            "full_workload_s_extrapolated": full_s}


def run_reference(args, rank):
    """CPU oracle timed per step on a bounded sample of the workload."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    c = synthetic.CONFIGS[WORKLOAD]
    q, k = synthetic.make_prefill(WORKLOAD)
    cores = host_cores()
    # each step: every host thread indexes random (group, head) units for a
    # bounded time (the whole run stays within a few minutes)
    step_s = max(0.5, min(4.0, 120.0 / max(1, args.steps + args.warmup)))
    for w in range(args.warmup):
        oracle_sample(c, q, k, step_s, cores, seed=1000 + w)
    tot_t, tot_q, tot_u = 0.0, 0, 0
    for s_ in range(args.steps):
        nq, nu, wall, _ = oracle_sample(c, q, k, step_s, cores, seed=2000 + s_)
        tot_t += wall
        tot_q += nq
        tot_u += nu
    value = tot_q / tot_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(c),
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": cores,
                             "sample": f"{tot_u} random (group, head) units of {WORKLOAD} over {args.steps} steps "
                                       f"of {step_s:.1f} s on {cores} threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def decode_only(args, qg, torch):
    """The MTP decode step alone on a few sequences of its workload, then the
    sparse attention over its index rows (a small case for profiling the decode
    kernels and the consumer); prints ms per step of each."""
    dc = synthetic.CONFIGS["C4"]
    B = min(args.decode_only, dc["B"])
    dq, dk, dcu, n_ctx = synthetic.gen_decode_device(dc["B"], dc["H"], dc["d"], dc["g"], dc["seed"], dc["lo"], dc["hi"],
                                                     dc["rho"], dc["heavy_frac"], dc["heavy_scale"], first=0, count=B)
    max_seqlen = int((n_ctx + dc["g"]).max())
    dout = torch.empty((B, dc["g"], dc["H"], dc["top_k"]), dtype=torch.int32, device="cuda")
    step = lambda: qg.pivot_decode_index(dq, dk, dcu, dc["g"], dc["top_k"], dc["Kc"], qg.REFINE, max_seqlen=max_seqlen,
                                         out=dout)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    step_ms = e0.elapsed_time(e1) / args.steps
    qg.sync_status()
    key_bytes = float(n_ctx.astype(np.int64).sum() + B * (dc["g"] - 1)) * dc["H"] * dc["d"] * 2
    # then the sparse attention over the step's index rows (a value cache of
    # the key cache's shape)
    gen_v = torch.Generator(device="cuda")
    gen_v.manual_seed(dc["seed"] * 7 + 1)
    dv = torch.randn(dk.shape, generator=gen_v, device="cuda", dtype=torch.bfloat16)
    att_out = torch.empty((B, dc["g"], dc["H"], dc["d"]), dtype=torch.float32, device="cuda")
    att = lambda: qg.sparse_attention(dq, dk, dv, dout, cu_seqlens=dcu, g=dc["g"], out=att_out)
    for _ in range(args.warmup):
        att()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(args.steps):
        att()
    e1.record()
    torch.cuda.synchronize()
    qg.sync_status()
    print(json.dumps({"decode_only_sequences": B, "ms_per_step": step_ms, "key_bytes": key_bytes,
                      "sparse_attention_ms": e0.elapsed_time(e1) / args.steps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip the Reuse/dense comparison runs")
    ap.add_argument("--e2e-steps", type=int, default=2, help="0 skips the end-to-end measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the CPU oracle")
    ap.add_argument("--no-configs", action="store_true", help="skip the records of the smaller prefill workloads")
    ap.add_argument("--decode-only", type=int, default=0, metavar="B",
                    help="profiling aid: run only the MTP decode step on the first B sequences of its workload")
    ap.add_argument("--heads", type=int, default=0,
                    help="profiling aid: index only this many heads of the workload (0 = all)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch

    import query_group_top_b200 as qg
    qg.load_library()
    torch.cuda.set_device(local)
    ranks = RankGroup("nccl", torch.device("cuda", local))
    barrier, max_over_ranks = ranks.barrier, ranks.max

    if args.decode_only > 0:
        decode_only(args, qg, torch)
        return

    c = dict(synthetic.CONFIGS[WORKLOAD])
    if args.heads > 0:
        c["H"] = min(args.heads, c["H"])
    L, H, d, g, top_k, Kc = c["L"], c["H"], c["d"], c["g"], c["top_k"], c["Kc"]
    if world > H:
        raise SystemExit(f"bench: {world} ranks but only {H} heads to split")
    # every rank draws the same layer and keeps its own heads, as a contiguous
    # [L, nh, d] layer (the layout a head-parallel model holds per GPU)
    h0, h1 = qg.head_range(H, rank, world)
    nh = h1 - h0
    q_all, k_all = synthetic.gen_prefill(L, H, d, c["seed"], c["rho"], c["heavy_frac"], c["heavy_scale"])
    q_np = np.ascontiguousarray(q_all[:, h0:h1])
    k_np = np.ascontiguousarray(k_all[:, h0:h1])
    del q_all, k_all
    cl = dict(c, H=nh)   # this rank's share of the layer
    q = torch.from_numpy(q_np.view(np.int16)).cuda().view(torch.bfloat16)
    k = torch.from_numpy(k_np.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty((L, nh, top_k), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        qg.pivot_index(q, k, g, top_k, Kc, qg.REFINE, out=out)

    for _ in range(args.warmup):
        step()
    qg.sync_status()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    barrier()
    torch.cuda.synchronize()
    qg.trace_enable(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    qg.trace_enable(False)
    trace = qg.trace_collect()
    ms = e0.elapsed_time(e1) / args.steps
    clk = clocks.stop()
    flags = qg.sync_status()
    ms_max = max_over_ranks(ms)
    value = job_value(L, H, ms_max)

    # roofline of the dominant kernel (per launch on this rank's heads)
    pk = peaks()
    alg = algorithmic(cl)
    kern = {name: {"ms_per_launch": tot / max(n, 1), "launches": n, "share": tot / (ms * args.steps)}
            for name, (tot, n) in trace.items()}
    dom = max(trace, key=lambda n: trace[n][0])
    bound, work = alg.get(dom, ("hbm", 0.0))
    t_launch = trace[dom][0] / trace[dom][1] / 1000.0
    if bound == "tensor":
        achieved = work / t_launch / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_sust"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_sust"], "traffic": None, "kernel": dom,
                "peak_note": f"{pk['src']} sustained bf16 dense (kernel timed inside a multi-ms step)"}
    else:
        achieved = work / t_launch / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "traffic": measured_traffic(dom, nh), "kernel": dom,
                "peak_note": f"{pk['src']} HBM copy bandwidth"}
    scan_t = trace.get("scan_filter", (0, 1))
    scan_rec = None
    if scan_t[0]:
        scan_tf = alg["scan_filter"][1] / (scan_t[0] / scan_t[1] / 1000.0) / 1e12
        # the fp32 proxy is scanned exactly as three bf16 terms: three bf16
        # MMAs per key tile carry each algorithmic multiply-add
        scan_rec = {"ms_per_launch": scan_t[0] / scan_t[1], "tflops": scan_tf,
                    "frac_of_bf16_sustained": scan_tf / pk["bf16_sust"],
                    "frac_of_bf16_burst": scan_tf / pk["bf16"],
                    "bf16_mma_terms": 3, "bf16_mma_tflops": 3 * scan_tf,
                    "bf16_mma_frac_of_sustained": 3 * scan_tf / pk["bf16_sust"]}
        # the exact top-Kc select that follows the scan's fused filter
        sel_ms = sum(trace[n][0] / trace[n][1] for n in ("finalize", "fallback") if n in trace)
        scan_rec["select_ms_per_call"] = sel_ms
        scan_rec["select_share_of_scan_and_select"] = sel_ms / (sel_ms + scan_rec["ms_per_launch"])
    gpu_launches = sum(n for _, n in trace.values())

    # end to end through the public API: pinned host inputs -> device -> indexer -> host result
    e2e = None
    try:
        if args.e2e_steps <= 0:
            raise RuntimeError("skipped (--e2e-steps 0)")
        q_h = torch.from_numpy(q_np.view(np.int16)).view(torch.bfloat16).pin_memory()
        k_h = torch.from_numpy(k_np.view(np.int16)).view(torch.bfloat16).pin_memory()
        try:
            out_h = torch.empty((L, nh, top_k), dtype=torch.int32, pin_memory=True)
            pinned = True
        except Exception:
            out_h = torch.empty((L, nh, top_k), dtype=torch.int32)
            pinned = False
        q_d = torch.empty_like(q)
        k_d = torch.empty_like(k)

        def e2e_step():
            q_d.copy_(q_h, non_blocking=True)
            k_d.copy_(k_h, non_blocking=True)
            qg.pivot_index(q_d, k_d, g, top_k, Kc, qg.REFINE, out=out)
            out_h.copy_(out, non_blocking=pinned)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1) / args.e2e_steps)
        e2e = {"value": job_value(L, H, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(q.numel() * 2 + k.numel() * 2),
               "d2h_bytes_per_step": int(out.numel() * 4), "pinned_output": pinned}
        del q_h, k_h, out_h, q_d, k_d
    except Exception as ex:  # pragma: no cover - host memory limits
        e2e = {"value": None, "unit": UNIT, "error": str(ex)[:200]}

    extras = {}
    if not args.no_extras:
        def timed(fn, n):
            fn()
            torch.cuda.synchronize()
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(n):
                fn()
            t1.record(stream)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / n
        out_reuse = torch.empty_like(out)
        reuse_ms = timed(lambda: qg.pivot_index(q, k, g, top_k, Kc, qg.REUSE, out=out_reuse), args.steps)
        out_dense = torch.empty_like(out)
        dense_ms = timed(lambda: qg.dense_index(q, k, top_k, out=out_dense), 1)
        qg.sync_status()
        reuse_ms, dense_ms = max_over_ranks(reuse_ms), max_over_ranks(dense_ms)
        # Recall@k against the dense indexer on a seeded 1% of rows
        rng = np.random.default_rng(7)
        rows = torch.from_numpy(rng.integers(1, L, size=L * nh // 100)).cuda()
        heads = torch.from_numpy(rng.integers(0, nh, size=rows.numel())).cuda()
        dn = out_dense[rows, heads].cpu().numpy()
        rec = {}
        for name, o in (("refine", out), ("reuse", out_reuse)):
            pv = o[rows, heads].cpu().numpy()
            hit = [np.intersect1d(a[a >= 0], b[b >= 0]).size / max(1, (b >= 0).sum()) for a, b in zip(pv, dn)]
            rec[name] = float(np.mean(hit))
        del out_dense
        # MTP decode workload: one step over 64 sequences (keys drawn on the
        # device), the sequences split across the ranks
        dc = synthetic.CONFIGS["C4"]
        b0, b1 = split(dc["B"], rank, world)
        dq, dk, dcu, n_ctx = synthetic.gen_decode_device(dc["B"], dc["H"], dc["d"], dc["g"], dc["seed"],
                                                         dc["lo"], dc["hi"], dc["rho"], dc["heavy_frac"],
                                                         dc["heavy_scale"], first=b0, count=b1 - b0)
        nb = b1 - b0
        max_seqlen = int((n_ctx + dc["g"]).max())
        dout = torch.empty((nb, dc["g"], dc["H"], dc["top_k"]), dtype=torch.int32, device="cuda")
        dstep = lambda: qg.pivot_decode_index(dq, dk, dcu, dc["g"], dc["top_k"], dc["Kc"], qg.REFINE,
                                              max_seqlen=max_seqlen, out=dout)
        for _ in range(2):
            dstep()
        torch.cuda.synchronize()
        qg.trace_enable(True)
        dec_ms = timed(dstep, args.steps)
        qg.trace_enable(False)
        dtr = qg.trace_collect()
        qg.sync_status()
        key_bytes = float(n_ctx.astype(np.int64).sum() + nb * (dc["g"] - 1)) * dc["H"] * dc["d"] * 2
        dscan = dtr.get("decode_scan", (0.0, 1))
        dscan_ms = dscan[0] / max(dscan[1], 1)
        dscan_gbs = key_bytes / (dscan_ms / 1000.0) / 1e9 if dscan_ms else None
        dec_ms_max = max_over_ranks(dec_ms)
        decode = {"workload": f"C4 MTP decode B={dc['B']} n_b~U[{dc['lo']},{dc['hi']}] H={dc['H']} d={dc['d']} "
                              f"g={dc['g']} top_k={dc['top_k']} Kc={dc['Kc']} PIVOT-Refine",
                  "sequences_per_rank": nb, "ms_per_step": dec_ms_max,
                  "query_heads_per_s": dc["B"] * dc["g"] * dc["H"] / (dec_ms_max / 1000.0),
                  "kernels_ms": {k: v[0] / max(v[1], 1) for k, v in dtr.items()},
                  "decode_scan_hbm_gbs": dscan_gbs,
                  # a read-only stream against the nominal HBM3e bandwidth, and
                  # against the measured copy (read + write) bandwidth
                  "decode_scan_hbm_frac": dscan_gbs / NOMINAL_HBM_GBS if dscan_gbs else None,
                  "decode_scan_frac_of_measured_copy": dscan_gbs / pk["hbm"] if dscan_gbs else None,
                  "decode_step_hbm_frac": (key_bytes / (dec_ms / 1000.0) / 1e9) / NOMINAL_HBM_GBS,
                  "key_bytes": key_bytes}
        # the sparse attention that consumes the step's index rows, over a
        # value cache of the key cache's shape (seeded normal values); its
        # algorithmic bytes: every selected key and value row once per query
        # head, plus q, the index rows and the fp32 output
        gen_v = torch.Generator(device="cuda")
        gen_v.manual_seed(dc["seed"] * 7 + 1)
        dv = torch.randn(dk.shape, generator=gen_v, device="cuda", dtype=torch.bfloat16)
        att_out = torch.empty((nb, dc["g"], dc["H"], dc["d"]), dtype=torch.float32, device="cuda")
        att = lambda: qg.sparse_attention(dq, dk, dv, dout, cu_seqlens=dcu, g=dc["g"], out=att_out)
        for _ in range(2):
            att()
        att_ms = timed(att, args.steps)
        qg.sync_status()
        n_valid = int((dout >= 0).sum().item())
        att_bytes = (n_valid * 2 * dc["d"] * 2 + dout.numel() * 4 + dq.numel() * 2 + att_out.numel() * 4)
        decode["sparse_attention"] = {
            "ms": att_ms, "selected_keys": n_valid, "algorithmic_bytes": att_bytes,
            "gbs": att_bytes / (att_ms / 1000.0) / 1e9,
            "hbm_frac_nominal": att_bytes / (att_ms / 1000.0) / 1e9 / NOMINAL_HBM_GBS,
            "note": "gathers of the selected key and value rows; the MTP step's g members select mostly the "
                    "same rows, so part of the gathers hit L2 and the rate can exceed the DRAM bandwidth"}
        del dq, dk, dv, dcu, dout, att_out
        torch.cuda.empty_cache()
        w3 = config_work(cl)
        extras = {"refine_ms": ms_max, "reuse_ms": reuse_ms, "dense_ms": dense_ms, "decode": decode,
                  "speedup_refine_vs_dense": dense_ms / ms_max, "speedup_reuse_vs_dense": dense_ms / reuse_ms,
                  "recall_at_k_vs_dense": rec, "recall_rows": int(rows.numel()),
                  "roofline_ms": {"refine": roofline_ms(w3["refine"], pk), "reuse": roofline_ms(w3["reuse"], pk),
                                  "dense": roofline_ms(w3["dense"], pk)},
                  "roofline_frac": {"refine": roofline_ms(w3["refine"], pk) / ms_max,
                                    "reuse": roofline_ms(w3["reuse"], pk) / reuse_ms,
                                    "dense": roofline_ms(w3["dense"], pk) / dense_ms}}
        del out_reuse
        if not args.no_configs and world == 1:
            del out
            torch.cuda.empty_cache()
            extras["configs"] = config_records(qg, torch, stream, pk, max(3, args.steps))

    if rank == 0:
        import oracle
        oracle.build()
        cpu = cpu_baseline(c, q_np, k_np) if (world == 1 and not args.no_cpu_baseline) else None
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(c, world),
                "roofline": roof, "scan": scan_rec, "kernels": kern, "gpu_launches": gpu_launches,
                "status_flags": flags, "clocks": clk, "e2e": e2e, "cpu_baseline": cpu, "extras": extras}
        print(json.dumps(line), flush=True)
    ranks.close()


if __name__ == "__main__":
    main()
