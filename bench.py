#!/usr/bin/env python
"""ZHA decode benchmark on B200: microseconds per decode step per layer.

A step is one pass of the decode hot path over one batch: append the new
token to the KV cache and the tree (zha_tree_append), then route and attend
the step's queries (zha_decode).  The default workload is the deep tree at
256K context (GQA 32/4, d=128, bf16, block 4, 6 levels, 16 reference
queries, p=0.95, batch 1), synthetic and seeded.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl zha|reference] [--workload NAME]
  python bench.py --profile [--workload NAME] [--n N] [--warmup W] [--steps K]   (untimed decodes, for ncu)
  python bench.py --sweep [N,N,...] [--steps K] [--warmup W]   (light sweep 32K..4M: ZHA vs dense, crossover)

One JSON line on stdout (rank 0).  Timing: CUDA events on the launching
stream around every step (and around the decode call alone), the L2 flushed
before every step (a 2x L2-sized write outside the timed events), warm-up
steps untimed, max over ranks.  Algorithmic bytes of the decode call are
counted from the nodes each query head scored and the keys it attended,
taking the union over each GQA group (the bytes the method has to move), on
untimed repeats of the timed decodes (one per query set).  With --gpus N > 1 every rank runs
an independent replica (the path does not shard across GPUs here).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "ZHA decode µs/layer (build+route+attend) at 256K-4M ctx; % of HBM roofline"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["zha", "reference"], default="zha")
    ap.add_argument("--workload", default="deep256k_bf16")
    ap.add_argument("--n", type=int, default=None, help="context length for the sweep workload")
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--dense-steps", type=int, default=30)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="build the workload's tree, run --warmup + --steps decodes untimed, exit (for ncu)")
    ap.add_argument("--multi", type=int, default=0,
                    help="with --profile: route --multi queries at once (zha_route_multi) instead of decoding; "
                         "without: time it and print one line")
    ap.add_argument("--sweep", nargs="?", const="32768,65536,131072,262144,524288,1048576,2097152,4194304",
                    default=None, help="run the light sweep workload at these context lengths (one process each) "
                                       "and print one line per N plus the measured dense/ZHA crossover")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        # NCCL between the GPU replicas; gloo lets the host-only reference arm run under torchrun on CPU
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------------ measured traffic
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic_deep256k.txt")


def kernel_source_hash() -> str:
    """Hash of the CUDA sources of the library (a traffic figure is valid only for the kernels it measured)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tree_indexed_sparse_03_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload_name: str):
    """DRAM bytes (read + write) of one decode call from the committed ncu summary, if it measured these
    kernels on this workload; else None."""
    try:
        vals = {}
        with open(TRAFFIC_FILE) as fh:
            for line in fh:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("workload") != workload_name or vals.get("source_hash") != kernel_source_hash():
            return None
        return int(float(vals["dram_bytes_per_decode"]))
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------------ workload
def load_workload(args):
    from synth.workloads import workload
    w = workload(args.workload, args.n) if args.n else workload(args.workload)
    return w


def union_bytes(w, scored: np.ndarray, nscored: np.ndarray, kept: np.ndarray, kcnt: np.ndarray, n_tokens: int):
    """Algorithmic bytes of one decode call: union over each GQA group of the planes scored and keys attended."""
    es = 2 if w.dtype == "bf16" else 4
    # mu and intercepts of a node (f is not read by routing); FP4 router planes: codes, scales, intercepts
    plane = w.n_refs * (w.d // 2 + w.d // 16 + 4) if w.planes == "fp4" else w.n_refs * (w.d * es + 4)
    kv = 2 * w.d * es
    n1 = n_tokens // w.block
    tail = n_tokens - n1 * w.block
    route = attend = 0
    keys_per_head = []
    B, Hq = kcnt.shape
    G = w.group
    for b in range(B):
        for g in range(w.n_kv_heads):
            hs = range(g * G, (g + 1) * G)
            codes = np.unique(np.concatenate([scored[b, h, : min(int(nscored[b, h]), scored.shape[2])] for h in hs]))
            route += codes.size * plane
            leaves = np.unique(np.concatenate([kept[b, h, : int(kcnt[b, h])] for h in hs]))
            toks = leaves.size * w.block + tail + (0 if (n1 == 0 or (leaves.size and leaves[0] == 0)) else 1)
            attend += toks * kv
            for h in hs:
                lk = int(kcnt[b, h])
                has0 = lk and (kept[b, h, :lk] == 0).any()
                keys_per_head.append(lk * w.block + tail + (0 if (n1 == 0 or has0) else 1))
    qo = B * Hq * w.d * (es + 4)
    return route, attend + qo, keys_per_head


# ------------------------------------------------------------------ oracle (CPU) arm
def oracle_sample(w, inp, n_tokens, budget_s, q_sets):
    """Time the fp64 oracle's route + attend on a bounded sample; return (us per full step, desc, threads)."""
    import oracle.zha_oracle as zo
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        threads = 1
    Kh = inp.K[0, :n_tokens].double().numpy()
    Vh = inp.V[0, :n_tokens].double().numpy()
    tree = zo.build_tree(Kh, inp.refs[0].double().numpy(), n_tokens, w.block, w.levels)
    pfn = zo.tree_planes_fn(tree)
    p = float(np.float32(w.p))
    per_head = []
    t_start = time.perf_counter()
    s = 0
    while time.perf_counter() - t_start < budget_s and s < 64:
        for h in range(w.group):
            q = inp.Q[s % q_sets, 0, h].double().numpy()
            t0 = time.perf_counter()
            zo.decode_head(Kh, Vh, pfn, q, p, n_tokens, w.block, w.levels)
            per_head.append(time.perf_counter() - t0)
        s += 1
    us = statistics.mean(per_head) * w.n_q_heads * w.batch * 1e6
    desc = (f"{len(per_head)} (query head, query set) decodes of KV head 0 at N={n_tokens}, oracle tree of that "
            f"head built beforehand (untimed); mean per head x {w.n_q_heads * w.batch} heads per step; "
            f"one-token append not included")
    if w.planes != "key":
        desc += "; the oracle routes on the unquantised slopes (its FP4 quantiser is not on this timed path)"
    return us, desc, threads


def parity_sample(w, inp, tree, Qs, runs):
    """Parity of the timed path on a bounded sample (KV head 0's query heads, the first timed query sets, on
    the final tree), outside the timed region: the oracle's route on the GPU-stored planes (exact heads and
    heads excused at a boundary of the cut), the oracle's attention on the GPU's kept blocks, and the whole
    path against the oracle's own tree built in fp64 from the raw keys (kept-set Jaccard, output error)."""
    import oracle.zha_oracle as zo
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity_helpers import compare_route, end_to_end, f64, oracle_attend_on_sets

    t0 = time.perf_counter()
    n = tree.size
    p = float(np.float32(w.p))
    heads = list(range(w.group))  # the query heads of KV head 0
    otree = zo.build_tree(f64(inp.K[0, :n]), f64(inp.refs[0]), n, w.block, w.levels)
    out = {"sample": f"query heads 0-{w.group - 1} (KV head 0), batch element 0, query sets "
                     f"{[r[0] for r in runs]}, N={n}", "heads": 0, "exact": 0, "flagged": 0, "failed": 0}
    jac, err, err_m, att, kept_mass = [], [], [], 0.0, []
    for qi, O, kept, cnt in runs:
        Q = Qs[qi].cpu()
        rep = compare_route(tree, Q, kept, cnt, p, n, w.block, w.levels, w.group, heads=heads)
        out["heads"] += rep.heads
        out["exact"] += rep.exact
        out["flagged"] += rep.flagged
        out["failed"] += len(rep.failures)
        ref = oracle_attend_on_sets(inp.K, inp.V, Q[:1], kept[:1], cnt[:1], n, w.block, w.group, heads=heads)
        att = max(att, float(np.abs(O[0, heads].numpy() - ref[0, heads]).max()))
        e2e = end_to_end(inp.K, inp.V, inp.refs, Q, O, kept, cnt, n, w.block, w.levels, p, w.group, 0, (0,),
                         oracle_tree=otree)
        jac += e2e.jaccard
        kept_mass += e2e.retained
        err += e2e.err
        err_m += e2e.err_matched
    out["attend_max_abs_err"] = att
    out["e2e_jaccard"] = round(float(np.mean(jac)), 5) if jac else None
    out["e2e_jaccard_min"] = round(float(np.min(jac)), 5) if jac else None
    out["e2e_matched_sets"] = len(err_m)
    out["max_abs_err"] = float(np.max(err)) if err else None
    out["max_abs_err_matched"] = float(np.max(err_m)) if err_m else None
    # estimated attention mass the oracle's routes keep over the whole descent, against the product of the
    # step thresholds that bounds it from below
    out["retained_mass_mean"] = round(float(np.mean(kept_mass)), 5) if kept_mass else None
    out["retained_mass_min"] = round(float(np.min(kept_mass)), 5) if kept_mass else None
    out["retained_mass_bound"] = round(p ** w.levels, 5)
    out["seconds"] = round(time.perf_counter() - t0, 1)
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return
    from synth.workloads import generate
    w = load_workload(args)
    inp = generate(w)
    n = w.n_tokens
    budget = max(5.0, min(120.0, 2.0 * (args.steps + args.warmup)))
    us, desc, threads = oracle_sample(w, inp, n, budget, w.n_query_sets)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us, 3), "unit": "us", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1000, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n_tokens": n, "block": w.block, "levels": w.levels, "n_refs": w.n_refs,
                   "p": w.p, "batch": w.batch, "gqa": f"{w.n_q_heads}/{w.n_kv_heads}", "d": w.d},
        "cpu_baseline": {"value": round(us, 3), "unit": "us", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(us, 3), "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ profiling mode
def run_profile(args):
    """Build the workload's tree and run decodes without timing, so a profiler can capture the kernels."""
    import tree_indexed_sparse_03_b200 as z
    from synth.workloads import generate

    w = load_workload(args)
    dev = torch.device("cuda", 0)
    inp = generate(w)
    n = w.n_tokens
    cfg = z.make_config(d=w.d, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, block=w.block, levels=w.levels,
                        n_refs=w.n_refs, p=w.p, dtype=w.dtype, capacity=n, max_batch=w.batch,
                        planes=w.planes)
    tree = z.ZhaTree(cfg, inp.K.to(dev), inp.V.to(dev), inp.refs.to(dev))
    tree.build(n)
    Qs = inp.Q.to(dev)
    if args.multi:
        from synth.workloads import random_queries
        Qm = random_queries(1, args.multi, w.n_q_heads, w.d, w.dtype, topics_from=inp).to(dev)
        for i in range(args.warmup + args.steps):
            tree.route_multi(Qm)
        torch.cuda.synchronize(dev)
        tree.status()
        log(f"[bench] profile mode: {args.warmup + args.steps} multi-query routes of {args.multi} queries")
        return
    for i in range(args.warmup + args.steps):
        tree.decode(Qs[i % w.n_query_sets])
    torch.cuda.synchronize(dev)
    tree.status()
    log(f"[bench] profile mode: {args.warmup + args.steps} decodes of {w.name} (N={n}), "
        f"{args.warmup} first, {args.steps} after")


# ------------------------------------------------------------------ GPU arm
def run_zha(args, world, rank, local):
    import tree_indexed_sparse_03_b200 as z
    from synth.workloads import generate

    w = load_workload(args)
    dev = torch.device("cuda", local if world > 1 else 0)
    n_build = w.n_tokens
    n0 = n_build + w.append  # context after the workload's own block append (if any)
    total_steps = args.warmup + args.steps + args.e2e_steps + 2
    t_gen = time.perf_counter()
    inp = generate(w, n_total=n0 + total_steps)
    log(f"[bench] generated {w.name} in {time.perf_counter() - t_gen:.1f}s")
    cap = n0 + total_steps
    cfg = z.make_config(d=w.d, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, block=w.block, levels=w.levels,
                        n_refs=w.n_refs, p=w.p, dtype=w.dtype, capacity=cap, max_batch=w.batch,
                        planes=w.planes)
    dt = inp.K.dtype
    K = torch.zeros(w.n_kv_heads, cap, w.d, dtype=dt, device=dev)
    V = torch.zeros_like(K)
    K[:, :n_build] = inp.K[:, :n_build].to(dev)
    V[:, :n_build] = inp.V[:, :n_build].to(dev)
    # per-step new tokens, each [Hkv, 1, d] contiguous
    Kn = inp.K[:, n0:].permute(1, 0, 2).contiguous().unsqueeze(2).to(dev)
    Vn = inp.V[:, n0:].permute(1, 0, 2).contiguous().unsqueeze(2).to(dev)
    Qs = inp.Q.to(dev)
    tree = z.ZhaTree(cfg, K, V, inp.refs.to(dev))
    stream = torch.cuda.current_stream(dev)

    # full build (reported separately; not part of a decode step): the first build loads the build kernels,
    # the second one, over the same tokens, is timed
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tree.build(n_build)
    torch.cuda.synchronize(dev)
    flush_b = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_b.zero_()
    e0.record(stream)
    tree.build(n_build)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    tree.status()
    del flush_b
    build_ms = e0.elapsed_time(e1)
    es_b = 2 if w.dtype == "bf16" else 4
    rec_b = w.n_refs * w.d * es_b + ((w.n_refs * 4 + 15) // 16) * 16
    build_bytes = n_build * w.n_kv_heads * w.d * es_b + sum(
        (n_build // w.block ** l) * w.n_kv_heads * (rec_b + 4 * w.n_refs) for l in range(1, w.levels + 1))
    append_block = None
    if w.append > 0:  # the workload's block append, timed once (new rows and newly complete nodes)
        Ka = inp.K[:, n_build:n0].contiguous().to(dev)
        Va = inp.V[:, n_build:n0].contiguous().to(dev)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        tree.append(Ka, Va)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        tree.status()
        append_block = {"tokens": w.append, "us": round(e0.elapsed_time(e1) * 1000, 3)}

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    O = torch.empty(w.batch, w.n_q_heads, w.d, dtype=torch.float32, device=dev)
    step_i = 0

    def one_step(i, q, ev=None):
        nonlocal step_i
        if ev is not None:
            ev[0].record(stream)
        tree.append(Kn[step_i], Vn[step_i])
        if ev is not None:
            ev[1].record(stream)
        tree.decode(q, out=O)
        if ev is not None:
            ev[2].record(stream)
        step_i += 1

    for i in range(args.warmup):
        flush.zero_()
        one_step(i, Qs[i % w.n_query_sets])
    torch.cuda.synchronize(dev)
    tree.status()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    route_b, attend_b, keys_ph = [], [], []
    launches0 = z.launch_count()
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index or 0) as clk:
        for i in range(args.steps):
            flush.zero_()
            q = Qs[(args.warmup + i) % w.n_query_sets]
            one_step(i, q, events[i])
        torch.cuda.synchronize(dev)
    barrier(world)
    launches = z.launch_count() - launches0
    tree.status()
    step_ms = [ev[0].elapsed_time(ev[2]) for ev in events]
    dec_ms = [ev[1].elapsed_time(ev[2]) for ev in events]
    app_ms = [ev[0].elapsed_time(ev[1]) for ev in events]

    # untimed repeat of each timed decode's query on the final tree for the byte counts; the scored-node
    # export is sized from the heads' own counters (a first decode with the counters alone)
    n_final = tree.size
    parity_runs = []  # (query set, O, kept, cnt) of the first repeats, for the oracle's parity sample
    for i in range(min(args.steps, w.n_query_sets)):
        qi = (args.warmup + i) % w.n_query_sets
        q = Qs[qi]
        _, st0 = tree.decode(q, want_stats=True)
        torch.cuda.synchronize(dev)
        scored_cap = max(1, int(st0[..., z.STAT_NODES_SCORED].max()))
        O_i, (kept, cnt), stats, scored = tree.decode(q, want_kept=True, want_stats=True, scored_cap=scored_cap)
        torch.cuda.synchronize(dev)
        assert int(stats[..., z.STAT_NODES_SCORED].max()) <= scored_cap
        mk = max(1, int(cnt.max()))
        rb, ab, kph = union_bytes(w, scored.cpu().numpy(), stats[..., 0].cpu().numpy(), kept[..., :mk].cpu().numpy(),
                                  cnt.cpu().numpy(), n_final)
        route_b.append(rb)
        attend_b.append(ab)
        keys_ph.extend(kph)
        if len(parity_runs) < 2:
            parity_runs.append((qi, O_i.cpu(), kept.cpu(), cnt.cpu()))
    alg_bytes = statistics.mean(route_b) + statistics.mean(attend_b)

    # end to end through the C ABI with pinned host buffers (copies inside the timed region)
    es = 2 if w.dtype == "bf16" else 4
    qh = torch.empty(w.batch, w.n_q_heads, w.d, dtype=dt).pin_memory()
    kh = torch.empty(w.n_kv_heads, w.d, dtype=dt).pin_memory()
    vh = torch.empty(w.n_kv_heads, w.d, dtype=dt).pin_memory()
    oh = torch.empty(w.batch, w.n_q_heads, w.d, dtype=torch.float32).pin_memory()
    e2e_ms = []
    for i in range(args.e2e_steps):
        qh.copy_(inp.Q[i % w.n_query_sets])
        kh.copy_(inp.K[:, n0 + step_i])
        vh.copy_(inp.V[:, n0 + step_i])
        flush.zero_()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        tree.decode_step_host(kh, vh, qh, oh)
        b_.record(stream)
        b_.synchronize()
        step_i += 1
        e2e_ms.append(a.elapsed_time(b_))
    tree.status()
    h2d = (qh.numel() + kh.numel() + vh.numel()) * es
    d2h = oh.numel() * 4

    # dense decode at the same context length (the comparator)
    dense = z.DenseDecoder(cfg, w.batch, tree.size, device=dev)
    dense_ms = []
    for i in range(args.dense_steps + 3 if args.dense_steps > 0 else 0):
        flush.zero_()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dense(K, V, tree.size, Qs[i % w.n_query_sets], out=O)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        if i >= 3:
            dense_ms.append(a.elapsed_time(b_))
    dense_bytes = 2 * tree.size * w.n_kv_heads * w.d * es + w.batch * w.n_q_heads * w.d * (es + 4)

    step_ms_mean = statistics.mean(step_ms)
    step_ms_max = max_over_ranks(sum(step_ms), world) / args.steps
    dec_mean = statistics.mean(dec_ms)
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = alg_bytes / (dec_mean * 1e-3) / 1e9
    res = {
        "metric": METRIC,
        "value": round(step_ms_max * 1000, 3),
        "unit": "us",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms_max, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "n_tokens": n0, "block": w.block, "levels": w.levels, "n_refs": w.n_refs,
                   "p": w.p, "batch": w.batch, "gqa": f"{w.n_q_heads}/{w.n_kv_heads}", "d": w.d,
                   "router_planes": w.planes, "built": n_build, "step": "append 1 token + route + attend", "l2": "flushed before every step",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "queries": f"{w.n_query_sets} seeded query sets, rotated"},
        "median_us": round(statistics.median(step_ms) * 1000, 3),
        "p10_us": round(float(np.percentile(step_ms, 10)) * 1000, 3),
        "p90_us": round(float(np.percentile(step_ms, 90)) * 1000, 3),
        "decode_us": round(dec_mean * 1000, 3),
        "append_us": round(statistics.mean(app_ms) * 1000, 3),
        "dense_us": round(statistics.mean(dense_ms) * 1000, 3) if dense_ms else None,
        "speedup_vs_dense": round(statistics.mean(dense_ms) / step_ms_mean, 3) if dense_ms else None,
        "dense_gbs": round(dense_bytes / (statistics.mean(dense_ms) * 1e-3) / 1e9, 1) if dense_ms else None,
        "build_ms": round(build_ms, 3),
        "build_gbs": round(build_bytes / (build_ms * 1e-3) / 1e9, 1),
        "append_block": append_block,
        "keys_per_head": round(statistics.mean(keys_ph), 1),
        "keys_frac": round(statistics.mean(keys_ph) / n_final, 6),
        "route_bytes": int(statistics.mean(route_b)),
        "attend_bytes": int(statistics.mean(attend_b)),
        "roofline": {"bound": "hbm",
                     "kernel": "zha_decode call: per routing step a scoring and a select kernel, then the "
                               "attention and combine kernels",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "frac_of_8tbs": round(achieved / 8000.0, 4), "traffic": measured_traffic(w.name),
                     "algorithmic_bytes": int(alg_bytes)},
        "clocks": clk.summary(),
        "e2e": ({"value": round(statistics.mean(e2e_ms) * 1000, 3), "unit": "us", "h2d_bytes_per_step": h2d,
                 "d2h_bytes_per_step": d2h} if e2e_ms else None),
        "gpu_launches": launches,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle leg: the CPU baseline timing, then the parity sample (untimed, after the GPU timing)
        us, desc, threads = oracle_sample(w, inp, n0, args.cpu_seconds, w.n_query_sets)
        res["cpu_baseline"] = {"value": round(us, 1), "unit": "us", "cores": 1, "kind": "oracle",
                               "sample": desc + f"; effectively one thread: the oracle's route is a Python loop "
                                               f"(numpy's BLAS pool has {threads} threads; the one-thread run "
                                               f"below takes the same time)",
                               "blas_threads": threads}
        try:  # the same sample with the BLAS pool limited to one thread
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                us1, desc1, _ = oracle_sample(w, inp, n0, min(args.cpu_seconds, 6.0), w.n_query_sets)
            res["cpu_baseline_1t"] = {"value": round(us1, 1), "unit": "us", "cores": 1, "kind": "oracle",
                                      "sample": desc1}
        except ImportError:
            pass
        res["parity"] = parity_sample(w, inp, tree, Qs, parity_runs)
    if rank == 0:
        print(json.dumps(res), flush=True)
    del tree


def run_multi(args):
    """Multi-query routing (zha_route_multi) of --multi queries on the workload's tree: time per call and per
    query against the same queries through zha_decode in groups of max_batch, one JSON line (not the
    decode metric)."""
    import tree_indexed_sparse_03_b200 as z
    from synth.workloads import generate, random_queries

    w = load_workload(args)
    dev = torch.device("cuda", 0)
    inp = generate(w)
    n = w.n_tokens
    mb = max(1, 1024 // w.n_q_heads)
    cfg = z.make_config(d=w.d, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, block=w.block, levels=w.levels,
                        n_refs=w.n_refs, p=w.p, dtype=w.dtype, capacity=n, max_batch=mb, planes=w.planes)
    tree = z.ZhaTree(cfg, inp.K.to(dev), inp.V.to(dev), inp.refs.to(dev))
    tree.build(n)
    Qm = random_queries(1, args.multi, w.n_q_heads, w.d, w.dtype, topics_from=inp).to(dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, reps):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps * 1000

    def per_decode():
        for q0 in range(0, args.multi, mb):
            tree.decode(Qm[q0:q0 + mb])

    reps = max(1, args.steps)
    us_multi = timed(lambda: tree.route_multi(Qm), reps)
    us_dec = timed(per_decode, reps)
    tree.status()
    print(json.dumps({"metric": "multi-query routing (route + attend of m queries of one context)",
                      "workload": w.name, "n_tokens": n, "queries": args.multi, "max_batch": mb,
                      "route_multi_us": round(us_multi, 2), "us_per_query": round(us_multi / args.multi, 3),
                      "decode_groups_us": round(us_dec, 2),
                      "speedup_first_step_contraction": round(us_dec / us_multi, 3)}), flush=True)


def run_sweep(args):
    """The light sweep: one bench process per context length, then the dense/ZHA crossover."""
    lines = []
    for n in [int(x) for x in args.sweep.split(",") if x]:
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", "sweep_bf16", "--n", str(n),
               "--steps", str(args.steps), "--warmup", str(args.warmup), "--e2e-steps", "0",
               "--dense-steps", str(max(args.dense_steps, 5)), "--no-cpu-baseline"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            log(r.stderr[-2000:])
            raise SystemExit(f"sweep point N={n} failed")
        line = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
        lines.append(line)
        print(json.dumps({"sweep_point": n, "decode_us": line["decode_us"], "dense_us": line["dense_us"],
                          "speedup_vs_dense": round(line["dense_us"] / line["decode_us"], 3),
                          "keys_per_head": line["keys_per_head"], "roofline_frac": line["roofline"]["frac"],
                          "levels": line["config"]["levels"], "clocks": line["clocks"]}), flush=True)
    cross = crossover([(ln["config"]["n_tokens"], ln["decode_us"], ln["dense_us"]) for ln in lines])
    print(json.dumps({"sweep": "light sweep bf16 (GQA 32/4, d=128, b=8, R=1, p=0.75, batch 1)",
                      "crossover_n": cross, "unit": "us per decode call"}), flush=True)


def crossover(points):
    """Context length from which the routed decode is faster than the dense one: points are
    (N, routed us, dense us) in increasing N; the last sign change of dense - routed from negative to
    non-negative, interpolated linearly in log N; "<= N0" if routed is never slower; None if never faster."""
    cross = None
    for (na, ra, da), (nb, rb, db) in zip(points, points[1:]):
        ga, gb = da - ra, db - rb
        if ga < 0 <= gb:
            la, lb = math.log(na), math.log(nb)
            cross = int(round(math.exp(la + (lb - la) * (-ga) / (gb - ga))))
    if points and cross is None and all(d >= r for _, r, d in points):
        cross = f"<= {points[0][0]}"
    return cross


def main():
    args = parse_args()
    if args.sweep:
        run_sweep(args)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.profile:
            run_profile(args)
        elif args.multi:
            run_multi(args)
        else:
            run_zha(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
