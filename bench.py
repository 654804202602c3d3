#!/usr/bin/env python
"""Throughput of the ForkAttention hot path: branch-token evals/s.

One step = one pass of the whole path over one batch of synthetic decision
requests already resident in HBM: tree-index build -> fork attention ->
Gated DeltaNet fork scan -> checkpoint save, all through libflide.so's C ABI
on one stream.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on the same workload

Multi-GPU (torchrun): requests are independent, so every rank runs its own
batch (seed offset by rank) with no data-path collective -- weak scaling; the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tree_forked_decision_b200 import flide, inputs  # noqa: E402

METRIC = "branch-token evals/sec (fork attn + GDN layer, 1 B200); % of roofline"
UNIT = "branch-token evals/s"
DEFAULT_WORKLOAD = "large_fanout_bf16"
# fallbacks when the measured-peaks file is absent (earlier measurements on this machine)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# workload arithmetic (measurement only)
# ---------------------------------------------------------------------------

def isolated_positions(tree: inputs.Tree) -> np.ndarray:
    """Length of each token's isolated sequence before it (past + ancestors +
    earlier tokens of its node), from the tree structure."""
    rp, pa, sl, pl = tree.arrays()
    before = np.zeros(tree.N, np.int64)
    for r in range(tree.R):
        for n in range(rp[r], rp[r + 1]):
            before[n] = pl[r] if pa[n] < 0 else before[rp[r] + pa[n]] + sl[rp[r] + pa[n]]
    offs = np.concatenate([np.arange(s) for s in sl]) if tree.N else np.zeros(0, np.int64)
    return np.repeat(before, sl) + offs


def attn_work(tree, a):
    """Algorithmic FLOPs (QK^T + PV over exactly the visible keys) and bytes
    (q, k, v, out once, plus the past rows once) of one fork-attention launch."""
    d, Hq, Hkv = a["d"], a["Hq"], a["Hkv"]
    vis = isolated_positions(tree) + 1
    flops = 4.0 * d * Hq * float(vis.sum())
    es = 2 if a["q"].dtype == torch.bfloat16 else 4
    byts = es * d * (2 * tree.T * Hq + 2 * tree.T * Hkv + 2 * tree.P_past * Hkv)
    return flops, byts


def gdn_work(tree, g, esize=None):
    """Algorithmic bytes of one GDN fork scan: q, k, v, out, g, beta once, one
    fp32 state write per saved node (roots and nodes with children), and one
    state read per parent with children (its checkpoint is broadcast to all
    its branches) and per resumed root.  esize: bytes per q, k, v element when
    they differ from the output's (e4m3 inputs, bf16 output)."""
    H, dk, dv = g["H"], g["dk"], g["dv"]
    es = 2 if g["q"].dtype == torch.bfloat16 else 4
    state = 4 * H * dk * dv
    has_child = np.zeros(tree.N, bool)
    rp = tree.req_node_ptr
    for r in range(tree.R):
        for n in range(rp[r], rp[r + 1]):
            if tree.parent[n] >= 0:
                has_child[rp[r] + tree.parent[n]] = True
    roots = int(np.sum(rp[1:] > rp[:-1]))
    writes = int(has_child.sum()) + roots - int(sum(has_child[rp[r]] for r in range(tree.R) if rp[r + 1] > rp[r]))
    reads = int(has_child.sum()) + int(np.sum(tree.past_len > 0))
    io = (2 * dk + 2 * dv) * es if esize is None else (2 * dk + dv) * esize + dv * es
    return tree.T * H * (io + 8) + state * (writes + reads)


# ---------------------------------------------------------------------------
# device step
# ---------------------------------------------------------------------------

class Step:
    """Device buffers and one call sequence of the hot path."""

    def __init__(self, tree, a, g, device):
        self.tree, self.a, self.g = tree, a, g
        self.dt = flide.DeviceTree(*tree.arrays(), max_depth=max(tree.levels, 1), device=device)
        self.idx = flide.TreeIndex(self.dt.R, self.dt.N, self.dt.T, self.dt.max_depth, device=device)
        dev = lambda t: t.to(device, non_blocking=False).contiguous()
        self.launches = 2
        if a is not None:
            self._init_attn(tree, a, dev, device)
        if g is not None:
            self._init_gdn(tree, g, dev, device)

    def _init_attn(self, tree, a, dev, device):
        self.q, self.k, self.v = dev(a["q"]), dev(a["k"]), dev(a["v"])
        self.pk = dev(a["past_k"]) if a["past_k"].shape[0] else None
        self.pv = dev(a["past_v"]) if a["past_v"].shape[0] else None
        self.o = torch.empty_like(self.q)
        self.scale = 1.0 / math.sqrt(a["d"])
        self.launches += 2
        self.ckpt_rows = tree.P_past + tree.root_tokens
        self.ck = torch.empty((max(self.ckpt_rows, 1), a["Hkv"], a["d"]), dtype=self.k.dtype,
                              device=device)
        self.cv = torch.empty_like(self.ck)
        self.launches += 1

    def _init_gdn(self, tree, g, dev, device):
        self.gq, self.gk, self.gv = dev(g["q"]), dev(g["k"]), dev(g["v"])
        self.gg, self.gb = dev(g["g"]), dev(g["beta"])
        self.state_in = dev(g["state_in"]) if np.any(tree.past_len > 0) else None
        self.go = torch.empty((tree.T, g["H"], g["dv"]), dtype=self.gq.dtype, device=device)
        # node-state capacity: the slots the tree index assigns (roots, plus
        # the inner nodes of the widest odd and even depth)
        self.slots = max(flide.state_slots(tree), 1)
        self.node_state = torch.empty((self.slots, g["H"], g["dv"], g["dk"]), dtype=torch.float32,
                                      device=device)
        self.cS = torch.empty((tree.R, g["H"], g["dv"], g["dk"]), dtype=torch.float32, device=device)
        # per tree level a grouping and a scan launch, then the state save
        self.launches += 2 * (self.dt.max_depth + 1) + 1

    def run(self, ev=None):
        """tree build -> fork attention -> GDN fork scan -> checkpoint save;
        ev = 3 CUDA events recorded around the two layers."""
        a, g = self.a is not None, self.g is not None
        flide.tree_build(self.dt, self.idx)
        if ev is not None:
            ev[0].record()
        if a:
            flide.fork_attn(self.q, self.k, self.v, self.idx, self.scale, past_k=self.pk,
                            past_v=self.pv, out=self.o)
        if ev is not None:
            ev[1].record()
        if g:
            flide.fork_gdn(self.gq, self.gk, self.gv, self.gg, self.gb, self.idx,
                           self.node_state, state_in=self.state_in, out=self.go)
        if ev is not None:
            ev[2].record()
        flide.state_save(self.idx, self.k if a else None, self.v if a else None,
                         self.ck if a else None, self.cv if a else None,
                         self.cS if g else None, past_k=self.pk if a else None,
                         past_v=self.pv if a else None,
                         node_state=self.node_state if g else None)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
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
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleSampler:
    """Times the oracle on seeded uniform samples of the workload's units --
    attention query rows and GDN (request, head) pairs -- and scales each time
    by (all units / sampled units).  The inputs are converted to fp32 once."""

    def __init__(self, tree, a, g):
        import oracle  # test infrastructure: only the CPU-baseline leg and the reference arm use it
        self.oracle, self.tree, self.a, self.g = oracle, tree, a, g
        f32 = lambda t: t.float().numpy()
        if a is not None:
            self.qa, self.ka, self.va = f32(a["q"]), f32(a["k"]), f32(a["v"])
            self.pka, self.pva = f32(a["past_k"]), f32(a["past_v"])
        if g is not None:
            self.gin = {nm: f32(g[nm]) for nm in ("q", "k", "v", "g", "beta")}
            self.st = f32(g["state_in"]) if np.any(tree.past_len > 0) else None

    def attention(self, n, rng):
        """Extrapolated seconds for all query rows, from n sampled rows."""
        tree, a = self.tree, self.a
        n_rows = tree.T * a["Hq"]
        pick = rng.choice(n_rows, size=min(n, n_rows), replace=False)
        rows = np.stack([pick // a["Hq"], pick % a["Hq"]], 1).astype(np.int32)
        t0 = time.perf_counter()
        self.oracle.attention_rows(tree.arrays(), self.qa, self.ka, self.va, self.pka, self.pva,
                                   1.0 / math.sqrt(a["d"]), rows)
        return (time.perf_counter() - t0) * n_rows / len(rows), f"{len(rows)} of {n_rows} attention query rows"

    def gdn(self, n, rng):
        """Extrapolated seconds for all (request, head) pairs, from n sampled pairs."""
        tree, H = self.tree, self.g["H"]
        all_pairs = [(r, h) for r in range(tree.R) for h in range(H)]
        sel = rng.choice(len(all_pairs), size=min(n, len(all_pairs)), replace=False)
        heads = sorted({all_pairs[i][1] for i in sel})
        # slice the selected heads so the oracle reads only their data
        hs = {nm: np.ascontiguousarray(x[:, heads]) for nm, x in self.gin.items()}
        pairs = [(all_pairs[i][0], heads.index(all_pairs[i][1])) for i in sel]
        st = np.ascontiguousarray(self.st[:, heads]) if self.st is not None else None
        t0 = time.perf_counter()
        self.oracle.gdn(tree.arrays(), hs["q"], hs["k"], hs["v"], hs["g"], hs["beta"], state_in=st,
                        memoise=True, pairs=pairs)
        return ((time.perf_counter() - t0) * len(all_pairs) / len(sel),
                f"{len(sel)} of {len(all_pairs)} GDN (request, head) pairs (memoised oracle)")

    def threads(self):
        return self.oracle.num_threads()


def cpu_oracle_rate(tree, a, g, attn_rows: int, gdn_pairs: int, seed: int = 0):
    """One sampled timing of the oracle: (evals/s, description, threads)."""
    smp = OracleSampler(tree, a, g)
    rng = np.random.default_rng(seed)
    t_attn = t_gdn = 0.0
    parts = []
    if a is not None:
        t_attn, d = smp.attention(attn_rows, rng)
        parts.append(d)
    if g is not None:
        t_gdn, d = smp.gdn(gdn_pairs, rng)
        parts.append(d)
    rate = tree.branch_tokens / (t_attn + t_gdn)
    desc = (" and ".join(parts) + f", seeded uniform sample; each time scaled by all/sampled "
            f"units: attention {t_attn:.1f} s + GDN {t_gdn:.1f} s per step extrapolated")
    return rate, desc, smp.threads()


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel_name: str, src_file: str):
    """dram read+write bytes of `kernel_name` per timed unit (one launch for
    attention, one layer = all tree levels for GDN) from the committed ncu
    summary, or None when the kernel source changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel_name]
    except (OSError, ValueError, KeyError):
        return None
    src = os.path.join(ROOT, "tree_forked_decision_b200", "csrc", src_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if rec.get("source_sha") != sha:
        return None
    return rec.get("bytes_per_layer", rec.get("bytes_per_launch"))


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def rank_seed(workload: str, seed, rank: int) -> int:
    """Seed of this rank's batch: ranks serve independent requests (weak
    scaling, no data-path collective), so each draws its own inputs."""
    base = seed if seed is not None else inputs.WORKLOADS[workload]["idx"]
    return base + 1000 * rank


def max_over_ranks(x: float, pg, device) -> float:
    """The job's time is its slowest rank's (a MAX all-reduce)."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def percentiles(xs):
    """(P50, P95) of a list of per-step times (nearest rank)."""
    v = sorted(xs)
    pick = lambda q: v[min(len(v) - 1, max(0, int(math.ceil(q * len(v))) - 1))]
    return pick(0.50), pick(0.95)


def all_ranks(flag: bool, pg, device) -> bool:
    """True only if `flag` holds on every rank (a MIN all-reduce), so that legs
    holding barriers or collectives run on all ranks or on none."""
    return -max_over_ranks(-float(bool(flag)), pg, device) > 0


def job_throughput(units_per_rank: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * steps * world / (ms_max / 1000.0)


def run_reference(args):
    """The oracle as the reference arm: every step times a sample of the
    workload on the host cores and extrapolates to all of it.  The attention
    sample shrinks as steps + warm-up grow (the same total over the run); a GDN
    sample (one (request, head) pair per core, each a whole request's
    sequence) is taken in about 13 of the steps, evenly spread, and the other
    steps reuse the latest GDN time, so any --steps/--warmup run ends within a
    few minutes."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    tree, a, g, dtype = inputs.make_inputs(args.workload, seed=args.seed)
    smp = OracleSampler(tree, a, g)
    total = max(args.steps + args.warmup, 1)
    rows = max(64, args.ref_rows * 13 // total)
    pairs = max(args.ref_pairs, smp.threads())
    t_gdn, gdn_desc, n_gdn = 0.0, "", 0
    rates, desc = [], ""
    t_start = None
    for s_ in range(total):
        if s_ == args.warmup:
            t_start = time.perf_counter()
        rng = np.random.default_rng(2 + s_)
        t_attn, parts = 0.0, []
        if a is not None:
            t_attn, d = smp.attention(rows, rng)
            parts.append(d)
        if g is not None and (s_ == 0 or (s_ * 13) // total != ((s_ - 1) * 13) // total):
            t_gdn, gdn_desc = smp.gdn(pairs, rng)
            n_gdn += 1
        if g is not None:
            parts.append(gdn_desc)
        if s_ >= args.warmup:
            rates.append(tree.branch_tokens / (t_attn + t_gdn))
            desc = (" and ".join(parts) + f" per step (GDN timed in {n_gdn} of {s_ + 1} steps so far, "
                    f"reused between); each time scaled by all/sampled units")
    wall = time.perf_counter() - t_start if t_start is not None else 0.0
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * tree.branch_tokens / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "requests": tree.R, "tokens": tree.T,
                   "branch_tokens": tree.branch_tokens, "seed": args.seed,
                   "oracle": "plain C fp64 oracle (memoised GDN), OpenMP over units"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.threads(), "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)
    return 0


def measure_workload(name, rank, steps, device, pg, local_rank, peak_tflops, hbm_gbs):
    """A few timed steps of another named workload (same call sequence as the
    headline step, rank-seeded batch): ms per step, branch-token evals/s and
    each layer's fraction of its roofline, with the clocks seen meanwhile."""
    tree, a, g, _ = inputs.make_inputs(name, seed=rank_seed(name, None, rank))
    st = Step(tree, a, g, device)
    for _ in range(3):
        st.run()
    torch.cuda.synchronize()
    # at least ~0.4 s of timed steps, so the clock sampler sees the load
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    st.run()
    t1.record()
    torch.cuda.synchronize()
    steps = max(steps, min(2000, int(math.ceil(400.0 / max(t0.elapsed_time(t1), 1e-3)))))
    steps = int(max_over_ranks(float(steps), pg, device))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(steps):
            evs[i][3].record()
            st.run(evs[i])
            evs[i][4].record()
        torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    if st.idx.status() != 0:
        raise SystemExit(f"device status {st.idx.status()} in the {name} timing")
    ws = pg.get_world_size() if pg is not None else 1
    step_ms = max_over_ranks(statistics.mean(e[3].elapsed_time(e[4]) for e in evs), pg, device)
    res = {"ms_per_step": step_ms, "value": job_throughput(tree.branch_tokens, 1, ws, step_ms),
           "unit": UNIT, "steps": steps, "warmup": 3, "requests_per_gpu": tree.R,
           "tokens_per_gpu": tree.T, "branch_tokens_per_gpu": tree.branch_tokens,
           "clocks": clk.summary()}
    if a is not None:
        ams = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in evs), pg, device)
        flops, _ = attn_work(tree, a)
        tf = flops / (ams / 1000.0) / 1e12
        res["fork_attn"] = {"ms": ams, "tflops": tf, "frac": tf / peak_tflops, "bound": "tensor",
                            "algorithmic_flops": flops}
    if g is not None:
        gms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in evs), pg, device)
        gb = gdn_work(tree, g)
        gbs = gb / (gms / 1000.0) / 1e9
        res["fork_gdn"] = {"ms": gms, "gbs": gbs, "frac": gbs / hbm_gbs, "bound": "hbm",
                           "algorithmic_bytes": gb}
    del st
    torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="flide", choices=["flide", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--layers", default="both", choices=["both", "attn", "gdn"],
                    help="profiling aid: run one layer only (not a headline number)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--no-warm", action="store_true", help="skip the resumed-prefix (warm) timing")
    ap.add_argument("--no-decision", action="store_true", help="skip the decision-scoring timing")
    ap.add_argument("--no-history", action="store_true", help="skip the paged history store timing")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 attention timing")
    ap.add_argument("--no-bounded", action="store_true", help="skip the memory-bounded GDN timing")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the short timings of the other bf16 workloads")
    ap.add_argument("--workload-steps", type=int, default=10,
                    help="least timed steps per extra workload (after 3 warm-up steps; more when a "
                         "step is short, for about 0.4 s under load)")
    ap.add_argument("--vocab", type=int, default=8192, help="LM-head vocabulary of the decision leg")
    ap.add_argument("--cpu-rows", type=int, default=6000)
    ap.add_argument("--cpu-pairs", type=int, default=16)
    ap.add_argument("--ref-rows", type=int, default=2000)
    ap.add_argument("--ref-pairs", type=int, default=16)
    args = ap.parse_args()
    if args.steps < 1 or args.warmup < 0 or args.gpus < 1:
        ap.error("--steps and --gpus must be at least 1, --warmup at least 0")
    if args.impl == "reference":
        return run_reference(args)

    ws, rank, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    pg = None
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
        pg = dist
    flide.load()

    seed = rank_seed(args.workload, args.seed, rank)
    tree, a, g, dtype = inputs.make_inputs(args.workload, seed=seed)
    if args.layers == "attn":
        g = None
    elif args.layers == "gdn":
        a = None
    if a is None and g is None:
        raise SystemExit(f"{args.workload}: no layer left to run")
    if args.layers == "both" and (a is None or g is None):
        raise SystemExit(f"{args.workload} lacks one of the two layers; use --layers")
    step = Step(tree, a, g, device)
    torch.cuda.synchronize()

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    # warm-up, then check the path ran clean
    for _ in range(max(args.warmup, 0)):
        step.run()
    torch.cuda.synchronize()
    if step.idx.status() != 0:
        raise SystemExit(f"device status {step.idx.status()} after warm-up")

    # timed region: inputs resident in HBM (GBs per step, far above the 126 MB L2)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local_rank) as clk:
        start.record()
        for i in range(args.steps):
            evs[i][3].record()
            step.run(evs[i])
            evs[i][4].record()
        stop.record()
        torch.cuda.synchronize()
    barrier()
    ms = start.elapsed_time(stop)
    attn_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    gdn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    p50_ms, p95_ms = percentiles([e[3].elapsed_time(e[4]) for e in evs])
    p50_ms, p95_ms = max_over_ranks(p50_ms, pg, device), max_over_ranks(p95_ms, pg, device)
    if step.idx.status() != 0:
        raise SystemExit(f"device status {step.idx.status()} in the timed region")
    ms = max_over_ranks(ms, pg, device)
    value = job_throughput(tree.branch_tokens, args.steps, ws, ms)

    # the same call sequence captured once as a CUDA graph and replayed
    graph = None
    if not args.no_graph:
        side = torch.cuda.Stream(device=device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step.run()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg):
            step.run()
        torch.cuda.synchronize()
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            gev[i][0].record()
            cg.replay()
            gev[i][1].record()
        torch.cuda.synchronize()
        barrier()
        if step.idx.status() != 0:
            raise SystemExit(f"device status {step.idx.status()} in the graph replays")
        g50, g95 = percentiles([e[0].elapsed_time(e[1]) for e in gev])
        g50, g95 = max_over_ranks(g50, pg, device), max_over_ranks(g95, pg, device)
        graph = {"replays": args.steps, "p50_ms": g50, "p95_ms": g95,
                 "value_at_p50": job_throughput(tree.branch_tokens, 1, ws, g50), "unit": UNIT}
        del cg

    # warm: the same batch resumed from this step's checkpoint (past K/V rows
    # and the roots' end states), so only branch tokens are computed
    warm = None
    if not args.no_warm and tree.root_tokens > 0:
        tree_w, keep = inputs.warm_variant(tree)
        ridx = torch.from_numpy(keep)
        a_w = g_w = None
        if a is not None:
            a_w = dict(a, q=a["q"][ridx], k=a["k"][ridx], v=a["v"][ridx],
                       past_k=step.ck[:tree_w.P_past], past_v=step.cv[:tree_w.P_past])
        if g is not None:
            g_w = dict(g, state_in=step.cS, **{nm: g[nm][ridx] for nm in ("q", "k", "v", "g", "beta")})
        wstep = Step(tree_w, a_w, g_w, device)
        for _ in range(max(args.warmup, 0)):
            wstep.run()
        wev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            wev[i][3].record()
            wstep.run(wev[i])
            wev[i][4].record()
        torch.cuda.synchronize()
        barrier()
        if wstep.idx.status() != 0:
            raise SystemExit(f"device status {wstep.idx.status()} in the warm leg")
        w_steps = [e[3].elapsed_time(e[4]) for e in wev]
        w_ms = max_over_ranks(statistics.mean(w_steps), pg, device)
        w50, w95 = percentiles(w_steps)
        warm = {"value": job_throughput(tree_w.branch_tokens, 1, ws, w_ms), "unit": UNIT,
                "ms_per_step": w_ms, "p50_ms": max_over_ranks(w50, pg, device),
                "p95_ms": max_over_ranks(w95, pg, device),
                "attn_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in wev) if a is not None else None,
                "gdn_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in wev) if g is not None else None,
                "resumed_past_rows": tree_w.P_past, "stream_tokens": tree_w.T,
                "note": "prefix resumed from the timed step's checkpoint; branch tokens only"}
        del wstep

    # end to end through the public API with host buffers: H2D of every input
    # from pinned memory, the call sequence, D2H of every branch token's output
    e2e = None
    if not args.no_e2e and a is not None and g is not None:
        host = {}
        for pre, src, names in (("a_", a, ("q", "k", "v", "past_k", "past_v")),
                                ("g_", g, ("q", "k", "v", "g", "beta", "state_in"))):
            for nm in names:
                t = src[nm]
                host[pre + nm] = t.pin_memory() if t.numel() else None
        if step.state_in is None:
            host["g_state_in"] = None
        tree_host = [torch.from_numpy(np.ascontiguousarray(x)).pin_memory() for x in tree.arrays()]
        # branch tokens are not contiguous across requests: gather their rows
        rp = tree.req_node_ptr
        starts = np.concatenate([[0], np.cumsum(tree.seg_len)])
        br_rows = np.concatenate([np.arange(starts[rp[r] + 1], starts[rp[r + 1]])
                                  for r in range(tree.R) if rp[r + 1] > rp[r]]).astype(np.int64)
        br_idx = torch.from_numpy(br_rows).to(device)
        out_a = torch.empty((len(br_rows),) + tuple(step.o.shape[1:]), dtype=step.o.dtype).pin_memory()
        out_g = torch.empty((len(br_rows),) + tuple(step.go.shape[1:]), dtype=step.go.dtype).pin_memory()
        status_h = torch.empty(1, dtype=torch.int32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
        h2d += sum(t.numel() * t.element_size() for t in tree_host)
        d2h = out_a.numel() * out_a.element_size() + out_g.numel() * out_g.element_size() + 4

        # two device buffer sets: step i+1's uploads run on a copy stream while
        # step i computes; every step's own uploads and read-back stay inside
        # the timed region
        sets = [step, Step(tree, a, g, device)]
        br_idx32 = br_idx.to(torch.int32)
        stage = [(torch.empty((len(br_rows),) + tuple(st.o.shape[1:]), dtype=st.o.dtype, device=device),
                  torch.empty((len(br_rows),) + tuple(st.go.shape[1:]), dtype=st.go.dtype, device=device))
                 for st in sets]
        cur = torch.cuda.current_stream(device)
        cs = torch.cuda.Stream(device)
        uploaded = [torch.cuda.Event() for _ in range(2)]
        released = [torch.cuda.Event() for _ in range(2)]
        for ev in released:
            ev.record(cur)

        def upload(b):
            st = sets[b]
            cs.wait_event(released[b])
            with torch.cuda.stream(cs):
                for dst, src in ((st.dt.req_node_ptr, tree_host[0]), (st.dt.parent, tree_host[1]),
                                 (st.dt.seg_len, tree_host[2]), (st.dt.past_len, tree_host[3])):
                    dst.copy_(src, non_blocking=True)
                for dst, nm in ((st.q, "a_q"), (st.k, "a_k"), (st.v, "a_v"), (st.pk, "a_past_k"),
                                (st.pv, "a_past_v"), (st.gq, "g_q"), (st.gk, "g_k"), (st.gv, "g_v"),
                                (st.gg, "g_g"), (st.gb, "g_beta"), (st.state_in, "g_state_in")):
                    if dst is not None:
                        dst.copy_(host[nm], non_blocking=True)
                uploaded[b].record(cs)

        def compute(b):
            st = sets[b]
            cur.wait_event(uploaded[b])
            st.run()
            oa, og = stage[b]
            for dst, srcx in ((oa, st.o), (og, st.go)):
                flide._check(flide._lib().flide_copy_rows(
                    flide._ptr(dst), flide._ptr(srcx), None, flide._ptr(br_idx32), len(br_rows),
                    srcx[0].numel() * srcx.element_size(), flide._stream()), "flide_copy_rows")
            out_a.copy_(oa, non_blocking=True)
            out_g.copy_(og, non_blocking=True)
            status_h.copy_(st.idx.array("status", 1), non_blocking=True)
            released[b].record(cur)

        def e2e_steps(n):
            upload(0)
            for i in range(n):
                if i + 1 < n:
                    upload((i + 1) % 2)
                compute(i % 2)

        e2e_steps(2)
        torch.cuda.synchronize()
        n_e2e = max(2, min(args.steps, 6))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        e0.record()
        cs.wait_event(e0)  # no upload starts before the timed region
        e2e_steps(n_e2e)
        cur.wait_stream(cs)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), pg, device)
        if int(status_h.item()) != 0:
            raise SystemExit(f"device status {int(status_h.item())} in the e2e leg")
        del sets[1]
        e2e = {"value": job_throughput(tree.branch_tokens, n_e2e, ws, ems), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "ms_per_step": ems / n_e2e,
               "h2d_gbs": h2d * n_e2e / (ems / 1000.0) / 1e9,
               "pipeline": "two device buffer sets; step i+1's host-to-device copies (copy stream) "
                           "overlap step i's compute; outputs gathered by flide_copy_rows, read back "
                           "from pinned memory every step"}

    peaks, peak_src = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    kernels, roofline, roofline_gdn = {}, None, None
    if g is not None:
        gbytes = gdn_work(tree, g)
        gdn_gbs = gbytes / (gdn_ms / 1000.0) / 1e9
        kernels["fork_gdn"] = {"ms": gdn_ms, "algorithmic_bytes": gbytes, "gbs": gdn_gbs,
                               "frac_of_hbm_peak": gdn_gbs / hbm, "bound": "hbm"}
        roofline_gdn = roofline = {
            "kernel": "gdn_ws_kernel (GDN fork scan, warp-specialised tcgen05; all tree levels)",
            "bound": "hbm", "achieved": gdn_gbs, "peak": hbm, "unit": "GB/s", "frac": gdn_gbs / hbm,
            "traffic": traffic_for("gdn_ws_kernel", "gdn_tc.cu"),
            "peak_source": f"{peak_src}: HBM copy bandwidth",
            "algorithmic_bytes_per_launch": gbytes, "avg_launch_ms": gdn_ms}
    if a is not None:
        flops, abytes = attn_work(tree, a)
        achieved = flops / (attn_ms / 1000.0) / 1e12
        kernels["fork_attn"] = {"ms": attn_ms, "tflops": achieved,
                                "frac_of_tensor_peak": achieved / peak, "bound": "tensor"}
        # the dominant kernel of the step
        if g is None or attn_ms >= gdn_ms:
            roofline = {
                "kernel": "attn_tc_kernel (fork attention, tcgen05)",
                "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic_for("attn_tc_kernel", "attn_tc.cu"),
                "peak_source": f"{peak_src}: sustained dense bf16 (kernel timed inside a long step)",
                "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": abytes,
                "avg_launch_ms": attn_ms,
            }

    # decision scoring on the step's attention output: log p of every branch
    # token under a random LM head, then the softmax over each request's options
    decision = None
    if not args.no_decision and a is not None and a["q"].dtype == torch.bfloat16 and tree.branch_tokens:
        D, V = step.o[0].numel(), args.vocab
        grng = torch.Generator(device="cpu").manual_seed(seed + 17)
        w_lm = (torch.randn((V, D), generator=grng) / math.sqrt(D)).to(torch.bfloat16).to(device)
        y = torch.randint(0, V, (tree.T,), generator=grng, dtype=torch.int32).to(device)
        h = step.o.view(tree.T, D)
        lp = torch.empty(tree.T, dtype=torch.float32, device=device)
        ws_buf = flide.branch_logprob_workspace(step.idx, V, device=device)
        pth = torch.empty(max(tree.N, 1), dtype=torch.float32, device=device)
        prb = torch.empty_like(pth)

        def dec_step():
            flide.branch_logprob(h, w_lm, y, step.idx, logp=lp, workspace=ws_buf)
            flide.option_probs(step.idx, lp, path_logp=pth, prob=prb)

        for _ in range(max(args.warmup, 1)):
            dec_step()
        dev_ = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            dev_[i][0].record()
            dec_step()
            dev_[i][1].record()
        torch.cuda.synchronize()
        barrier()
        if step.idx.status() != 0:
            raise SystemExit(f"device status {step.idx.status()} in the decision leg")
        d_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in dev_), pg, device)
        dflops = 2.0 * tree.branch_tokens * D * V
        decision = {"ms": d_ms, "tflops": dflops / (d_ms / 1000.0) / 1e12,
                    "frac_of_tensor_peak": dflops / (d_ms / 1000.0) / 1e12 / peak,
                    "algorithmic_flops": dflops, "D": D, "V": V, "options": int(np.sum(prb[:tree.N].cpu().numpy() > 0)),
                    "note": "log p of every branch token under a random bf16 LM head on the attention "
                            "output, path sums and softmax over each request's leaves"}

    # the paged history store: append the step's roots (rows + end states) and
    # gather the histories back as the next step's past (copies: HBM-bound)
    history = None
    if not args.no_history and a is not None and tree.root_tokens > 0:
        from tree_forked_decision_b200.history import HistoryStore
        brows = 256
        nb = sum(-(-int(tree.seg_len[tree.req_node_ptr[r]]) // brows)
                 for r in range(tree.R) if tree.req_node_ptr[r + 1] > tree.req_node_ptr[r]) + tree.R
        gd = g if g is not None else {"H": 0, "dk": 0, "dv": 0}
        store = HistoryStore(nb, brows, tree.R, nb, a["Hkv"], a["d"], H=gd["H"], dk=gd["dk"],
                             dv=gd["dv"], dtype=step.k.dtype, device=device)
        slots = list(range(tree.R))
        ns = step.node_state if g is not None else None
        store.commit(slots, tree, step.idx, step.k, step.v, ns)
        store.resume(slots)
        torch.cuda.synchronize()
        hev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            hev[i][0].record()
            store.resume(slots)
            hev[i][1].record()
        torch.cuda.synchronize()
        barrier()
        if int(store.status.item()) != 0:
            raise SystemExit(f"history store status {int(store.status.item())}")
        h_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in hev), pg, device)
        rows = sum(store.length(s_) for s_ in slots)
        row_b = a["Hkv"] * a["d"] * step.k.element_size()
        st_b = 4 * gd["H"] * gd["dk"] * gd["dv"] * tree.R
        hbytes = 2 * (2 * rows * row_b) + 2 * st_b  # read + write of K, V rows and states
        history = {"gather_ms": h_ms, "rows": rows, "block_rows": brows, "bytes": hbytes,
                   "gbs": hbytes / (h_ms / 1000.0) / 1e9,
                   "frac_of_hbm_peak": hbytes / (h_ms / 1000.0) / 1e9 / hbm,
                   "note": "resume of every request's history (roots of this step) from the block pool "
                           "into packed past K/V and GDN state_in"}
        # the resumed batch (branch tokens only, past = the histories) with its
        # attention reading the past in place from the blocks, against the same
        # attention over the packed copy
        tree_w, keep = inputs.warm_variant(tree)
        # the same legs on every rank (they hold barriers)
        run_paged = all_ranks(tree_w.P_past == rows and a["d"] == 128 and step.q.dtype == torch.bfloat16,
                              pg, device)
        if run_paged:
            ridx = torch.from_numpy(keep).to(device)
            qw, kw, vw = (t[ridx].contiguous() for t in (step.q, step.k, step.v))
            dtw = flide.DeviceTree(*tree_w.arrays(), max_depth=max(tree_w.levels, 1), device=device)
            idxw = flide.TreeIndex(dtw.R, dtw.N, dtw.T, dtw.max_depth, device=device)
            flide.tree_build(dtw, idxw)
            _, pkw, pvw, _ = store.resume(slots)
            ow1 = torch.empty_like(qw)
            ow2 = torch.empty_like(qw)
            pk_run = lambda: flide.fork_attn(qw, kw, vw, idxw, step.scale, past_k=pkw, past_v=pvw, out=ow1)
            pg_run = lambda: store.fork_attn_paged(qw, kw, vw, idxw, step.scale, slots, out=ow2)
            for _ in range(max(args.warmup, 1)):
                pk_run()
                pg_run()
            pev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
            barrier()
            for i in range(args.steps):
                pev[i][0].record()
                pk_run()
                pev[i][1].record()
                pg_run()
                pev[i][2].record()
            torch.cuda.synchronize()
            barrier()
            if idxw.status() != 0:
                raise SystemExit(f"device status {idxw.status()} in the paged attention")
            history.update(
                packed_attn_ms=max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in pev), pg, device),
                paged_attn_ms=max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in pev), pg, device),
                paged_equals_packed=bool(torch.equal(ow1, ow2)),
                paged_note="resumed batch: attention over the packed copy vs past read in place from "
                           "the blocks (flide_fork_attn_paged, no gather)")
        del store

    # e4m3 fork attention on the same tree and values: q, k, v and the past
    # rows quantised with one scale per tensor (past and new K/V rows share
    # one), then the attention on kind::f8f6f4 MMAs.  Both are timed: the
    # quantisation (two HBM passes: amax, then scale + convert) and the
    # attention, against the e4m3 tensor peak = 2 x the measured bf16 one (the
    # nominal dense ratio of the two formats).
    fp8 = None
    attn_ok = a is not None and a["q"].dtype == torch.bfloat16 and a["d"] == 128
    gdn_ok = g is not None and g["q"].dtype == torch.bfloat16 and g["dk"] == 128 and g["dv"] == 128
    if not args.no_fp8 and (attn_ok or gdn_ok):
        att8, gdn8 = {}, {}
        u8g = lambda t: torch.empty(t.shape, dtype=torch.uint8, device=device)
        if attn_ok:
            am = torch.zeros(3, dtype=torch.float32, device=device)
            ds = torch.empty(3, dtype=torch.float32, device=device)
            u8 = lambda t: None if t is None else torch.empty(t.shape, dtype=torch.uint8, device=device)
            q8, k8, v8, pk8, pv8 = u8(step.q), u8(step.k), u8(step.v), u8(step.pk), u8(step.pv)
            o8 = torch.empty_like(step.q)

            def quant():
                for i, (x, px) in enumerate(((step.q, None), (step.k, step.pk), (step.v, step.pv))):
                    flide.amax(x, out=am[i:i + 1])
                    if px is not None:
                        flide.amax(px, out=am[i:i + 1], accumulate=True)
                for i, (x, x8, px, px8) in enumerate(((step.q, q8, None, None), (step.k, k8, step.pk, pk8),
                                                      (step.v, v8, step.pv, pv8))):
                    flide.quantize_e4m3(x, am[i:i + 1], out=x8, descale=ds[i:i + 1])
                    if px is not None:
                        flide.quantize_e4m3(px, am[i:i + 1], out=px8, descale=None)

            def attn8():
                flide.fork_attn_fp8(q8, k8, v8, step.idx, step.scale, ds, past_k=pk8, past_v=pv8, out=o8)

            for _ in range(max(args.warmup, 1)):
                quant()
                attn8()
            qev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
            barrier()
            for i in range(args.steps):
                qev[i][0].record()
                quant()
                qev[i][1].record()
                attn8()
                qev[i][2].record()
            torch.cuda.synchronize()
            barrier()
            if step.idx.status() != 0:
                raise SystemExit(f"device status {step.idx.status()} in the fp8 leg")
            q_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in qev), pg, device)
            a8_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in qev), pg, device)
            flops = attn_work(tree, a)[0]
            elems = sum(t.numel() for t in (step.q, step.k, step.v, step.pk, step.pv) if t is not None)
            qbytes = elems * (2 + 2 + 1)  # amax read, convert read + write
            peak8 = 2.0 * peak
            diff = (o8.float() - step.o.float()).norm() / step.o.float().norm()
            att8 = {"attn_ms": a8_ms, "tflops": flops / (a8_ms / 1000.0) / 1e12, "peak": peak8,
                    "frac_of_tensor_peak": flops / (a8_ms / 1000.0) / 1e12 / peak8,
                    "speedup_vs_bf16_attn": (kernels.get("fork_attn") or {}).get("ms", float("nan")) / a8_ms,
                    "quant_ms": q_ms, "quant_bytes": qbytes, "quant_gbs": qbytes / (q_ms / 1000.0) / 1e9,
                    "quant_frac_of_hbm_peak": qbytes / (q_ms / 1000.0) / 1e9 / hbm,
                    "rel_l2_vs_bf16_output": float(diff)}
        if gdn_ok:
            gam = torch.zeros(3, dtype=torch.float32, device=device)
            gds = torch.empty(3, dtype=torch.float32, device=device)
            gq8, gk8, gv8 = u8g(step.gq), u8g(step.gk), u8g(step.gv)
            go8 = torch.empty_like(step.go)
            ns8 = torch.empty_like(step.node_state)

            def gquant():
                for i, (x, x8) in enumerate(((step.gq, gq8), (step.gk, gk8), (step.gv, gv8))):
                    flide.amax(x, out=gam[i:i + 1])
                    flide.quantize_e4m3(x, gam[i:i + 1], out=x8, descale=gds[i:i + 1])

            def gdn8_run():
                flide.fork_gdn_fp8(gq8, gk8, gv8, step.gg, step.gb, step.idx, ns8, gds,
                                   state_in=step.state_in, out=go8)

            for _ in range(max(args.warmup, 1)):
                gquant()
                gdn8_run()
            gev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
            barrier()
            for i in range(args.steps):
                gev[i][0].record()
                gquant()
                gev[i][1].record()
                gdn8_run()
                gev[i][2].record()
            torch.cuda.synchronize()
            barrier()
            if step.idx.status() != 0:
                raise SystemExit(f"device status {step.idx.status()} in the fp8 GDN leg")
            gq_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in gev), pg, device)
            g8_ms = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in gev), pg, device)
            gb8 = gdn_work(tree, g, esize=1)
            gdn8 = {"gdn_ms": g8_ms, "gdn_algorithmic_bytes": gb8, "gdn_gbs": gb8 / (g8_ms / 1000.0) / 1e9,
                    "gdn_frac_of_hbm_peak": gb8 / (g8_ms / 1000.0) / 1e9 / hbm,
                    "gdn_speedup_vs_bf16": gdn_ms / g8_ms,
                    "gdn_quant_ms": gq_ms,
                    "gdn_rel_l2_vs_bf16_output": float((go8.float() - step.go.float()).norm()
                                                       / step.go.float().norm())}
        fp8 = {**att8, **gdn8,
               "note": "e4m3 q/k/v with per-tensor scales; attention: P rounded to e4m3, fp32 "
                       "accumulation, peak = 2 x measured bf16 (nominal dense e4m3/bf16 ratio); GDN: "
                       "codes converted exactly to bf16 in the kernel, HBM bytes with 1-byte q/k/v"}

    # memory-bounded GDN schedule: the same layer with at most a quarter of the
    # one-shot node-state slots live (roots first, then groups of level-1
    # subtrees resumed from the roots' states); only where the batch has inner
    # nodes below its roots
    bounded = None
    # every rank takes the same legs (each has barriers): the leg runs only if
    # every rank's batch has inner nodes below its roots
    run_bounded = all_ranks(not args.no_bounded and g is not None and flide.state_slots(tree) > tree.R,
                            pg, device)
    if run_bounded:
        from tree_forked_decision_b200.schedule import BoundedGdn, plan_state_groups
        full = flide.state_slots(tree)
        budget = max(-(-full // 4), 1)
        try:
            plan_state_groups(tree, budget)
        except flide.FlideError:
            budget = full
        # the schedule of this tree shape is built once, like the step's index
        bplan = BoundedGdn(tree, budget, g["H"], g["dk"], g["dv"], device=device)
        n_groups = bplan.groups
        bo = torch.empty_like(step.go)

        def bnd():
            bplan.run(step.gq, step.gk, step.gv, step.gg, step.gb, state_in=step.state_in, out=bo)

        for _ in range(max(args.warmup, 1)):
            bnd()
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            bev[i][0].record()
            bnd()
            bev[i][1].record()
        torch.cuda.synchronize()
        barrier()
        if bplan.status() != 0:
            raise SystemExit(f"device status {bplan.status()} in the bounded GDN leg")
        state_b = 4 * g["H"] * g["dk"] * g["dv"]
        bounded = {"ms": max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in bev), pg, device),
                   "one_shot_ms": gdn_ms, "slot_budget": budget, "one_shot_slots": full,
                   "groups": n_groups, "state_bytes": budget * state_b,
                   "one_shot_state_bytes": full * state_b,
                   "rel_l2_vs_one_shot": float((bo.float() - step.go.float()).norm() / step.go.float().norm()),
                   "note": "GDN layer with at most slot_budget node states live: roots, then groups of "
                           "level-1 subtrees resumed from the roots' states (planned once per tree "
                           "shape on the host; timed: row gathers, tree builds, GDN launches, scatters)"}

    # combined roofline of the step: the layers' roofline times summed, over the
    # measured per-step P50
    combined = None
    parts = {}
    if a is not None:
        parts["fork_attn_ms"] = 1000.0 * attn_work(tree, a)[0] / (peak * 1e12)
    if g is not None:
        parts["fork_gdn_ms"] = 1000.0 * gdn_work(tree, g) / (hbm * 1e9)
    if parts:
        rt = sum(parts.values())
        combined = {"roofline_ms": rt, "measured_p50_ms": p50_ms, "frac": rt / p50_ms, "parts": parts,
                    "peaks": "attention: sustained dense bf16; GDN: HBM copy (measured)"}

    # the other bf16 workloads, a few timed steps each (their tree shapes and
    # head counts differ from the headline one: attention-only fan-out, GDN-only
    # fan-out, and the mixed hybrid batch of depth 1-3 trees with resumed requests)
    workloads = None
    if not args.no_workloads and args.layers == "both":
        workloads = {}
        for name in ("attn_fanout_bf16", "gdn_fanout_bf16", "mixed_hybrid_bf16"):
            if name == args.workload:
                continue
            workloads[name] = measure_workload(name, rank, args.workload_steps, device, pg,
                                               local_rank, peak, hbm)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, desc, threads = cpu_oracle_rate(tree, a, g, args.cpu_rows, args.cpu_pairs)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "cpu_model": cpu_model(), "kind": "oracle",
               "sample": desc}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "requests_per_gpu": tree.R, "tokens_per_gpu": tree.T,
                   "branch_tokens_per_gpu": tree.branch_tokens,
                   "attn": f"Hq={a['Hq']} Hkv={a['Hkv']} d={a['d']}" if a is not None else None,
                   "gdn": f"H={g['H']} dk={g['dk']} dv={g['dv']}" if g is not None else None,
                   "layers": args.layers,
                   "l2": "inputs larger than L2 (GBs per step), no flush",
                   "parallelism": f"dp{ws} (independent requests per rank)", "seed": seed},
        "roofline": roofline,
        "roofline_gdn": roofline_gdn,
        "roofline_combined": combined,
        "workloads": workloads,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "p50_ms": p50_ms, "p95_ms": p95_ms,
        "graph": graph,
        "warm": warm,
        "decision": decision,
        "history": history,
        "fp8": fp8,
        "bounded": bounded,
        "gpu_launches": step.launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
