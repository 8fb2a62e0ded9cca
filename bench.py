"""Benchmark of one hybrid CSA/HCA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl cskv|reference]

A step = every row of the hot path on one batch of synthetic input: CSA
compression of the entries the new tokens complete, the Lightning Indexer
scan + exact top-k, CSA attention (top-k + window + sink), HCA compression,
HCA dense attention (+ window + sink), split merges.  Inputs are resident in
HBM.  Prints one JSON line on rank 0.

L2 discipline (--l2): "rotate" (default) keeps R device replicas of the whole
workload and runs their steps round-robin, R chosen so that the other
replicas' step bytes exceed three L2 capacities: every step reads inputs that
are not in L2, and L2 holds what a real model leaves there (mostly clean
lines).  The timed steps replay CUDA graphs that each hold R consecutive steps
(replicas 0..R-1, each step waiting for the one before), as a decode
iteration's layers replay from one graph; the same K steps as single-step
graph replays are reported beside it (single_step_graphs_us_per_step: every
graph launch adds the GPU's per-graph overhead).  "flush" instead writes a
256 MiB buffer before every timed step, outside its events, which leaves L2
full of dirty lines, and replays one single-step graph per step.

--impl reference times the CPU oracle (plain fp64 numpy) on the machine's host
cores on a bounded sample of the same workload.
Multi-GPU (torchrun, N > 1): every rank runs an independent replica of the
workload (weak scaling); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import Workload, spec_by_name  # noqa: E402

METRIC = "hybrid decode attention query-tokens/s at 1M ctx"
UNIT = "query-tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
INDEXER_PROFILE = os.path.join(ROOT, "profiles", "lindex_topk_b1_ctx1m.md")
INDEXER_SOURCES = ("indexer.cu", "sm100.cuh", "common.cuh", "launch.cuh")


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def indexer_digest() -> str:
    """Digest of the sources the indexer kernel is compiled from, comments and blank lines
    left out (a comment edit does not change the kernel the counters were taken on)."""
    h = hashlib.sha256()
    for f in INDEXER_SOURCES:
        with open(os.path.join(ROOT, "compressed_sparse_kv_compress_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes (read + write) per indexer launch from the committed ncu summary, when it
    was taken on this workload and the kernel's sources are unchanged since; else None."""
    if workload != "b1_ctx1m":
        return None
    try:
        with open(INDEXER_PROFILE) as f:
            text = f.read()
    except OSError:
        return None
    dg = re.search(r"source digest: (\w+)", text)
    tb = re.search(r"dram bytes per launch \(read \+ write\): (\d+)", text)
    if not dg or not tb or dg.group(1) != indexer_digest():
        return None
    return int(tb.group(1))


# ---------------------------------------------------------------------- byte model
def step_bytes(w: Workload) -> dict:
    """Algorithmic HBM bytes of one step (what the method must move), per kernel family."""
    m = w.meta
    s = w.spec
    kvb = 2 if s.dtype == "bf16" else 4
    ib = 1 if s.idx_dtype == "fp8" else 4
    row = 256 * kvb
    T, H, Hi, di, k, W = m["T"], m["H"], m["Hi"], m["di"], m["k"], m["W"]
    vis_c = [(p + 1) // 4 for p in m["q_pos"]]
    vis_h = [(p + 1) // 128 for p in m["q_pos"]]
    key = di * ib + (4 if s.idx_dtype == "fp8" else 0)
    idx = sum(v * key for v in vis_c) + T * Hi * key + T * k * 8
    q = H * 128 * kvb
    o = H * 128 * 4 + H * 4
    csa_attn = sum(min(k, v) * row + min(W, p + 1) * row + q + o + k * 4 for v, p in zip(vis_c, m["q_pos"]))
    hca_attn = sum(v * row + min(W, p + 1) * row + q + o for v, p in zip(vis_h, m["q_pos"]))
    comp = 0
    for b in range(m["B"]):
        n = m["n"][b]
        for i in range(m["csa_first"][b], m["csa_first"][b] + m["csa_num"][b]):
            a_tok = min(4, n - 4 * i)
            comp += (a_tok + (4 if i >= 1 else 0)) * 2 * row + row
        for i in range(m["hca_first"][b], m["hca_first"][b] + m["hca_num"][b]):
            comp += min(128, n - 128 * i) * 2 * row + row
    return dict(indexer=idx, csa_attn=csa_attn, hca_attn=hca_attn, compress=comp,
                total=idx + csa_attn + hca_attn + comp)


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu  # nvidia-smi's -i selector: the GPU's UUID (or PCI bus id)
        self.proc = None
        self.path = None

    @staticmethod
    def selector(dev: int) -> str:
        """The CUDA device's identity in a form nvidia-smi -i accepts whatever the two tools'
        numbering: its UUID, else its PCI bus id.  (A CUDA index is relative to
        CUDA_VISIBLE_DEVICES and CUDA's enumeration order, which nvidia-smi does not use.)"""
        props = torch.cuda.get_device_properties(dev)
        try:
            u = str(props.uuid)
            if u:
                return u if u.startswith("GPU-") else f"GPU-{u}"
        except Exception:
            pass
        return f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "gpu": self.gpu}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "gpu": self.gpu}


# ---------------------------------------------------------------------- oracle timing
def oracle_sample(w: Workload, budget_s: float = 12.0, max_queries: int = 64):
    """Times the CPU oracle on whole queries of the workload until the budget is spent."""
    from oracle import step as ostep
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    a = {k: w.numpy(k) for k in w.arrays}
    dt = {"kv": w.spec.dtype, "idx": w.spec.idx_dtype}
    t0 = time.perf_counter()
    done = 0
    for j in range(max_queries):  # cycles over the workload's queries until the budget is spent
        ostep.run_step(w.meta, a, dt, queries=[j % w.meta["T"]])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} whole query step(s) of {w.spec.name} (each: compress of the step's entries, "
                      f"full indexer scan + top-k, CSA and HCA attention), {el:.1f} s"}


# ---------------------------------------------------------------------- bulk compression
def bulk_compress_rate(n: int = 1 << 20, seed: int = 1234, reps: int = 5) -> dict:
    """Compression of a whole n-token cache in one call per layer (CSA 4:1 two streams, HCA
    128:1) from seeded rows generated on the device (x ~ N(0,1)/sqrt(128), z ~ N(0,1), bf16),
    and the pooling of n per-token indexer keys (64 dims, bf16) into E4M3 entry keys:
    algorithmic bytes over event time, against the measured copy bandwidth."""
    from compressed_sparse_kv_compress_b200 import api
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)

    def rows(scale):
        return (torch.randn(n, 256, generator=g, device="cuda") * scale).to(torch.bfloat16)

    xa, za, xb, zb, xh, zh = rows(128 ** -0.5), rows(1.0), rows(128 ** -0.5), rows(1.0), rows(128 ** -0.5), rows(1.0)
    nc, nh = (n + 3) // 4, (n + 127) // 128
    di = 64  # per-token indexer keys -> E4M3 entry keys + scales
    kt = (torch.randn(n, di, generator=g, device="cuda") * di ** -0.5).to(torch.bfloat16)
    k_codes = torch.empty(nc, di, dtype=torch.uint8, device="cuda")
    k_scales = torch.empty(nc, dtype=torch.float32, device="cuda")
    i64 = dict(dtype=torch.int64, device="cuda")
    tok_off, csa_off, hca_off = torch.tensor([0, n], **i64), torch.tensor([0, nc], **i64), torch.tensor([0, nh], **i64)
    out_c = torch.empty(nc, 256, dtype=torch.bfloat16, device="cuda")
    out_h = torch.empty(nh, 256, dtype=torch.bfloat16, device="cuda")
    calls = {
        "csa": (lambda: api.csa_compress(xa, za, xb, zb, tok_off, csa_off, out_c, max_blocks=nc),
                4 * n * 512 + nc * 512),
        "hca": (lambda: api.hca_compress(xh, zh, tok_off, hca_off, out_h, max_blocks=nh), 2 * n * 512 + nh * 512),
        "key_pool": (lambda: api.lindex_pool_keys(kt, tok_off, csa_off, k_codes, k_scales, max_blocks=nc),
                     n * di * 2 + nc * (di + 4)),
    }
    hbm, _ = peaks()
    res = {"n_tokens": n, "data": "seeded normal rows generated on the device"}
    for name, (fn, nbytes) in calls.items():
        for _ in range(2):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        us = a.elapsed_time(b) * 1e3 / reps
        res[f"{name}_us"] = us
        res[f"{name}_gbs"] = nbytes / (us * 1e-6) / 1e9
        res[f"{name}_frac_of_measured_hbm"] = res[f"{name}_gbs"] / hbm
        res[f"{name}_bytes"] = nbytes
    del xa, za, xb, zb, xh, zh, out_c, out_h, kt, k_codes, k_scales
    torch.cuda.empty_cache()
    return res


def combined_rate(bulk: dict, step_bytes: float, step_ms: float, hbm: float) -> dict:
    """Bytes and time of building the whole cache (both compressions) plus one decode step,
    summed: the figure across compress + index/top-k + attention together, beside the two
    it combines."""
    nbytes = bulk["csa_bytes"] + bulk["hca_bytes"] + step_bytes
    us = bulk["csa_us"] + bulk["hca_us"] + step_ms * 1e3
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"bytes": nbytes, "us": us, "gbs": gbs, "frac_of_measured_hbm": gbs / hbm}


# ---------------------------------------------------------------------- distributed
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def reduce_max(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, ws: int, ms_max: float) -> float:
    """Units all ranks processed per second, over the slowest rank's time (weak scaling:
    every rank runs its own replica of the workload)."""
    return units_per_rank * ws / (ms_max / 1e3)


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------- arms
def workload_config(name: str, w: Workload) -> dict:
    """The workload part of the line's config (the same in both arms)."""
    m, spec = w.meta, w.spec
    return {"workload": name, "batch": m["B"], "context": max(m["n"]), "query_tokens_per_step": m["T"],
            "heads": m["H"], "topk": m["k"], "window": m["W"], "indexer": f"{m['Hi']}x{m['di']} {spec.idx_dtype}"}


def run_reference(args, ws, rank):
    if rank != 0:
        return
    w = Workload(spec_by_name(args.workload))
    vals = []
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state
    t0 = time.perf_counter()
    per = []
    for _ in range(args.steps):
        r = oracle_sample(w, budget_s=args.ref_budget, max_queries=1)
        per.append(1.0 / r["value"])
        vals.append(r)
    el = time.perf_counter() - t0
    value = len(per) / sum(per)
    cb = dict(vals[-1])
    cb["value"] = value
    cb["sample"] = f"{len(per)} step(s) of one whole query of {args.workload} each, {el:.1f} s"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(per),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {**workload_config(args.workload, w), "l2": "not applicable (the oracle on host cores)"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def replica_count(args, dev: dict, step_total: int) -> int:
    """Replicas for the rotate discipline: the other R-1 replicas move >= 3 L2 capacities."""
    if args.l2 != "rotate":
        return 1
    l2 = getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "L2_cache_size", 0) or (126 << 20)
    per = sum(v.numel() * v.element_size() for v in dev.values() if torch.is_tensor(v))
    r = math.ceil(3 * l2 / max(step_total, 1)) + 1
    r = min(r, max(2, (40 << 30) // max(per, 1)))  # at most ~40 GB of replicas
    return max(2, r)


def run_cskv(args, ws, rank, local):
    from compressed_sparse_kv_compress_b200 import _lib, api
    from compressed_sparse_kv_compress_b200.step import DecodeStep

    lib = _lib.load()
    spec = spec_by_name(args.workload)
    spec = spec.replace(seed=spec.seed + rank)
    w = Workload(spec)
    m = w.meta
    by = step_bytes(w)
    dev0 = w.device("cuda")
    R = replica_count(args, dev0, by["total"])
    devs = [dev0] + [{k: (v.clone() if torch.is_tensor(v) else v) for k, v in dev0.items()} for _ in range(R - 1)]
    bd = dict(max_csa_blocks=max(m["csa_num"]), max_hca_blocks=max(m["hca_num"]),
              max_csa_visible=max((p + 1) // 4 for p in m["q_pos"]),
              max_hca_visible=max((p + 1) // 128 for p in m["q_pos"]))
    steps = []
    for dev in devs:
        # a prefill chunk's queries are one sequence's consecutive positions (an even count per
        # sequence): the HCA attention takes them in pairs
        st = DecodeStep(dev, k=m["k"], window=m["W"], scale=m["scale"], two_streams=not args.one_stream,
                        adjacent_pairs=m["Q"] >= 2 and m["Q"] % 2 == 0, **bd)
        if spec.cache == "compress":
            st.bulk_compress(max(m["ncsa"]), max(m["nhca"]))
        torch.cuda.synchronize()
        n1 = lib.cskv_launch_count()
        st.capture()
        launches_per_step = (lib.cskv_launch_count() - n1) // 2  # capture() runs the step eagerly, then captures
        steps.append(st)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if args.l2 == "flush" else None
    stream = torch.cuda.current_stream()

    def pre(i):  # what runs before step i, outside its timing
        if flush is not None:
            flush.fill_(i & 0xFF)

    def timed(body, K):
        """Device ms per step of body(i), i < K: one event pair around all K (rotate), or
        one pair per step after an L2 flush outside it (flush)."""
        torch.cuda.synchronize()
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(K):
                body(i)
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / K
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            pre(i)
            evs[i][0].record(stream)
            body(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.mean(x.elapsed_time(y) for x, y in evs)

    for i in range(max(args.warmup, R)):  # every replica's graph runs at least once before timing
        pre(i)
        steps[i % R].replay()
    torch.cuda.synchronize()
    for st in steps:
        if int(st.status.item()) != 0:
            raise RuntimeError(f"device status {int(st.status.item())} during warm-up")

    # ---- the timed steps run from CUDA graphs of consecutive steps, one per replica in turn
    #      (as a decode iteration's layers run from one graph): `chain_all` holds steps 0..R-1,
    #      `chain_part` the first K mod R; K steps = (K div R) x chain_all + chain_part.  Each
    #      step in a graph still waits for the one before (both of its streams).
    def chain_graph(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for st in steps[:n]:
                st.run()
        return g

    chain_all = chain_graph(R)
    n_full, rem = divmod(args.steps, R)
    chain_part = chain_graph(rem) if rem else None
    for _ in range(2):
        chain_all.replay()
        if chain_part is not None:
            chain_part.replay()
    torch.cuda.synchronize()

    def chained_steps():
        for _ in range(n_full):
            chain_all.replay()
        if chain_part is not None:
            chain_part.replay()

    # ---- timed region: K steps
    clocks = ClockSampler(ClockSampler.selector(torch.cuda.current_device()))
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    if flush is None:
        ms_local = timed(lambda i: chained_steps() if i == 0 else None, 1) / args.steps
    else:  # a flush between steps: one single-step graph per step, events around each
        ms_local = timed(lambda i: steps[i % R].replay(), args.steps)
    barrier(ws)
    # the same K steps as K single-step graph replays (each graph launch adds the GPU's
    # per-graph overhead, several microseconds for a two-stream graph)
    ms_single = timed(lambda i: steps[i % R].replay(), args.steps)

    # ---- dominant kernel alone (indexer scan + top-k), same L2 discipline.  (1) back to back:
    #      one graph holding one launch per replica in a row (each a dependent launch of the one
    #      before, as inside a step, so a launch's set-up overlaps the previous kernel), replayed;
    #      the duration per launch is the roofline's denominator.  (2) isolated: one single-launch
    #      graph per replica, an event pair around each replay (that adds the GPU's launch
    #      latency, several microseconds on this part, to the kernel's own time).
    chain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(chain):
        for st in steps:
            st.csa_select()
    idx_graphs = []
    for st in steps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            st.csa_select()
        idx_graphs.append(g)
    torch.cuda.synchronize()
    n_chain = max(1, args.steps // R)
    chain_ms = timed(lambda i: chain.replay(), n_chain)
    idx_us = 1e3 * chain_ms / R
    kev = []

    def one_indexer(i):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        idx_graphs[i % R].replay()
        b.record(stream)
        kev.append((a, b))

    timed(one_indexer, args.steps)
    idx_isolated_us = 1e3 * statistics.mean(a.elapsed_time(b) for a, b in kev)

    # ---- end to end through the public API with host buffers: per step, the step's new
    #      inputs go host -> device from pinned memory and both outputs come back, all in the
    #      step's graph (DecodeStep.capture_io; small transfers zero-copy, large ones by copies)
    def host_pairs(st):
        t = st.t
        pairs = []  # (pinned host tensor, device destination view)

        def add(dst):
            h = torch.empty(dst.shape, dtype=dst.dtype, pin_memory=True)
            h.copy_(dst.cpu())
            pairs.append((h, dst))

        for name in ("q_c", "q_h", "q_idx", "q_scale"):
            if t.get(name) is not None:
                add(t[name])
        for b in range(m["B"]):  # the newest token's rows of every per-token array
            for name, off in (("x_a", "csa_x_off"), ("z_a", "csa_x_off"), ("x_b", "csa_x_off"),
                              ("z_b", "csa_x_off"), ("x_h", "hca_x_off"), ("z_h", "hca_x_off"),
                              ("raw_c", "raw_off"), ("raw_h", "raw_off")):
                r = m[off][b + 1] - 1
                add(t[name][r:r + 1])
            e = m["ncsa"][b] - 1 + m["csa_off"][b]  # the indexer key of the newest entry
            add(t["k_idx"][e:e + 1])
            if t.get("k_scale") is not None:
                add(t["k_scale"][e:e + 1])
        outs = [(st.o_all, torch.empty(st.o_all.shape, dtype=st.o_all.dtype, pin_memory=True))]  # o_c and o_h
        return pairs, outs

    io = [host_pairs(st) for st in steps]
    h2d = sum(h.numel() * h.element_size() for h, _ in io[0][0])
    d2h = sum(h.numel() * h.element_size() for _, h in io[0][1])

    for st, (pairs, outs) in zip(steps, io):  # staged upload, step and read-back in one graph
        st.capture_io(pairs, outs)
    torch.cuda.synchronize()

    def e2e_step(i):
        steps[i % R].replay_io()

    ms_e2e = timed(e2e_step, args.steps)
    # the same end-to-end steps by the host's wall clock: synchronised on both sides, so the
    # figure includes every host-side cost of a replay and of waiting for the read-back
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for i in range(args.steps):
        e2e_step(i)
    torch.cuda.synchronize()
    wall_us = (time.perf_counter() - w0) * 1e6 / args.steps
    clk = clocks.stop()

    ms = reduce_max(ms_local, ws)
    ms_e2e = reduce_max(ms_e2e, ws)
    T = m["T"]
    value = whole_job_rate(T, ws, ms)
    hbm, hbm_src = peaks()
    achieved = by["indexer"] / (idx_us * 1e-6) / 1e9
    if flush is not None:
        l2 = "flushed (256 MiB write) before every timed step, outside its events"
    else:
        l2 = (f"inputs larger than L2: {R} device replicas replayed round-robin "
              f"({R - 1} x {by['total'] / 1e6:.1f} MB of step reads between two reads of a replica)")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if
        spec.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {**workload_config(args.workload, w), "l2": l2,
                   "replay": (f"CUDA graphs of consecutive steps ({R} steps, one per replica, per graph)"
                              if flush is None else "one single-step CUDA graph per step"),
                   "streams": 1 if args.one_stream else 2},
        "single_step_graphs_us_per_step": reduce_max(ms_single, ws) * 1e3,
        "step_hbm_bytes": by["total"], "step_gbs": by["total"] / (ms * 1e-3) / 1e9,
        "step_frac_of_measured_hbm": by["total"] / (ms * 1e-3) / 1e9 / hbm,
        "roofline": {"kernel": "lindex_topk_kernel (indexer scan + top-k)", "bound": "hbm", "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "peak_source": hbm_src,
                     "bytes_per_launch": by["indexer"], "us_per_launch": idx_us,
                     "timing": f"{R * n_chain} launches back to back ({R} replicas in one graph, replayed "
                               f"{n_chain} times), CUDA events",
                     "us_per_isolated_launch": idx_isolated_us,
                     "traffic": profiled_traffic(args.workload)},
        "e2e": {"value": whole_job_rate(T, ws, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "device_us_per_step": ms_e2e * 1e3,
                "host_wall_us_per_step": wall_us,
                "transfer": {"upload": "zero copy" if steps[0].io_zero_copy[0] else "copy + scatter",
                             "read_back": "zero copy" if steps[0].io_zero_copy[1] else "copy"}},
        "gpu_launches": int(launches_per_step) * args.steps,
        "clocks": clk,
    }
    if T >= 256 and spec.idx_dtype == "fp8" and m["Hi"] in (8, 16) and m["di"] in (64, 128):
        # many queries: the indexer runs on the tensor cores (E4M3 products, two passes over the
        # keys); its work against the E4M3 tensor peak (2 x the measured sustained bf16 peak) and
        # against the FP32 pipe (the epilogue's ReLU + weighted head sum: 2 ops per (query,
        # head, entry) and pass)
        tf_bf16 = 1375.3
        try:
            with open(PEAKS_FILE) as f:
                tf_bf16 = float(json.load(f)["bf16_tflops_sustained"])
        except Exception:
            pass
        qhe = sum(m["Hi"] * ((p + 1) // 4) for p in m["q_pos"])  # (query, head, visible entry)
        flops = 2.0 * m["di"] * qhe
        sm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        alu_peak = sm * 128 * 1.965e9  # FP32 lanes x the part's maximum SM clock: ops/s
        t_s = idx_us * 1e-6
        line["prefill_indexer_roofline"] = {
            "bound": "alu", "kernel": "lindex_tc_kernel + exact top-k over the candidate lists",
            "us_per_call": idx_us, "tensor_tflops": flops / t_s / 1e12, "tensor_peak_tflops": 2 * tf_bf16,
            "tensor_frac": flops / t_s / 1e12 / (2 * tf_bf16),
            "alu_ops_per_s": 2 * 2 * qhe / t_s, "alu_peak_ops_per_s": alu_peak,
            "alu_frac": 2 * 2 * qhe / t_s / alu_peak,
            "note": "tensor peak: E4M3 = 2 x measured sustained bf16; alu: FP32 pipe at 1965 MHz"}
    if rank == 0 and ws == 1 and not args.no_bulk:
        line["bulk_compress"] = bulk_compress_rate()
        line["bulk_compress"]["combined_with_one_step"] = combined_rate(line["bulk_compress"], by["total"], ms, hbm)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(w, budget_s=args.ref_budget, max_queries=10000)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del idx_graphs, chain, chain_all, chain_part, steps
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="b1_ctx1m")
    ap.add_argument("--impl", default="cskv", choices=["cskv", "reference"])
    ap.add_argument("--one-stream", action="store_true")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bulk", action="store_true", help="skip the whole-cache compression figures")
    ap.add_argument("--ref-budget", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        else:
            run_cskv(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
