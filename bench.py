"""Benchmark of one token-sparse decode step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole decode path over one batch.  For the default
workload, the 128K shared-index cross-decoder stack (batch 2, one shared cache of
131072 tokens x 8 KV heads, d 128; an indexer scores every token with the
full-dimension q.k, takes one top-2048 per (sequence, KV head), and 8 layers of 32
q heads attend over that index), that is one ``aoh_shared_index_step`` call.  For
the sparse workloads it is the importance scan, the top-N_fac select and focused
attention of every SPARSE KV head (``aoh_sparse_decode``), plus the window
attention of DENSE / STREAM heads when the workload has any.  The metric is KV
tokens scanned per second (sum over sequences of L_b per step, all ranks
together), and the algorithmic HBM bytes per second of the step and of its
dominant kernel against the measured copy bandwidth.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on
the launching stream.  Every step starts with its inputs out of L2: the steps
rotate over R device copies of the inputs, R chosen so that the other copies'
traffic between two uses of a copy is at least twice the L2 size (a step too
small for that at R <= 8 flushes L2 instead, by rewriting a 2 x L2 buffer
outside the events).  Barrier + synchronize on both sides, max over ranks.  Multi-GPU: every rank decodes its own independent batch (weak scaling,
no collective on the data path); NCCL is used only for the barrier and the
max-reduction of the timings.

``--impl reference`` times the float64 CPU oracle on the host cores instead
(same metric and workload, each step a bounded sample of rows), once with one
worker process per core of the process affinity (each limited to one BLAS
thread) and once on a single thread.

``--gpus N`` outside torchrun re-launches this script under
``torch.distributed.run`` with N ranks on this node.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import ROLE_SPARSE, make_workload, preset  # noqa: E402

METRIC = "sparse decode: KV tokens scanned/s/GPU; achieved HBM GB/s vs B200 peak"
DEFAULT_WORKLOAD = "clsa_shared_L128k"
MAX_POOL = 32  # oracle worker processes at most (each holds one float64 row: up to ~0.3 GB)
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------------------ bookkeeping

def algorithmic_bytes(w, in_place: bool = False) -> dict:
    """Bytes the method must move per step (inputs' K / V columns and rows; q and outputs excluded).

    importance scan: 4 * n_dom bytes per (token, SPARSE KV head) with the packed dominant columns,
    2 * d (the K row) when the scan reads K in place (`in_place`);
    focused attention: 4 * d bytes (a K row and a V row) per selected token and KV head;
    DENSE / STREAM heads: 4 * d bytes per attended token; shared index: the indexer's full K rows
    (2 * d bytes per token and head) plus 4 * d per indexed token and head.
    """
    sp = w.spec
    d = sp.head_dim
    L = w.lengths.astype(np.int64)
    roles = w.roles.numpy()
    out = {"tip": 0, "fac": 0, "window": 0, "indexer": 0, "gather": 0, "select": 0}
    if sp.n_layers > 0:
        out["indexer"] = int(L.sum()) * sp.n_kv_heads * d * 2
        out["gather"] = int(np.minimum(L, sp.topk_shared).sum()) * sp.n_kv_heads * 4 * d
        out["select"] = int(L.sum()) * sp.n_kv_heads * 4
    else:
        n_sparse = int((roles == ROLE_SPARSE).sum())
        nfac = w.n_fac_per_seq.numpy().astype(np.int64)
        out["tip"] = int(L.sum()) * n_sparse * (2 * d if in_place else 4 * sp.n_dom)
        out["fac"] = int(np.minimum(L, nfac).sum()) * n_sparse * 4 * d
        out["select"] = int(L.sum()) * n_sparse * 4
        for g, r in enumerate(roles):
            if r == 1:
                out["window"] += int(L.sum()) * 4 * d
            elif r == 2:
                a = np.minimum(L, sp.sink)
                n = a + (L - np.maximum(a, L - sp.window))
                out["window"] += int(n.sum()) * 4 * d
    # the scores the select reads are an intermediate of the three-kernel form, not step traffic
    out["total"] = sum(v for k, v in out.items() if k != "select")
    return out


def measured_peak_gbs():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C / C++ source without comments and blank space (a comment edit changes no kernel)."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    """Hash of the library's sources (kernels and launch code), comments and spacing ignored."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "token_sparse_decode_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source
    (`workload` carries the suffix ":in_place" for the step whose scan reads K in place)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            data = json.load(f)
        ent = data[workload][kernel]
        if ent.get("source_hash") != kernel_source_hash():
            return None
        return int(ent["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        loaded = [x for x in sm if smax and x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ our arm

def build_step(w, dev, pack: bool = True):
    """The workload's step on `dev`; pack=False keeps no packed dominant columns (the scan reads K in place)."""
    from token_sparse_decode_b200.step import SharedIndexStep, SparseDecodeStep

    k, v = w.k.to(dev), w.v.to(dev)
    offsets = w.offsets.to(dev)
    if w.spec.n_layers > 0:
        step = SharedIndexStep(k, v, offsets, w.max_len, w.total_tokens, w.spec.n_layers, w.spec.n_q_heads,
                               w.spec.topk_shared, w.scale)
        q = (w.q.to(dev), w.q_layers.to(dev))
        return step, q
    idom = None if w.idom is None else w.idom.to(dev)
    step = SparseDecodeStep(k, v, offsets, w.max_len, w.total_tokens, w.spec.n_q_heads, w.roles.tolist(),
                            w.scale, idom=idom, n_fac=int(w.n_fac_per_seq.max()),
                            n_fac_per_seq=w.n_fac_per_seq.to(dev), n_fac_cap=int(w.n_fac_per_seq.max()),
                            sink=w.spec.sink, window=w.spec.window, pack_dominant=pack)
    return step, (w.q.to(dev),)


def step_calls(w, step, q):
    """The public calls one step makes, by name (the same arguments as the step)."""
    from token_sparse_decode_b200 import binding as B

    if w.spec.n_layers > 0:
        return [("shared_index_step", lambda: step(*q))]
    return [("decode_step", lambda: B.decode_step(
        q[0], step.kv, step.idom, step.n_dom, step.n_fac, step.n_fac_per_seq, step.n_fac_cap, step.roles, step.sink,
        step.window, step.scale, step.out, step.ws, step.idx, step.count))]


def launches_per_step(step, q) -> dict:
    """Kernels one eager step launches, by kernel name (the library's launch counters)."""
    from token_sparse_decode_b200 import binding as B

    c0 = B.launch_counts()
    step(*q)
    torch.cuda.synchronize()
    c1 = B.launch_counts()
    return {k: c1[k] - c0[k] for k in c0 if c1[k] != c0[k]}


def kernel_timing(w, copies, steps: int, between) -> dict:
    """Device time of every kernel of the step, per public call.

    Each call runs with the library's launch-event recording armed, so every kernel is
    bracketed by CUDA events recorded on its own stream right before and after it.  Sample i
    runs on input copy i mod R (see cold_copies) behind a device-side sleep, so that the host
    has queued the calls before the first one starts; `between()` runs before every sample.
    """
    from token_sparse_decode_b200 import binding as B

    per_copy = [step_calls(w, step, q) for step, q in copies]
    for calls in per_copy:
        for _, fn in calls:
            fn()
    torch.cuda.synchronize()
    names = [n for n, _ in per_copy[0]]
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in names]
    per, call_ms, order = {}, {n: [] for n in names}, {}
    for it in range(steps):
        between()
        torch.cuda._sleep(1000000)
        calls = per_copy[it % len(per_copy)]
        recs = [(name, B.timed_launches(fn, evs)) for (name, fn), evs in zip(calls, evsets)]
        torch.cuda.synchronize()
        for name, r in recs:
            order[name] = [k for k, _, _ in r]
            for i, (kern, e0, e1) in enumerate(r):
                per.setdefault((name, i, kern), []).append(e0.elapsed_time(e1))
            if r:
                call_ms[name].append(r[0][1].elapsed_time(r[-1][2]))
    kernels = [{"call": n, "index": i, "kernel": k, "ms": float(np.mean(t))} for (n, i, k), t in sorted(per.items())]
    return {"calls": {n: float(np.mean(t)) for n, t in call_ms.items() if t}, "kernels": kernels, "order": order}


MAX_COPIES = 8


def cold_copies(step_bytes: int, l2_bytes: int) -> int:
    """Input copies R to rotate over so that every step starts with its inputs out of L2.

    Copy i is reused R steps later, after R - 1 other steps have moved (R - 1) * step_bytes
    through L2; R is the smallest count (at least 2) for which that is at least twice the L2
    size.  Returns 0 when more than MAX_COPIES would be needed (then L2 is flushed instead).
    """
    r = 2
    while (r - 1) * step_bytes < 2 * l2_bytes:
        r += 1
        if r > MAX_COPIES:
            return 0
    return r


def kernel_bytes(w, ab: dict, call: str, kernel: str, order: list, index: int = -1) -> int:
    """Algorithmic bytes one launch of `kernel` (launch `index` of `order`) moves inside `call`
    (see algorithmic_bytes).

    A call that launches the row kernel alone runs the whole path in it (window heads
    included); in the three-kernel form the scan reads the score columns, the select kernels
    read the fp32 scores (4 bytes per token and scored KV head) and the gather reads the
    selected K / V rows; a later gather of the same call attends the window heads.
    """
    fused = order == ["sparse_row_kernel"]
    if call == "stream_decode":
        return ab["window"]
    if call == "shared_index_step":
        if fused:
            return ab["indexer"] + ab["gather"]
        return {"tip_score_kernel": ab["indexer"], "flash_gather_kernel": ab["gather"]}.get(kernel, ab["select"])
    if fused:
        return ab["tip"] + ab["fac"] + ab["window"]
    if kernel == "flash_gather_kernel":
        first = order.index("flash_gather_kernel")
        sparse_gather = "tip_score_kernel" in order and (index < 0 or index == first)
        return ab["fac"] if sparse_gather else ab["window"]
    return {"tip_score_kernel": ab["tip"], "sparse_row_kernel": ab["tip"] + ab["fac"]}.get(kernel, ab["select"])


def capture_graph(fn):
    """Capture the launches of fn() (all on the current stream) into a CUDA graph."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def shard_spec(spec, rank: int, world: int):
    """Rank `rank`'s batch: the same shape with its own seed (independent sequences, weak scaling)."""
    if world <= 1:
        return spec
    from dataclasses import replace

    return replace(spec, seed=spec.seed + 1000 * rank)


def max_over_ranks(values, world: int, device):
    """Element-wise maximum of per-rank timings (identity on one rank)."""
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_throughput(tokens_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank scans its own batch in the (max-over-ranks) step time."""
    return tokens_per_rank_step * world / (ms_per_step * 1e-3)


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    spec = shard_spec(preset(args.workload), rank, world)
    w = make_workload(spec)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ab = algorithmic_bytes(w, args.in_place_scan)
    # Cold inputs every step: rotate over R device copies of the inputs (each step's traffic
    # pushes the other copies out of L2), or, for steps too small for that, flush L2 by
    # rewriting a buffer of twice its size between steps (outside the events).
    R = cold_copies(ab["total"], l2) if args.copies == 0 else (args.copies if args.copies > 1 else 0)
    copies = [build_step(w, dev, not args.in_place_scan) for _ in range(max(R, 1))]
    step, q = copies[0]
    if R:
        def between():
            pass
        l2_note = (f"inputs rotated over {R} device copies ({R - 1} x {ab['total']} B of step traffic "
                   f"between reuses of a copy, >= 2 x L2); no flush")
    else:
        flush_buf = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

        def between():
            flush_buf.fill_(1)
        l2_note = "flushed between timed steps (2 x L2 buffer rewritten, outside the events)"

    for s_, q_ in copies:
        s_(*q_)  # first call outside capture (sets kernel attributes)
    torch.cuda.synchronize()
    per_step = launches_per_step(step, q)
    if args.graph:
        graphs = [capture_graph(lambda s_=s_, q_=q_: s_(*q_)) for s_, q_ in copies]

        def one(i):
            graphs[i % len(graphs)].replay()
    else:
        def one(i):
            s_, q_ = copies[i % len(copies)]
            return s_(*q_)

    st = torch.cuda.current_stream()
    sampler = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    t_wall0 = time.time()
    for i in range(args.warmup):
        one(i)
        between()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if R:
        # nothing to do between steps: the K steps back to back between one pair of events
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))]
        evs[0][0].record(st)
        for i in range(args.steps):
            one(args.warmup + i)
        evs[0][1].record(st)
        timing_note = "one event pair around the K steps"
    else:
        # the flush stays outside the timed region: one pair of events per step
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i, (e0, e1) in enumerate(evs):
            e0.record(st)
            one(args.warmup + i)
            e1.record(st)
            between()
        timing_note = "one event pair per step (L2 flushed between steps)"
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    # keep the GPU loaded until the clock sampler has seen a few samples
    i = 0
    while time.time() - t_wall0 < 1.5:
        one(i)
        between()
        i += 1
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None

    # end-to-end through the public API with host buffers: H2D of q, the step, D2H of the output
    q_host = [t.cpu().pin_memory() for t in q]
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in q_host)
    d2h = out_host.numel() * out_host.element_size()

    def host_step(s_, q_):
        for a, b_ in zip(q_, q_host):
            a.copy_(b_, non_blocking=True)
        out = s_(*q_)
        out_host.copy_(out, non_blocking=True)

    if args.graph:
        e2e_graphs = [capture_graph(lambda s_=s_, q_=q_: host_step(s_, q_)) for s_, q_ in copies]

        def e2e_one(i):
            e2e_graphs[i % len(e2e_graphs)].replay()
    else:
        def e2e_one(i):
            host_step(*copies[i % len(copies)])
    for i in range(max(1, args.warmup)):
        e2e_one(i)
        between()
    torch.cuda.synchronize()
    e2e_ms = 0.0
    for i in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        e2e_one(i)
        e1.record(st)
        torch.cuda.synchronize()
        e2e_ms += e0.elapsed_time(e1)
        between()

    kt = kernel_timing(w, copies, args.steps if args.steps <= 200 else 200, between)

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, dev)

    tokens_step = int(w.lengths.sum())
    ms_step = ms / args.steps
    value = aggregate_throughput(tokens_step, world, ms_step)
    e2e_value = aggregate_throughput(tokens_step, world, e2e_ms / args.steps)
    peak, peak_kind = measured_peak_gbs()
    # the dominant kernel: the largest device time of one step
    dom = max(kt["kernels"], key=lambda e: e["ms"]) if kt["kernels"] else None
    dom_bytes = kernel_bytes(w, ab, dom["call"], dom["kernel"], kt["order"][dom["call"]], dom["index"]) if dom else 0
    dom_ms = dom["ms"] if dom else None
    one_kernel_step = dom is not None and len(kt["kernels"]) == 1
    if one_kernel_step:
        # the step is that one kernel: its graph-replayed time per step is the kernel's time
        # (the per-launch events add the event records' own overhead around an eager launch)
        dom_ms = ms_step
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9 if dom_ms else None
    step_gbs = ab["total"] / (ms_step * 1e-3) / 1e9
    return {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; bf16 N(0,1) post-RoPE q/K, V; planted salient keys where the workload has them)",
        "config": dict(workload_config(w, world), l2=l2_note, timing=timing_note, algorithmic_bytes_per_step=ab["total"],
                       launch="CUDA graph replay" if args.graph else "direct launches",
                       **({"scan": "K read in place (no packed dominant columns)"} if args.in_place_scan else {})),
        "step_hbm": {"achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                     "bytes_per_step": ab["total"]},
        "roofline": {"kernel": dom["kernel"] if dom else None, "call": dom["call"] if dom else None, "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": (achieved / peak) if achieved else None, "peak_source": peak_kind,
                     "bytes_per_launch": dom_bytes, "ms_per_launch": dom_ms,
                     "timing": "graph-replayed step (one-kernel step)" if one_kernel_step
                     else "CUDA events around the kernel inside the call",
                     "traffic": ncu_traffic(w.spec.name + (":in_place" if args.in_place_scan else ""),
                                            dom["kernel"]) if dom else None},
        "call_ms": kt["calls"],
        "kernel_ms": [{"call": e["call"], "kernel": e["kernel"], "ms": e["ms"],
                       "bytes": kernel_bytes(w, ab, e["call"], e["kernel"], kt["order"][e["call"]], e["index"])}
                      for e in kt["kernels"]],
        "launches_per_step": per_step,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(per_step.values()) * args.steps,
        "clocks": clocks,
        "_w": w,
    }


# ------------------------------------------------------------------------------ the other rows of the path

def _event_ms(fn, steps: int, warmup: int) -> float:
    """Mean device time of fn() over `steps` calls (CUDA events on the current stream)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def measure_append(dev, steps: int = 200, warmup: int = 5) -> dict:
    """aoh_kv_append for a serving batch: 64 sequences, 32 q / 8 KV heads of 128, AoH split
    (2 retrieval, 2 sparse, 4 streaming heads with sink 128 + window 4096)."""
    from token_sparse_decode_b200 import binding as B
    from token_sparse_decode_b200.step import AppendDecodeStep
    from workloads import ROLE_DENSE, ROLE_STREAM, token_draws

    Bn, Hq, Hkv, d = 64, 32, 8, 128
    roles = [ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, ROLE_STREAM, ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, ROLE_STREAM]
    idom = torch.stack([torch.randperm(64, generator=torch.Generator().manual_seed(g))[:16].sort().values
                        for g in range(Hkv)]).to(torch.int32).to(dev)
    step = AppendDecodeStep(Bn, Hq, Hkv, d, 5e5, roles, [steps + warmup + 8] * Bn, 128, 4096, d ** -0.5,
                            idom=idom, n_fac=64)
    q, k, v = (t.to(dev) for t in token_draws(1, 0, Bn, Hq, Hkv, d))
    ms = _event_ms(lambda: step.append(q, k, v), steps, warmup)
    st, _ = B.device_check()
    n_lin = sum(1 for r in roles if r != ROLE_STREAM)
    moved = Bn * (2 * Hq * d * 2 + Hkv * d * 2 * 2 + Hkv * d * 2 * 2 + 2 * n_lin * B.k_dom_cols(16))
    return {"us_per_call": ms * 1e3, "tokens_per_call": Bn, "us_per_token": ms * 1e3 / Bn,
            "bytes_per_call": moved, "device_check": st,
            "workload": "64 sequences x (32 q, 8 KV heads, d 128): 2 retrieval + 2 sparse heads to the linear "
                        "cache, 4 streaming heads to a 128 + 4096 ring"}


def measure_offload(dev, steps: int = 20, warmup: int = 3) -> dict:
    """FASA-M on the 8B-shaped layer: V and the non-dominant K dims in pinned host memory."""
    from token_sparse_decode_b200.step import OffloadDecodeStep

    w = make_workload(preset("llama8b_gqa4_L32k"))
    k, v = w.k.to(dev), w.v.to(dev)
    offs, idom = w.offsets.to(dev), w.idom.to(dev)
    nfac = int(w.n_fac_per_seq.max())
    step = OffloadDecodeStep(k, v, offs, w.max_len, w.total_tokens, w.spec.n_q_heads, idom, w.scale, n_fac=nfac,
                             n_fac_cap=nfac)
    del k, v
    torch.cuda.empty_cache()
    q = w.q.to(dev)
    ms = _event_ms(lambda: step(q), steps, warmup)
    link = step.link_bytes_per_step()
    # the host link's measured copy bandwidth: 256 MB pinned host -> device
    src = torch.empty(256 << 20, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    copy_ms = _event_ms(lambda: dst.copy_(src, non_blocking=True), 5, 2)
    peak = src.numel() / (copy_ms * 1e-3) / 1e9
    achieved = link / (ms * 1e-3) / 1e9
    return {"ms_per_step": ms, "tokens_per_step": int(w.lengths.sum()),
            "value": int(w.lengths.sum()) / (ms * 1e-3), "unit": "tokens/s",
            "link_bytes_per_step": link, "link_achieved_gbs": achieved, "link_peak_gbs": peak,
            "link_frac": achieved / peak, "peak_source": "measured pinned host-to-device copy of 256 MB",
            "device_bytes": int(step.k_dom.numel() * 2),
            "host_bytes": int((step.k_rest.numel() + step.v_host.numel()) * 2),
            "workload": "llama8b_gqa4_L32k with V and the non-dominant K dims in pinned host memory"}


def measure_classify(dev, steps: int = 5, warmup: int = 1) -> dict:
    """The AoH head classifier on 8B-shaped projection weights (32 q / 8 KV heads, d_model 4096)."""
    from token_sparse_decode_b200 import binding as B
    from workloads import HEAD_WEIGHT_PRESETS, head_weights

    sp = HEAD_WEIGHT_PRESETS["llama8b_heads"]
    wq, wk, _ = head_weights(sp)
    wq, wk = wq.to(dev), wk.to(dev)
    er_h = torch.empty(sp.n_q_heads, dtype=torch.float64, device=dev)
    er_g = torch.empty(sp.n_kv_heads, dtype=torch.float64, device=dev)
    roles = torch.empty(sp.n_kv_heads, dtype=torch.uint8, device=dev)
    ws = B.workspace(B.head_classify_workspace_size(sp.d_model, sp.n_q_heads, sp.n_kv_heads, sp.head_dim), dev)
    fn = lambda: B.head_classify(wq, wk, sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.n_retrieval, er_h, er_g,  # noqa: E731
                                 roles, ws)
    ms = _event_ms(fn, steps, warmup)
    gram_flops = 2 * (sp.n_q_heads + sp.n_kv_heads) * sp.head_dim ** 2 * sp.d_model
    rec = B.timed_launches(fn)
    torch.cuda.synchronize()
    per = {n: e0.elapsed_time(e1) for n, e0, e1 in rec}
    return {"ms_per_call": ms, "kernel_ms": per, "gram_flops": gram_flops,
            "weight_bytes": int((wq.numel() + wk.numel()) * 2), "roles": roles.cpu().tolist(),
            "workload": "llama8b_heads: W_Q [4096, 4096], W_K [1024, 4096] bf16, 4 of 8 groups retrieval"}


# ------------------------------------------------------------------------------ oracle (CPU) arms
#
# The oracle runs on whole (sequence, KV head) rows: the select needs every score of a row.
# A row task carries that row's bf16 inputs (compact copies), so a worker process needs
# nothing else; every run keeps BLAS to one thread per process, and the all-cores run uses
# one spawned worker process per core of this process's affinity (at most MAX_POOL).

def host_cores() -> dict:
    """Logical CPUs of the host and of this process's affinity mask."""
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        aff = os.cpu_count() or 1
    return {"host_cpu_count": os.cpu_count(), "affinity_cores": aff}


def row_task(w, b: int, g: int):
    """The inputs of oracle row (b, g) as compact bf16 tensors, and its token count."""
    sp = w.spec
    G = sp.group
    o0, o1 = int(w.offsets[b]), int(w.offsets[b + 1])
    keys = w.k[o0:o1, g].clone()
    vals = w.v[o0:o1, g].clone()
    if sp.n_layers > 0:
        return ("shared", w.q[b, g * G:(g + 1) * G].clone(), w.q_layers[:, b, g * G:(g + 1) * G].clone(),
                keys, vals, sp.topk_shared, w.scale), o1 - o0
    return ("row", w.q[b, g * G:(g + 1) * G].clone(), keys, vals, int(w.roles[g]), w.scale,
            None if w.idom is None else w.idom[g].tolist(), int(w.n_fac_per_seq[b]), sp.sink, sp.window), o1 - o0


def oracle_row(task) -> float:
    """Run the oracle on one row task; returns its wall time in seconds (one BLAS thread)."""
    import oracle
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        if task[0] == "shared":
            _, qi, ql, keys, vals, topk, scale = task
            kk = np.ascontiguousarray(keys.double().numpy()[:, None, :])
            vv = np.ascontiguousarray(vals.double().numpy()[:, None, :])
            oracle.shared_index_step(qi.double().numpy()[None], ql.double().numpy()[:, None], kk, vv,
                                     [0, kk.shape[0]], topk, scale)
        else:
            _, qg, keys, vals, role, scale, idom, n_fac, sink, window = task
            oracle.decode_row(qg.double().numpy(), keys.double().numpy(), vals.double().numpy(), role, scale, idom,
                              n_fac, sink, window)
        return time.perf_counter() - t0


def _oracle_repeat(arg) -> float:
    """Worker body: one row task run `repeat` times; returns the busy time."""
    task, repeat = arg
    return sum(oracle_row(task) for _ in range(repeat))


def _pool_ready(_):
    import oracle  # noqa: F401  (the workers' imports happen before any timing)
    from threadpoolctl import threadpool_limits  # noqa: F401

    return os.getpid()


class OraclePool:
    """Spawned worker processes (never forked: the parent may hold a CUDA context)."""

    def __init__(self, workers: int):
        import multiprocessing
        from concurrent.futures import ProcessPoolExecutor

        self.workers = workers
        self.ex = ProcessPoolExecutor(max_workers=workers, mp_context=multiprocessing.get_context("spawn"))
        list(self.ex.map(_pool_ready, range(workers)))

    def run(self, tasks, repeat: int) -> float:
        """Wall time of every worker running its task `repeat` times (one task per worker)."""
        t0 = time.perf_counter()
        list(self.ex.map(_oracle_repeat, [(t, repeat) for t in tasks]))
        return time.perf_counter() - t0

    def close(self):
        self.ex.shutdown(wait=True)


def all_rows(w):
    return [(b, g) for b in range(w.spec.batch) for g in range(w.spec.n_kv_heads)]


def oracle_single_thread(w, seconds: float) -> dict:
    """Rows of the workload in order, one thread, until `seconds` have passed (at least one row)."""
    rows = all_rows(w)
    done, tokens, busy = 0, 0, 0.0
    while busy < seconds:
        b, g = rows[done % len(rows)]
        task, n_tok = row_task(w, b, g)
        busy += oracle_row(task)
        done += 1
        tokens += n_tok
    return {"value": tokens / busy, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} (sequence, KV head) rows ({len(rows)} make one step), float64 numpy, "
                      f"one process, BLAS limited to 1 thread, {busy:.1f} s",
            "s_per_row": busy / done}


def pool_size(w) -> int:
    return max(1, min(host_cores()["affinity_cores"], MAX_POOL))


def repeats_for(s_per_row: float, target_s: float = 1.0) -> int:
    """Times a worker repeats its row so that one batch is about target_s of work per worker."""
    return max(1, int(round(target_s / max(s_per_row, 1e-6))))


class PoolSteps:
    """Batches of the pool: worker j runs row (i * workers + j) mod rows, `repeat` times."""

    def __init__(self, w, pool: OraclePool, repeat: int):
        self.w, self.pool, self.repeat = w, pool, repeat
        self.rows = all_rows(w)
        self.i = 0

    def batch(self):
        tasks = [row_task(self.w, *self.rows[(self.i * self.pool.workers + j) % len(self.rows)])
                 for j in range(self.pool.workers)]
        self.i += 1
        wall = self.pool.run([t for t, _ in tasks], self.repeat)
        return wall, sum(n for _, n in tasks) * self.repeat

    def describe(self, rows_done: int, wall: float) -> str:
        return (f"{rows_done} (sequence, KV head) row runs ({len(self.rows)} rows make one step) in batches of "
                f"{self.pool.workers} rows x {self.repeat} repeats, float64 numpy, {self.pool.workers} spawned "
                f"worker processes with 1 BLAS thread each, {wall:.1f} s of wall time")


def cpu_baseline(w, seconds: float = 10.0) -> dict:
    """The oracle on all cores of this process's affinity and on one thread (both reported)."""
    single = oracle_single_thread(w, seconds)
    pool = OraclePool(pool_size(w))
    try:
        ps = PoolSteps(w, pool, repeats_for(single["s_per_row"]))
        wall, tokens, runs = 0.0, 0, 0
        while wall < seconds:
            dt, n = ps.batch()
            wall += dt
            tokens += n
            runs += pool.workers * ps.repeat
        multi = {"value": tokens / wall, "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
                 "sample": ps.describe(runs, wall)}
    finally:
        pool.close()
    return dict(multi, **host_cores(), single_thread=single)


def workload_config(w, world: int) -> dict:
    """The `config` of the JSON line: the workload, its shape and the step's algorithmic bytes."""
    return {
        "workload": w.spec.name, "batch": w.spec.batch, "seq_len": int(w.max_len),
        "tokens_per_step_per_gpu": int(w.lengths.sum()), "q_heads": w.spec.n_q_heads,
        "kv_heads": w.spec.n_kv_heads, "head_dim": w.spec.head_dim, "n_dom": w.spec.n_dom,
        "n_fac": int(w.n_fac_per_seq.max()), "n_layers": w.spec.n_layers,
        "parallelism": f"independent sequences per rank x{world}",
        "algorithmic_bytes_per_step": algorithmic_bytes(w)["total"],
    }


def run_reference(args, rank, world):
    """The oracle on the host cores: each step is one batch of rows on the worker pool."""
    if rank != 0:
        return None
    w = make_workload(preset(args.workload))
    single = oracle_single_thread(w, 5.0)
    pool = OraclePool(pool_size(w))
    try:
        ps = PoolSteps(w, pool, repeats_for(single["s_per_row"], 2.0))
        for _ in range(args.warmup):
            ps.batch()
        t, tokens = 0.0, 0
        for _ in range(args.steps):
            dt, n = ps.batch()
            t += dt
            tokens += n
    finally:
        pool.close()
    ms_step = t / args.steps * 1e3
    value = tokens / t
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, same inputs)",
        "config": workload_config(w, world),
        "cpu_baseline": dict({"value": value, "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
                              "sample": ps.describe(args.steps * pool.workers * ps.repeat, t)},
                             **host_cores(), single_thread=single),
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------------------ main

def torchrun_command(n: int, port: int, argv) -> list:
    """The command that runs this script with the same arguments as n ranks on this node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def relaunch_under_torchrun(n: int) -> int:
    import socket

    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    return subprocess.call(torchrun_command(n, port, sys.argv[1:]))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--in-place-scan", action="store_true",
                    help="keep no packed dominant columns: the importance scan reads the 16-byte segments of K")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the append, host-offload and head-classifier measurements")
    ap.add_argument("--graph", type=int, default=1, help="replay each step from a CUDA graph (1) or launch (0)")
    ap.add_argument("--copies", type=int, default=0,
                    help="input copies to rotate over (0: enough for cold inputs; 1: one copy, L2 flushed)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: run this same command under torchrun with N ranks
        sys.exit(relaunch_under_torchrun(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; measuring {world} ranks", file=sys.stderr)

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    w = res.pop("_w")
    if rank == 0:
        if not args.no_extras:
            dev = torch.device("cuda", local_rank)
            res["append"] = measure_append(dev)
            res["offload"] = measure_offload(dev)
            res["classify"] = measure_classify(dev)
        if not args.no_cpu_baseline and world == 1:
            res["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
