"""Benchmark: top-k context-sparse decode at 128K context and 50x sparsity.

One step = one decode step of the long-context index-reuse workload: layer 0
scores all 131072 cached keys of each of 8 kv-heads, selects the top 2621 and
attends over them (32 query heads, GQA 4); layers 1-3 reuse layer 0's indices
(no scan).  Inputs are synthetic (seeded N(0,1) bf16), resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload reuse128k|llama8b|large_batch|hybrid|tiny]

Prints one JSON line.  `value` = algorithmic HBM bytes of the step (full K scan
of layer 0 + gathered K/V rows of every layer + Q, O, indices) / device time,
in TB/s, summed over all ranks (each rank runs its own replica: the units of
the workload are independent, so ranks share no data).  `--impl reference`
times the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = ("decode-step µs & achieved HBM TB/s (score+top-k+sparse attn), 128K ctx, 50×")
FALLBACK_HBM_GBS = 6650.0


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None when
    the kernel's source has changed since the counters were taken."""
    import hashlib

    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[kernel]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    return rec["bytes_per_launch"] if sha == rec["source_sha256"] else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- workload model

class Plan:
    """The layers of one step and their algorithmic bytes."""

    def __init__(self, w, lens):
        self.w = w
        self.lens = [int(x) for x in lens]
        self.kreq = w.k_per_seq(self.lens)
        self.k_max = max(self.kreq)
        g = w.Hq // w.Hkv
        d, blk = w.d, w.block
        self.kb = []
        for n, k in zip(self.lens, self.kreq):
            units = n if blk == 1 else -(-n // blk)
            self.kb.append(min(k, units))
        q_o = w.B * w.Hq * d * (2 + 4)
        idx_b = w.B * w.Hkv * self.k_max * 4
        gather = 0
        for n, kb in zip(self.lens, self.kb):
            rows = kb if blk == 1 else min(kb * blk, n)  # block mode: expanded valid rows (bound)
            gather += w.Hkv * rows * d * 2 * 2
        scan = sum(w.Hkv * (n if blk == 1 else -(-n // blk)) * d * (2 if blk == 1 else 4)
                   for n in self.lens)
        full = sum(w.Hkv * n * d * 2 * 2 for n in self.lens)
        self.bytes = {"select": scan + gather + q_o + idx_b, "reuse": gather + q_o + idx_b,
                      "full": full + q_o, "scan": scan, "gather": gather}
        self.layer_bytes = [self.bytes[{0: "full", 1: "select", 2: "reuse"}[m]] for m in w.route]
        self.step_bytes = sum(self.layer_bytes)
        self.tokens_attended = sum(w.Hq * (kb if blk == 1 else min(kb * blk, n))
                                   for n, kb in zip(self.lens, self.kb))


def config_of(w, plan, world):
    """The workload as both arms report it (the same dict, so that the two lines
    can be compared key by key)."""
    kv_bytes = w.layers * w.B * w.Hkv * w.Ncap * w.d * 2 * 2
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.Ncap, "k": plan.k_max,
            "layers": w.layers, "route": "".join("FSR"[m] for m in w.route), "block": w.block,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (%.2f GB of K/V per step)" % (kv_bytes / 1e9)}


def make_layers(w, dev, lens):
    from top_sparse_attention_02_b200 import inputs

    layers, Q = [], None
    for li in range(w.layers):
        if w.q_drift > 0 and li > 0:
            Q = inputs.drift_query(Q, w.q_drift, seed=w.seed + 100 + li)
        L = inputs.decode_layer(w.B, w.Hq, w.Hkv, w.Ncap, lens, plant_frac=w.plant_frac,
                                seed=w.seed + li, device=dev, Q=Q if w.q_drift > 0 else None)
        Q = L.Q
        layers.append(L)
    return layers


def workload_of(args):
    """The named workload; --ncap shrinks its context (a smaller case for profiler
    captures, never a bench line of the named workload)."""
    from top_sparse_attention_02_b200 import workloads

    w = workloads.ALL[args.workload]
    if args.ncap:
        n = int(args.ncap)
        lens = None if w.lens is None else (min(w.lens[0], n), min(w.lens[1], n))
        w = dataclasses.replace(w, Ncap=n, lens=lens, name=f"{w.name} [reduced to N={n} for profiling]")
    return w


def workload_lens(w):
    from top_sparse_attention_02_b200 import inputs

    if w.lens is None:
        return [w.Ncap] * w.B
    return inputs.draw_lengths(w.B, w.lens[0], w.lens[1], seed=w.seed + 1000).tolist()


# ---------------------------------------------------------------- clocks

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        try:  # query the GPU by UUID: CUDA and nvidia-smi may number devices differently
            u = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.idx = u if u.startswith("GPU-") else f"GPU-{u}"
        except Exception:
            self.idx = str(gpu_index)
        self.proc = None
        # the raw samples; TSA_CLOCKS_CSV keeps them where the caller wants them
        self.path = os.environ.get("TSA_CLOCKS_CSV") or os.path.join(tempfile.gettempdir(),
                                                                     f"tsa_clocks_dev{gpu_index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, dev):
    from top_sparse_attention_02_b200 import binding as tsa
    from top_sparse_attention_02_b200 import workloads

    w = workload_of(args)
    lens = workload_lens(w)
    plan = Plan(w, lens)
    layers = make_layers(w, dev, lens)
    B, Hq, Hkv, d = w.B, w.Hq, w.Hkv, w.d
    shape = tsa.shape_of(layers[0].Q, layers[0].K)
    kreq_t = torch.tensor(plan.kreq, dtype=torch.int32, device=dev)
    ws_bytes = max(tsa.workspace_size(shape, plan.k_max, w.block, m) for m in set(w.route))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    tsa.workspace_init(ws)
    O = [torch.empty(B, Hq, d, dtype=torch.float32, device=dev) for _ in range(w.layers)]
    idx = [torch.full((B, Hkv, plan.k_max), -1, dtype=torch.int32, device=dev)
           for _ in range(w.layers)]
    Kmean = []
    for li, L in enumerate(layers):
        if w.block > 1 and w.route[li] == tsa.SELECT:
            NB = -(-w.Ncap // w.block)
            km = torch.zeros(B, Hkv, NB, d, dtype=torch.float32, device=dev)
            tsa.block_summarize(L.K, L.seq_lens, w.block, km, ws, shape=shape)
            Kmean.append(km)
        else:
            Kmean.append(None)
    # Every layer's lengths, k's, K, V and reused indices were written before the
    # step (or by a layer at least two launches back), so each layer may read them
    # before the kernel just before it has finished (TSA_EARLY_INPUTS); Q, the
    # workspace and O are still touched only after it.
    def make_step_args(flags):
        out = []
        for li, L in enumerate(layers):
            mode = w.route[li]
            src = w.reuse_from[li]
            out.append(tsa.step_args(
                L.Q, L.K, L.V, L.seq_lens, O[li], ws, mode=mode, scale=w.scale, k_max=plan.k_max,
                block=w.block, k_per_seq=kreq_t, Kmean=Kmean[li],
                idx_in=idx[src] if mode == tsa.REUSE else None,
                idx_out=idx[li] if mode == tsa.SELECT else None, flags=flags))
        return out

    step_args = make_step_args(tsa.EARLY_INPUTS)
    # The step is captured once into a CUDA graph (the library never allocates or
    # synchronises, so its calls capture cleanly) and replayed: the timing is
    # device time, not Python/ctypes launch overhead.
    stream = torch.cuda.Stream(device=dev)

    def step():
        for a in step_args:
            tsa.decode_step(a, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    tsa.check_device_status(ws, stream)
    l0 = tsa.launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    launches_per_step = tsa.launch_count() - l0
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    stream.synchronize()
    tsa.check_device_status(ws, stream)

    # timed region: K whole steps; inputs (K, V of every layer) exceed L2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    launches = launches_per_step * args.steps
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, world, dev)
    tsa.check_device_status(ws, stream)
    del graph

    # the same step with every kernel waiting for its predecessor before its
    # first read (no TSA_EARLY_INPUTS), for comparison
    plain_args = make_step_args(0)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        for a in plain_args:
            tsa.decode_step(a, stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g2.replay()
        e0.record(stream)
        for _ in range(args.steps):
            g2.replay()
        e1.record(stream)
    stream.synchronize()
    ms_plain = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    tsa.check_device_status(ws, stream)
    del g2

    # per-stage device times: each stage alone, repeated in its own graph
    stages = stage_times(tsa, w, plan, layers, Kmean, ws, kreq_t, idx, O, stream)
    # each layer's share of the step as captured: the step cut after layer i,
    # timed the same way (a graph of back-to-back copies), minus the step cut
    # after layer i - 1 (with early inputs a layer's launch overlaps the end of
    # the one before, which the stages timed alone do not show)
    prefix = [graph_us(lambda n=n: [tsa.decode_step(a, stream) for a in step_args[:n]], stream, 10)
              for n in range(1, w.layers + 1)]
    kinds = {tsa.SELECT: "select_step", tsa.REUSE: "attn", tsa.FULL: "full"}
    stages["in_step"] = {f"L{li}_{kinds[w.route[li]]}": prefix[li] - (prefix[li - 1] if li else 0.0)
                         for li in range(w.layers)}
    stages["in_step_note"] = ("us a layer adds to the captured step (TSA_EARLY_INPUTS): the step cut after the "
                              "layer minus the step cut before it, each timed as 10 back-to-back copies in a graph")
    copy_gbs = copy_probe(tsa, dev, stream)
    read_gbs = read_probe(tsa, dev, ws, stream)
    gather = gather_probe(tsa, w, plan, layers, idx, ws, stream)

    peak, peak_kind = measured_peaks()
    score_us = stages["score_us"]
    score_bytes = plan.bytes["scan"]
    achieved = score_bytes / (score_us * 1e-6) / 1e9
    res = {
        "metric": METRIC, "value": whole_job_value(plan.step_bytes, ms, world), "unit": "TB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "us_per_step": ms * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 Q/K/V, resident in HBM)",
        "config": config_of(w, plan, world),
        "algorithmic_bytes_per_step": plan.step_bytes,
        "step_flags": "TSA_EARLY_INPUTS on every layer (its inputs are not written by the kernel before it)",
        "ms_per_step_without_early_inputs": ms_plain,
        "tokens_attended_per_s": world * plan.tokens_attended * w.layers / (ms * 1e-3),
        "stages_us": stages,
        "roofline": {"kernel": "score_tc_kernel (layer-0 K scan)", "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, torch copy)",
                     "copy_probe_gbs_this_run": copy_gbs,
                     "read_probe_gbs_this_run": read_gbs,
                     "frac_of_read_probe": achieved / read_gbs,
                     "traffic": recorded_traffic("score_tc_kernel") if w is workloads.REUSE128K else None,
                     "algorithmic_bytes_per_launch": score_bytes},
        "attn_roofline": attn_roofline(w, plan, stages, gather),
        "clocks": clk.summary(),
        "gpu_launches": launches,
        "timing": "CUDA graph of one whole step, replayed K times between CUDA events",
    }
    if not args.no_e2e:
        res["e2e"] = e2e_measure(tsa, w, plan, layers, step_args, O, idx, ws, kreq_t, stream, args)
    if args.offload:
        res["offload"] = offload_probe(tsa, w, plan, layers, Kmean, ws, kreq_t, idx, O, stream)
    if args.probes:
        res["probes"] = {"handoff": handoff_probe(tsa, w, plan, layers, kreq_t, stream),
                         "overlap": overlap_probe(tsa, w, plan, lens, dev, stream)}
        if w.block == 1:
            res["probes"]["sequence_sharded"] = shard_probe(tsa, w, plan, layers, kreq_t, stream)
    return res


class L2Flush:
    """Reads a 256 MB buffer (twice L2) into one scalar: afterwards L2 holds only
    clean lines of that buffer, so the next launch reads its data from HBM."""

    def __init__(self, dev):
        self.buf = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        torch.sum(self.buf, dim=0, out=self.out)


def graph_us(fn, stream, reps):
    """Device time of `reps` calls of fn captured in one CUDA graph, per call."""
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / reps


def stage_times(tsa, w, plan, layers, Kmean, ws, kreq_t, idx, O, stream, reps=10):
    """Device time of each stage two ways, each in a CUDA graph of `reps` launches:
    back to back ("warm": the top-k and attention stages read L2-sized data, so
    their repeats hit L2), and each launch after an L2 flush, minus the flushes
    alone ("cold": HBM reads, as inside a step; it includes the launch latency
    that programmatic dependent launch hides inside a step)."""
    from top_sparse_attention_02_b200 import binding as _b

    shape = _b.shape_of(layers[0].Q, layers[0].K)
    NB = -(-w.Ncap // w.block)
    rows = w.Ncap if w.block == 1 else NB
    scores = torch.empty(w.B, w.Hkv, rows, dtype=torch.float32, device=layers[0].Q.device)
    calls = {}
    for li, L in enumerate(layers):
        m = w.route[li]
        if m == tsa.SELECT:
            keys = L.K if w.block == 1 else Kmean[li]
            calls[f"L{li}_score"] = lambda L=L, keys=keys: tsa.sparse_decode_score(
                L.Q, keys, L.seq_lens, shape, w.block, w.scale, scores, ws, stream)
            calls[f"L{li}_topk"] = lambda L=L, li=li: tsa.topk_select(
                scores, L.seq_lens, kreq_t, plan.k_max, shape, w.block, idx[li], ws, stream)
            calls[f"L{li}_attn"] = lambda L=L, li=li: tsa.sparse_decode_attn(
                L.Q, L.K, L.V, L.seq_lens, idx[li], kreq_t, plan.k_max, w.block, w.scale, O[li], ws, stream)
            # the whole SELECT step, as the decode step runs it (its top-k starts
            # from the scorer's first-digit histogram, which the stand-alone
            # stages above do not have)
            sa = tsa.step_args(L.Q, L.K, L.V, L.seq_lens, O[li], ws, mode=tsa.SELECT, scale=w.scale,
                               k_max=plan.k_max, block=w.block, k_per_seq=kreq_t, Kmean=Kmean[li],
                               idx_out=idx[li])
            calls[f"L{li}_select_step"] = lambda sa=sa: tsa.decode_step(sa, stream)
        elif m == tsa.REUSE:
            calls[f"L{li}_attn"] = lambda L=L, li=li: tsa.sparse_decode_attn(
                L.Q, L.K, L.V, L.seq_lens, idx[w.reuse_from[li]], kreq_t, plan.k_max, w.block, w.scale,
                O[li], ws, stream)
        else:
            calls[f"L{li}_attn"] = lambda L=L, li=li: tsa.sparse_decode_attn(
                L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, w.scale, O[li], ws, stream)
            if li == w.route.index(tsa.FULL):
                # the first full layer once more, handing on its top-k (what a
                # sensitive layer does before reuse layers): the cost of the hand-off
                km = None
                if w.block > 1:
                    km = torch.zeros(w.B, w.Hkv, NB, w.d, dtype=torch.float32, device=L.Q.device)
                    tsa.block_summarize(L.K, L.seq_lens, w.block, km, ws, shape=shape)
                idx_emit = torch.full_like(idx[li], -1)
                fa = tsa.step_args(L.Q, L.K, L.V, L.seq_lens, O[li], ws, mode=tsa.FULL, scale=w.scale,
                                   k_max=plan.k_max, block=w.block, k_per_seq=kreq_t, Kmean=km,
                                   idx_out=idx_emit)
                calls[f"L{li}_full_emit_step"] = lambda fa=fa, km=km, ie=idx_emit: tsa.decode_step(fa, stream)
    flush = L2Flush(layers[0].Q.device)
    flush_us = graph_us(flush, stream, reps)
    warm, cold = {}, {}
    for name, fn in calls.items():
        warm[name] = graph_us(fn, stream, reps)
        cold[name] = graph_us(lambda fn=fn: (flush(), fn()), stream, reps) - flush_us
    del flush
    sel = [li for li, m in enumerate(w.route) if m == tsa.SELECT]
    return {"warm": warm, "cold": cold,
            "score_us": statistics.mean(warm[f"L{li}_score"] for li in sel) if sel else float("nan"),
            "note": f"per launch, {reps} launches per CUDA graph; warm = back to back, cold = after an L2 "
                    "flush (minus the flush alone)"}


def offload_probe(tsa, w, plan, layers, Kmean, ws, kreq_t, idx, O, stream, reps=5):
    """Index-guided offload: the first SELECT layer of a block-mode stack, and a
    REUSE step over its blocks, with that layer's K and V in page-locked host
    memory (the block means stay on the device).  Only the selected blocks cross
    the host link.  Timed with CUDA events around single launches, each after an
    L2 flush (the pointer check that the offload path makes on the host is kept
    out of graph capture), against a 1 GiB pinned host-to-device copy."""
    assert w.block > 1, "the offload probe needs a block-mode workload"
    li = w.route.index(tsa.SELECT)
    L = layers[li]
    dev = L.Q.device
    Kh = torch.empty(L.K.shape, dtype=L.K.dtype, pin_memory=True)
    Vh = torch.empty(L.V.shape, dtype=L.V.dtype, pin_memory=True)
    Kh.copy_(L.K)
    Vh.copy_(L.V)
    flush = L2Flush(dev)

    def timed(fn):
        ts = []
        for _ in range(reps + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                flush()
                e0.record(stream)
                fn()
                e1.record(stream)
            stream.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(ts[1:])

    sel = tsa.step_args(L.Q, Kh, Vh, L.seq_lens, O[li], ws, mode=tsa.SELECT, scale=w.scale, k_max=plan.k_max,
                        block=w.block, k_per_seq=kreq_t, Kmean=Kmean[li], idx_out=idx[li], flags=tsa.KV_HOST)
    reu = tsa.step_args(L.Q, Kh, Vh, L.seq_lens, O[li], ws, mode=tsa.REUSE, scale=w.scale, k_max=plan.k_max,
                        block=w.block, k_per_seq=kreq_t, idx_in=idx[li], flags=tsa.KV_HOST)
    select_us = timed(lambda: tsa.decode_step(sel, stream))
    reuse_us = timed(lambda: tsa.decode_step(reu, stream))
    tsa.check_device_status(ws, stream)
    # rows the attention fetches: every valid row of each selected block, K and V
    lens = [int(x) for x in L.seq_lens.cpu()]
    ix = idx[li].cpu().numpy()
    rows = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            for e in ix[b, h]:
                if e >= 0:
                    rows += max(0, min(w.block, lens[b] - int(e) * w.block))
    fetched = rows * 2 * w.d * 2
    src = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    h2d = []
    for _ in range(4):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            dst.copy_(src, non_blocking=True)
            e1.record(stream)
        stream.synchronize()
        h2d.append(src.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    h2d_gbs = max(h2d[1:])
    del Kh, Vh, src, dst, flush
    achieved = fetched / (reuse_us * 1e-6) / 1e9
    whole = (L.K.numel() + L.V.numel()) * 2
    return {"layer": li, "select_step_us": select_us, "reuse_step_us": reuse_us, "fetched_bytes": fetched,
            "reuse_achieved_gbs": achieved, "h2d_copy_gbs": h2d_gbs, "frac_of_h2d_copy": achieved / h2d_gbs,
            "whole_layer_kv_bytes": whole, "whole_layer_copy_us": whole / (h2d_gbs * 1e9) * 1e6,
            "note": "K and V of one layer in pinned host memory; attention reads only the selected "
                    "128-token blocks across the host link; cold L2, median of %d single launches" % reps}


def handoff_probe(tsa, w, plan, layers, kreq_t, stream, reps=10, only=None):
    """Layer 0's tensors as a full layer (dense attention), as a full layer that
    hands on its top-k (HyLRA's sensitive layer), and as a SELECT step: each in a
    CUDA graph of `reps` decode steps, warm and after an L2 flush (cold)."""
    L = layers[0]
    dev = L.Q.device
    shape = tsa.shape_of(L.Q, L.K)
    ws = torch.empty(max(tsa.workspace_size(shape, plan.k_max, w.block, m) for m in (tsa.FULL, tsa.SELECT)),
                     dtype=torch.uint8, device=dev)
    tsa.workspace_init(ws)
    km = None
    if w.block > 1:
        km = torch.zeros(w.B, w.Hkv, -(-w.Ncap // w.block), w.d, dtype=torch.float32, device=dev)
        tsa.block_summarize(L.K, L.seq_lens, w.block, km, ws, shape=shape)
    O = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
    ix = torch.full((w.B, w.Hkv, plan.k_max), -1, dtype=torch.int32, device=dev)
    common = dict(scale=w.scale, k_max=plan.k_max, block=w.block, k_per_seq=kreq_t, Kmean=km)
    steps = {"full": tsa.step_args(L.Q, L.K, L.V, L.seq_lens, O, ws, mode=tsa.FULL, scale=w.scale),
             "full_handing_on_topk": tsa.step_args(L.Q, L.K, L.V, L.seq_lens, O, ws, mode=tsa.FULL,
                                                   idx_out=ix, **common),
             "select": tsa.step_args(L.Q, L.K, L.V, L.seq_lens, O, ws, mode=tsa.SELECT, idx_out=ix, **common)}
    if reps == 0:  # --profile: the chosen step twice, untimed
        for _ in range(2):
            tsa.decode_step(steps[only], stream)
        tsa.check_device_status(ws, stream)
        return {}
    flush = L2Flush(dev)
    f_us = graph_us(flush, stream, reps)
    out = {}
    for name, a in steps.items():
        out[name] = {"warm_us": graph_us(lambda a=a: tsa.decode_step(a, stream), stream, reps),
                     "cold_us": graph_us(lambda a=a: (flush(), tsa.decode_step(a, stream)), stream, reps) - f_us}
    tsa.check_device_status(ws, stream)
    out["kv_bytes"] = (L.K.numel() + L.V.numel()) * 2
    return out


def shard_probe(tsa, w, plan, layers, kreq_t, stream, R=2, reps=10):
    """Layer 0 as a sequence-sharded SELECT step with R shards emulated on one GPU
    (each shard's calls on its own slice of the cache, one after another; the two
    all-gathers replaced by writing straight into the stacked buffers, which is
    what they deliver).  Each call timed alone in a CUDA graph of `reps`
    launches, warm and after an L2 flush; the whole emulated step is their sum."""
    L = layers[0]
    dev = L.Q.device
    B, Hkv, N = w.B, w.Hkv, w.Ncap
    bounds = [N * r // R for r in range(R + 1)]
    k = plan.k_max
    shards = []
    for r in range(R):
        lo, hi = bounds[r], bounds[r + 1]
        K_r, V_r = L.K[:, :, lo:hi].contiguous(), L.V[:, :, lo:hi].contiguous()
        lens_r = (L.seq_lens - lo).clamp(0, hi - lo).to(torch.int32)
        ws = torch.empty(tsa.shard_workspace_size(tsa.shape_of(L.Q, K_r), k, R), dtype=torch.uint8, device=dev)
        tsa.workspace_init(ws)
        shards.append((lo, K_r, V_r, lens_r, ws))
    cs = torch.empty(R, B, Hkv, k, dtype=torch.float32, device=dev)
    cr = torch.empty(R, B, Hkv, k, dtype=torch.int32, device=dev)
    idx = torch.empty(B, Hkv, k, dtype=torch.int32, device=dev)
    O_parts = torch.empty(R, B, w.Hq, 128, dtype=torch.float32, device=dev)
    lse = torch.empty(R, B, w.Hq, dtype=torch.float32, device=dev)
    O = torch.empty(B, w.Hq, 128, dtype=torch.float32, device=dev)
    shape = tsa.shape_of(L.Q, L.K)
    lo0, K0, V0, l0, ws0 = shards[0]
    calls = {
        "shard_select (one shard)": lambda: tsa.shard_select(L.Q, K0, l0, kreq_t, k, w.scale, lo0, cs[0], cr[0],
                                                             ws0, stream),
        "shard_merge": lambda: tsa.shard_merge(cs, cr, shape, kreq_t, k, idx, ws0, stream),
        "shard_attend (one shard)": lambda: tsa.shard_attend(L.Q, K0, V0, l0, idx, kreq_t, k, lo0, w.scale,
                                                             O_parts[0], lse[0], ws0, stream),
        "shard_combine": lambda: tsa.shard_combine(O_parts, lse, shape, O, stream),
    }
    for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):  # fill every shard's candidates and parts once
        with torch.cuda.stream(stream):
            tsa.shard_select(L.Q, K_r, lens_r, kreq_t, k, w.scale, lo, cs[r], cr[r], ws, stream)
    with torch.cuda.stream(stream):
        tsa.shard_merge(cs, cr, shape, kreq_t, k, idx, ws0, stream)
    for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):
        with torch.cuda.stream(stream):
            tsa.shard_attend(L.Q, K_r, V_r, lens_r, idx, kreq_t, k, lo, w.scale, O_parts[r], lse[r], ws, stream)
    if reps == 0:  # --profile: every shard's calls once more, untimed
        for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):
            tsa.shard_select(L.Q, K_r, lens_r, kreq_t, k, w.scale, lo, cs[r], cr[r], ws, stream)
        tsa.shard_merge(cs, cr, shape, kreq_t, k, idx, ws0, stream)
        for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):
            tsa.shard_attend(L.Q, K_r, V_r, lens_r, idx, kreq_t, k, lo, w.scale, O_parts[r], lse[r], ws, stream)
        tsa.shard_combine(O_parts, lse, shape, O, stream)
        stream.synchronize()
        return {}
    flush = L2Flush(dev)
    f_us = graph_us(flush, stream, reps)
    out = {}
    for name, fn in calls.items():
        out[name] = {"warm_us": graph_us(fn, stream, reps),
                     "cold_us": graph_us(lambda fn=fn: (flush(), fn()), stream, reps) - f_us}
    for _, _, _, _, ws in shards:
        tsa.check_device_status(ws, stream)
    per_shard = out["shard_select (one shard)"]["cold_us"] + out["shard_attend (one shard)"]["cold_us"]
    out["shards"] = R
    out["exchanged_bytes"] = {"candidates": R * B * Hkv * k * 8, "parts": R * B * w.Hq * 129 * 4}
    out["step_cold_us_one_gpu_emulation"] = (per_shard * R + out["shard_merge"]["cold_us"] +
                                             out["shard_combine"]["cold_us"])
    out["note"] = ("one GPU runs every shard in turn; on R GPUs the shards' select and attend calls run at once "
                   "and two all-gathers of the exchanged bytes are added")
    return out


def overlap_probe(tsa, w, plan, lens, dev, stream, n_layers=32, keep=0.7, reps=10):
    """tsa_index_overlap over `n_layers` layers' index lists of this workload's
    shape (synthetic lists: each layer keeps a fraction `keep` of the previous
    layer's rows), timed with CUDA events around `reps` launches."""
    from top_sparse_attention_02_b200 import inputs

    n = [int(lens[b]) if w.block == 1 else -(-int(lens[b]) // w.block) for b in range(w.B) for _ in range(w.Hkv)]
    k = [int(plan.kreq[b]) for b in range(w.B) for _ in range(w.Hkv)]
    idx = inputs.layer_index_lists(n_layers, n, k, plan.k_max, keep, seed=5).to(dev)
    units = idx.shape[1]
    counts = torch.empty(n_layers, n_layers, units, dtype=torch.int32, device=dev)
    M = torch.empty(n_layers, n_layers, dtype=torch.float64, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    tsa.index_overlap(idx, counts, M, ws, stream)
    if reps == 0:  # --profile: one launch, untimed
        stream.synchronize()
        return {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            tsa.index_overlap(idx, counts, M, ws, stream)
        e1.record(stream)
    stream.synchronize()
    tsa.check_device_status(ws, stream)
    return {"layers": n_layers, "units": units, "k_max": plan.k_max, "us": e0.elapsed_time(e1) * 1e3 / reps,
            "M_next_layer_mean": float(torch.diagonal(M, -1).mean()) if n_layers > 1 else 1.0}


def copy_probe(tsa, dev, stream, nbytes=2 << 30):
    a = torch.empty(nbytes // 2, dtype=torch.uint8, device=dev)
    b = torch.empty_like(a)
    a.fill_(1)
    best = 0.0
    for _ in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        tsa.hbm_copy(a, b, a.numel(), stream)
        e1.record(stream)
        torch.cuda.synchronize()
        best = max(best, 2 * a.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del a, b
    return best


def read_probe(tsa, dev, ws, stream, nbytes=2 << 30, reps=10):
    """Read-only stream ceiling: tsa_hbm_read over 2 GiB (no stores), `reps`
    launches back to back between two events, best of 3."""
    a = torch.ones(nbytes, dtype=torch.uint8, device=dev)
    tsa.hbm_read(a, a.numel(), ws, stream)
    best = 0.0
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            tsa.hbm_read(a, a.numel(), ws, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        best = max(best, reps * a.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del a
    return best


def gather_probe(tsa, w, plan, layers, idx, ws, stream, reps=10):
    """Random-row gather ceiling on the attention stage's own rows: the rows layer 0
    selected, fetched from a reuse layer's K and V by tsa_hbm_gather (bulk copies
    into shared memory, nothing kept), each pair of launches after an L2 flush
    (minus the flush alone), as the cold attention stage is timed.  Returns GB/s
    over the bytes fetched."""
    sel = [li for li, m in enumerate(w.route) if m == 1]
    if not sel or w.block != 1:
        return None
    src_layer = layers[1] if len(layers) > 1 else layers[0]
    ix = idx[sel[0]].reshape(w.B * w.Hkv, -1).long()
    base = torch.arange(w.B * w.Hkv, device=ix.device).unsqueeze(1) * w.Ncap
    rows = (ix + base)[ix >= 0].to(torch.int32).contiguous()
    K2 = src_layer.K.view(torch.uint8).reshape(-1)
    V2 = src_layer.V.view(torch.uint8).reshape(-1)

    def both():
        tsa.hbm_gather(K2, rows, ws, stream)
        tsa.hbm_gather(V2, rows, ws, stream)

    flush = L2Flush(ix.device)
    us = graph_us(lambda: (flush(), both()), stream, reps) - graph_us(flush, stream, reps)
    warm_us = graph_us(both, stream, reps)
    # the same kind of gather at a volume where the fixed latency no longer
    # counts: every row of that cache's K, in a random order (256-byte rows)
    nall = K2.numel() // 256
    mult = 1000003  # a prime: i -> i * mult mod nall is a permutation when nall is not its multiple
    while nall % mult == 0:
        mult += 2
    perm = (torch.arange(nall, device=ix.device, dtype=torch.int64) * mult % nall).to(torch.int32)
    assert int(perm.min()) >= 0 and int(perm.max()) < nall
    big_us = graph_us(lambda: tsa.hbm_gather(K2, perm, ws, stream), stream, 3)
    del flush, perm
    tsa.check_device_status(ws, stream)
    nbytes = 2 * rows.numel() * 256
    return {"gbs": nbytes / (us * 1e-6) / 1e9, "us": us, "bytes": nbytes,
            "warm_gbs": nbytes / (warm_us * 1e-6) / 1e9,
            "asymptotic_gbs": nall * 256 / (big_us * 1e-6) / 1e9,
            "rows": "the K and V rows layer 0 selected, in another layer's cache; after an L2 flush"}


def attn_roofline(w, plan, stages, gather):
    """The attention stage against the random-row gather ceiling measured in this run."""
    if gather is None:
        return None
    cold = stages["cold"]
    reuse = [k for k in cold if k.endswith("_attn") and not k.startswith("L0")]
    us = statistics.mean(cold[k] for k in reuse) if reuse else cold.get("L0_attn")
    achieved = plan.bytes["gather"] / (us * 1e-6) / 1e9
    return {"kernel": "attn_kernel (one reuse layer)", "bound": "hbm random-row gather",
            "achieved": achieved, "peak": gather["asymptotic_gbs"], "unit": "GB/s",
            "frac": achieved / gather["asymptotic_gbs"],
            "peak_source": "tsa_hbm_gather of every row of a 256 MB cache in random order, this run: the "
                           "bandwidth of 256-byte row gathers once latency no longer counts",
            "same_size_probe_gbs": gather["gbs"], "frac_of_same_size_probe": achieved / gather["gbs"],
            "note": "a 10.7 MB gather is latency-bound: the probe of the same rows, with no math, reaches only "
                    "the same_size_probe_gbs",
            "algorithmic_bytes_per_launch": plan.bytes["gather"]}


def e2e_measure(tsa, w, plan, layers, step_args, O, idx, ws, kreq_t, stream, args):
    """The same step through the C ABI from host buffers, inside the timed region:
    - every layer's Q and lengths are copied host -> device from pinned memory;
    - a layer that scans its cache (SELECT in token mode, FULL) gets its K and V
      copied host -> device (the scorer reads every K row);
    - a REUSE layer leaves its K and V in pinned host memory and reads only the
      selected rows across the host link (TSA_KV_HOST, index-guided offload);
    - every layer's O and the selected indices are copied back.
    h2d_bytes_per_step counts the copies plus the rows the reuse layers read
    through the mapping."""
    from top_sparse_attention_02_b200 import binding as _b

    offload = [m == tsa.REUSE for m in w.route]
    host_in, dev_in, hkv = [], [], []
    for li, L in enumerate(layers):
        if offload[li]:
            host_in.append([L.Q.cpu().pin_memory(), L.seq_lens.cpu().pin_memory()])
            dev_in.append((L.Q, L.seq_lens))
            hkv.append((L.K.cpu().pin_memory(), L.V.cpu().pin_memory()))
        else:
            host_in.append([t.cpu().pin_memory() for t in (L.Q, L.K, L.V, L.seq_lens)])
            dev_in.append((L.Q, L.K, L.V, L.seq_lens))
            hkv.append(None)
    e2e_args = []
    for li, (a, L) in enumerate(zip(step_args, layers)):
        if not offload[li]:
            e2e_args.append(a)
            continue
        Kh, Vh = hkv[li]
        e2e_args.append(_b.step_args(L.Q, Kh, Vh, L.seq_lens, O[li], ws, mode=tsa.REUSE, scale=w.scale,
                                     k_max=plan.k_max, block=w.block, k_per_seq=kreq_t,
                                     idx_in=idx[w.reuse_from[li]], flags=tsa.KV_HOST))
    O_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in O]
    sel = [li for li, m in enumerate(w.route) if m == tsa.SELECT]
    idx_host = [torch.empty(idx[li].shape, dtype=torch.int32).pin_memory() for li in sel]
    copied = sum(t.numel() * t.element_size() for hs in host_in for t in hs)
    mapped = sum(1 for m in offload if m) * plan.bytes["gather"]
    d2h = sum(t.numel() * t.element_size() for t in O_host + idx_host)
    reps = max(1, min(args.steps, 5))

    def one():
        for hs, ds in zip(host_in, dev_in):
            for h, d in zip(hs, ds):
                d.copy_(h, non_blocking=True)
        for a in e2e_args:
            tsa.decode_step(a, stream)
        for oh, od in zip(O_host, O):
            oh.copy_(od, non_blocking=True)
        for ih, li in zip(idx_host, sel):
            ih.copy_(idx[li], non_blocking=True)

    with torch.cuda.stream(stream):  # one untimed pass: the host pointer checks, first touches
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):  # copies and kernels in one stream order
        e0.record(stream)
        for _ in range(reps):
            one()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del hkv
    return {"value": plan.step_bytes / (ms * 1e-3) / 1e12, "unit": "TB/s", "ms_per_step": ms,
            "h2d_bytes_per_step": copied + mapped, "d2h_bytes_per_step": d2h, "steps": reps,
            "h2d_copied_bytes_per_step": copied, "h2d_mapped_read_bytes_per_step": mapped,
            "note": "from pinned host buffers each step: Q and lengths of every layer and K, V of the scanning "
                    "layers copied host->device; reuse layers read only their selected K/V rows from pinned "
                    "host memory (TSA_KV_HOST); O and indices copied back; all inside the timed region"}


# ---------------------------------------------------------------- reference arm (oracle on CPU)

def run_reference(args, w_name, rank, world):
    import numpy as np

    import oracle
    from top_sparse_attention_02_b200 import workloads

    w = workloads.ALL[w_name]
    lens = workload_lens(w)
    plan = Plan(w, lens)
    layers = make_layers(w, "cpu", lens)
    cores = oracle.num_threads()
    kreq = plan.kreq

    def one_step():
        idx = {}
        for li, L in enumerate(layers):
            m = w.route[li]
            if m == 2:
                oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, kreq, plan.k_max, w.scale, mode=2,
                                   block=w.block, idx_in=idx[w.reuse_from[li]])
            else:
                _, ix, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, kreq, plan.k_max, w.scale,
                                              mode=m, block=w.block)
                idx[li] = ix

    for _ in range(min(args.warmup, 1)):
        one_step()
    t0 = time.perf_counter()
    n = 0
    while n < args.steps:
        one_step()
        n += 1
        if time.perf_counter() - t0 > 60:
            break
    s = (time.perf_counter() - t0) / n
    val = plan.step_bytes / s / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TB/s", "n_gpus": world,
        "steps": n, "warmup": args.warmup, "ms_per_step": s * 1e3, "us_per_step": s * 1e6,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V)",
        "config": config_of(w, plan, world),
        "cpu_baseline": {"value": val, "unit": "TB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} whole step(s) of the workload (all layers, all units)"},
        "e2e": {"value": val, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def cpu_baseline(w_name, budget_s=20.0, single_core_s=8.0):
    """The oracle, as it stands, on a bounded sample of the workload: whole layers of
    the step until about budget_s of host time on all host cores, then again until
    about single_core_s on one core; scaled to the metric's unit."""
    import oracle
    from top_sparse_attention_02_b200 import workloads

    w = workloads.ALL[w_name]
    lens = workload_lens(w)
    plan = Plan(w, lens)
    layers = make_layers(w, "cpu", lens)

    def run(budget):
        t0 = time.perf_counter()
        done_bytes, nlayers, idx = 0, 0, {}
        while True:
            for li, L in enumerate(layers):
                m = w.route[li]
                if m == 2:
                    oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, plan.kreq, plan.k_max, w.scale, mode=2,
                                       block=w.block, idx_in=idx[w.reuse_from[li]])
                else:
                    _, ix, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, plan.kreq, plan.k_max,
                                                  w.scale, mode=m, block=w.block)
                    idx[li] = ix
                done_bytes += plan.layer_bytes[li]
                nlayers += 1
            if time.perf_counter() - t0 > budget:
                break
        return done_bytes, nlayers, time.perf_counter() - t0

    cores = oracle.num_threads()
    done_bytes, nlayers, s = run(budget_s)
    res = {"value": done_bytes / s / 1e12, "unit": "TB/s", "cores": cores, "kind": "oracle", "seconds": s,
           "sample": f"{nlayers} layers = {nlayers // w.layers} whole step(s) of the workload "
                     "(every unit), fp64 C oracle, OpenMP over (seq, kv-head) units"}
    if single_core_s > 0:
        oracle.set_threads(1)
        try:
            b1, n1, s1 = run(single_core_s)
        finally:
            oracle.set_threads(cores)
        res["single_core"] = {"value": b1 / s1 / 1e12, "unit": "TB/s", "cores": 1, "seconds": s1,
                              "sample": f"{n1} layers = {n1 // w.layers} whole step(s), one thread"}
    return res


# ---------------------------------------------------------------- distributed plumbing

def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world, dev):
    """The slowest rank's time: every rank takes part (one all-reduce of the timing only)."""
    if world <= 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=dev)  # dev: the rank's GPU (NCCL) or "cpu" (gloo)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(step_bytes: int, ms: float, world: int) -> float:
    """TB/s of the whole job: every rank runs its own replica of the workload."""
    return world * step_bytes / (ms * 1e-3) / 1e12


def launch_ranks(n, argv):
    """Start this script as n ranks on this node (torch.distributed.run, one
    process per GPU, rendezvous on 127.0.0.1), bounded by an outer timeout."""
    import socket

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def profile_case(args, dev):
    """--profile NAME: one call path of the library, run twice eagerly and not
    timed, so that a profiler capture (-k <kernel> -s 1 -c 1) lands on a known
    launch: "handoff" (a full layer handing on its top-k: the dense attention
    writing scores and their histogram, then the top-k), "overlap" (the layer
    overlap matrix), "shard" (the four sequence-sharded calls, two shards)."""
    from top_sparse_attention_02_b200 import binding as tsa

    w = workload_of(args)
    lens = workload_lens(w)
    plan = Plan(w, lens)
    stream = torch.cuda.Stream(device=dev)
    kreq_t = torch.tensor(plan.kreq, dtype=torch.int32, device=dev)
    if args.profile == "overlap":
        for _ in range(2):
            overlap_probe(tsa, w, plan, lens, dev, stream, reps=0)
    else:
        from top_sparse_attention_02_b200 import inputs

        L0 = inputs.decode_layer(w.B, w.Hq, w.Hkv, w.Ncap, lens, plant_frac=w.plant_frac, seed=w.seed, device=dev)
        if args.profile == "handoff":
            handoff_probe(tsa, w, plan, [L0], kreq_t, stream, reps=0, only="full_handing_on_topk")
        elif args.profile == "shard":
            shard_probe(tsa, w, plan, [L0], kreq_t, stream, reps=0)
        else:
            raise SystemExit(f"--profile: unknown case {args.profile!r}")
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "workload": w.name}), flush=True)


def dry_run(args, rank, world):
    """The multi-rank plumbing alone, on the CPU (gloo, no CUDA): every rank takes
    a stand-in time, the max goes over the ranks, rank 0 prints the line."""
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        barrier(world)
        ms = max_over_ranks(1.0 + 0.25 * rank, world, "cpu")
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": whole_job_value(10 ** 9, ms, world), "unit": "TB/s",
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                              "dry_run": True}), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="reuse128k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--probes", action="store_true",
                    help="also time layer 0 as a full layer with and without handing on its top-k, "
                         "and the layer overlap matrix over 32 layers of this shape")
    ap.add_argument("--offload", action="store_true",
                    help="block-mode workloads: also time a layer whose K/V sit in pinned host memory")
    ap.add_argument("--ncap", type=int, default=0,
                    help="shrink the workload's context to this many tokens (profiler captures only)")
    ap.add_argument("--dry-run", action="store_true",
                    help="only the rank plumbing (start, barrier, max over ranks) on the CPU over gloo")
    ap.add_argument("--profile", default="",
                    help="run one call path twice, untimed, for a profiler capture: handoff | overlap | shard")
    args = ap.parse_args()

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # not started as a rank: start --gpus ranks of this same command
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        sys.exit(2)
    if args.dry_run:
        dry_run(args, rank, world)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        res = run_reference(args, args.workload, rank, world)
        print(json.dumps(res), flush=True)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.profile:
        profile_case(args, dev)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        res = run_ours(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args.workload)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
