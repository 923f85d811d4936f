"""Benchmark: decode of one CSA layer at 128K context (B=32 sequences, 1 new token each, 32768 FP4
compressed entries per sequence, top-512, window 128, 64 heads x 512) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path for one decode token of every sequence: compress the completed group
(pooling), FP4-pack the new entry and its indexer key, lightning-indexer scores over all entries,
top-k, attention over the selected entries plus the window.  Eight independent layer states (3.7 GB)
are rotated so every step reads its caches from HBM, not from the 126 MB L2.  Steps are replayed from
CUDA graphs; timing uses CUDA events on the launching stream, max over ranks.  Under torchrun every
rank runs its own batch of 32 sequences (weak scaling, no collective on the data path).
`--impl reference` times the CPU oracle (the reference arm) on a bounded sample.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode CSA tokens/sec (all heads) at 128K ctx on 1 B200; HBM GB/s as % of peak"
UNIT = "tokens/s"
LAYERS = 8
CSRC = os.path.join(ROOT, "compressed_sparse_attention_18_b200", "csrc")
# committed ncu summaries; their dram figures count only while the kernel sources still hash the same
ATTN_PROFILE = os.path.join(ROOT, "profiles", "attention_cfg2_decode.txt")
ATTN_SRC = [os.path.join(CSRC, "attn_tc.cu"), os.path.join(CSRC, "attn.cu")]
SCORE_PROFILE = os.path.join(ROOT, "profiles", "index_score_tc_kernel_cfg2_decode.txt")
INDEX_SRC = [os.path.join(CSRC, "index_tc.cu")]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=64)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=400)
    p.add_argument("--cpu-sample", type=int, default=2, help="sequences the CPU oracle times (cpu_baseline)")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other workloads (cfg1, cfg3 prefill, cfg4, cfg5) that a 1-GPU run times after the "
                        "headline")
    p.add_argument("--profile", action="store_true",
                   help="profiling case: one layer state, --steps eager steps, no timing (for ncu)")
    p.add_argument("--rows", action="store_true",
                   help="time the hot-path rows outside the decode step (HCA pooling and dense attention, "
                        "cross-layer reuse, hierarchical index), one JSON line each")
    p.add_argument("--spec", action="store_true",
                   help="multi-query decode with speculative positions: 5 draft positions per sequence, "
                        "B=32 at 128K context (index + top-k + attention), one JSON line")
    p.add_argument("--prefill", action="store_true",
                   help="chunked causal prefill of one 32768-token sequence (4096-token chunks), one JSON line")
    p.add_argument("--flops", action="store_true",
                   help="analytic precision-weighted decode FLOPs per token from 4K to 1M context next to the "
                        "measured decode step at each context, one JSON line each")
    return p.parse_args()


def dist_init(n, backend=None):
    """One process per GPU (torchrun env); NCCL on GPUs, gloo when the host has none (CPU tests)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x, world, device):
    """The slowest rank's time: every multi-GPU number is the max over ranks."""
    if world > 1:
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return float(x)


def whole_job_rate(units_per_rank, world, ms):
    """Units all ranks processed per second over the max-over-ranks time (weak scaling: fixed work per rank)."""
    return units_per_rank * world / (ms / 1e3)


def config_dict(s):
    return {"workload": s.name, "B": s.B, "context_tokens": s.T, "entries": s.n_c, "ratio": s.r, "heads": s.H,
            "head_dim": s.d, "fp4_dims": s.d_n, "rope_dims": s.d_r, "indexer": f"{s.H_I}x{s.d_I} fp4", "top_k": s.k,
            "window": s.W, "layers_rotated": LAYERS, "l2": "inputs larger than L2 (8 rotated layer states)",
            "cuda_graph": True}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def score_kernel_bytes(s, B):
    """Algorithmic bytes of one index-score launch: every visible key (64 B codes + 4 B scales), the
    score written per key, the queries (bf16) and head weights."""
    return B * (s.n_c * (s.d_I // 2 + s.d_I // 32 + 4) + s.H_I * s.d_I * 2 + s.H_I * 4)


def index_topk_bytes(s, B):
    """Algorithmic bytes of one on-chip index + top-k launch (CSA_ONCHIP_TOPK): every visible key (64 B
    codes + 4 B scales), the queries (bf16) and head weights in, the k selected ids out."""
    return B * (s.n_c * (s.d_I // 2 + s.d_I // 32) + s.H_I * s.d_I * 2 + s.H_I * 4 + s.k * 4)


def attention_bytes(s, B):
    """Algorithmic bytes of the attention stage for one decode step: per sequence the k selected entries
    as stored (FP4 codes, 16 B of E4M3 scales, bf16 RoPE slice) and their ids, the window rows (bf16), the
    query heads (bf16) in, the output heads (bf16) and lse out."""
    entry = s.d_n // 2 + 16 + s.d_r * 2
    return B * (s.k * (entry + 4) + s.W * s.d * 2 + s.H * s.d * 2 * 2 + s.H * 4)


# Precision weights of the decode-FLOP curve ("DeepSeek-V4.1-Flash - Pushing the Limits of KV Cache
# Compression", Fig. 2: BF16 operations count 1, FP8 0.5, FP4 0.25).
FLOP_WEIGHT = {"bf16": 1.0, "fp8": 0.5, "fp4": 0.25, "fp32": 1.0}


def decode_flops(T, s, mode="full", pool=16384):
    """Precision-weighted FLOPs of one decode token of one attention layer at context T (tokens), by part.

    Counted as this path computes them: the indexer's q_I.k_I products in FP4 (2 H_I d_I per scored
    entry) and its ReLU-weighted head sum in fp32 (2 H_I per entry); the attention's two tensor-core
    products in bf16 (2 H d each per key, keys = min(k, entries) + window; HCA: every entry + window);
    the compressor's k_I projection of the new entry in bf16 (2 d d_I, once per r tokens).  The C, Z
    projections come from upstream layers and the top-k compares, so neither counts.  Modes: "full"
    scores every visible entry, "reindex" only a candidate pool of `pool` entries (the hierarchical
    indexer's later layers), "reuse" runs no indexer, "hca" is the dense 128x layer."""
    w = FLOP_WEIGHT
    r = 128 if mode == "hca" else s.r
    n = T // r
    parts = {}
    if mode != "hca":
        parts["compressor_k_I"] = w["bf16"] * 2 * s.d * s.d_I / r
    scored = {"full": n, "reindex": min(n, pool), "reuse": 0, "hca": 0}[mode]
    parts["indexer"] = w["fp4"] * 2 * s.H_I * s.d_I * scored + w["fp32"] * 2 * s.H_I * scored
    keys = (n if mode == "hca" else min(s.k, n)) + min(s.W, T)
    parts["attention"] = w["bf16"] * 4 * s.H * s.d * keys
    return {"total": sum(parts.values()), "parts": parts, "entries": n, "keys": keys}


def sources_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(p, "rb").read())
    return h.hexdigest()


def profiled_traffic(path, srcs):
    """dram bytes per launch from a committed ncu summary, if it was taken on the current sources."""
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"sources_sha256:\s*([0-9a-f]+)", text)
    if not m or not h:
        return None
    return float(m.group(1)) if h.group(1) == sources_hash(srcs) else None


class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index):
        self.dev = dev_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if "Active" in r[5 + i] and "Not" not in r[5 + i]:
                    reasons.add(n)
        # the samples while the GPU is busy (the top half of the clock readings)
        busy = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return
    from csa_workloads import CFG2
    from oracle import csa_oracle as O
    import numpy as np
    from threadpoolctl import threadpool_limits
    s = CFG2
    # each step: one sequence's decode through the oracle (index over 32768 entries, top-k, attention)
    n = s.n_c
    g = torch.Generator().manual_seed(1)
    kv = torch.randn((n, s.d), generator=g).to(torch.bfloat16).double().numpy()
    ki = torch.randn((n, s.d_I), generator=g).to(torch.bfloat16).double().numpy()
    win = torch.randn((s.W, s.d), generator=g).to(torch.bfloat16).double().numpy()
    with threadpool_limits(1):
        kc, ks, _ = O.pack_fp4(ki, 0, 1.0)
        c, sc, rp = O.pack_fp4(kv, s.d_r, 1.0)
        rows = O.entry_kv(c, sc, rp, s.d_n, 1.0)

        def step(i):
            gg = torch.Generator().manual_seed(100 + i)
            q = torch.randn((1, s.H, s.d), generator=gg).to(torch.bfloat16).double().numpy()
            qI = torch.randn((1, s.H_I, s.d_I), generator=gg).to(torch.bfloat16).double().numpy()
            w = (torch.randn((1, s.H_I), generator=gg) * s.H_I ** -0.5).double().numpy()
            scr, ids = O.index_scores(qI, w, 1.0, kc, ks, 1.0, [s.T - 1], n, s.r)
            idx, _ = O.topk(scr, ids, s.k)
            O.attention(q, [s.T - 1], rows, idx, n, win, s.T - s.W, s.W, s.d ** -0.5)

        for i in range(min(args.warmup, 1)):
            step(i)
        budget = 90.0
        t0 = time.perf_counter()
        done = 0
        while done < args.steps and (done == 0 or time.perf_counter() - t0 < budget):
            step(done)
            done += 1
        el = time.perf_counter() - t0
    val = done / el
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": done, "warmup": min(args.warmup, 1),
            "ms_per_step": el * 1e3 / done, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference", "config": config_dict(s),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{done} decode tokens (one sequence each: index over {n} entries, top-{s.k}, "
                                       f"attention over {s.k}+{s.W} keys), numpy fp64, 1 thread"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------- our arm

class StepGraphs:
    """CUDA graphs of 1..L consecutive layer steps, captured before timing starts.

    run(k) replays k steps as k // L graphs of L steps plus one graph of k % L steps.  prepare() captures
    (and replays once) every graph run() will need for the given step counts; freeze() forbids any
    later capture, so a timed region that asked for an unprepared graph raises instead of timing a
    capture and an instantiation."""

    def __init__(self, run_layers, set_early, stream, layers, graph_cls=None, capture=None):
        self.run_layers, self.set_early, self.stream, self.L = run_layers, set_early, stream, layers
        self.graph_cls = graph_cls or torch.cuda.CUDAGraph
        self.capture = capture or (lambda g: torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"))
        self.graphs = {}
        self.frozen = False
        self.captures = 0

    def needed(self, k, with_marks=False):
        keys = set()
        if k >= self.L:
            keys.add((self.L, with_marks))
        if k % self.L:
            keys.add((k % self.L, with_marks))
        return keys

    def graph_for(self, n, with_marks):
        key = (n, with_marks)
        if key not in self.graphs:
            if self.frozen:
                raise RuntimeError(f"graph of {n} steps (marks={with_marks}) was not captured before timing")
            g = self.graph_cls()
            # the marked graph runs the same launch plan (the early start included); its events serialise
            # the stages, so its kernels only lose the overlap with their predecessors
            self.set_early(True)
            with self.capture(g):
                self.run_layers(n, with_marks)
            self.graphs[key] = g
            self.captures += 1
        return self.graphs[key]

    def prepare(self, *counts, with_marks=False):
        keys = set()
        for k in counts:
            keys |= self.needed(k, with_marks)
        for n, m in sorted(keys):
            self.graph_for(n, m)
            with torch.cuda.stream(self.stream):
                self.graphs[(n, m)].replay()

    def freeze(self):
        self.frozen = True

    def run(self, k, with_marks=False):
        with torch.cuda.stream(self.stream):
            for _ in range(k // self.L):
                self.graph_for(self.L, with_marks).replay()
            if k % self.L:
                self.graph_for(k % self.L, with_marks).replay()


def cpu_baseline(nseq):
    """The oracle as it stands on a bounded sample: nseq decode tokens on 1 host thread."""
    from csa_workloads import CFG2
    from oracle import csa_oracle as O
    from threadpoolctl import threadpool_limits
    s = CFG2
    g = torch.Generator().manual_seed(2)
    kv = torch.randn((s.n_c, s.d), generator=g).to(torch.bfloat16).double().numpy()
    ki = torch.randn((s.n_c, s.d_I), generator=g).to(torch.bfloat16).double().numpy()
    win = torch.randn((s.W, s.d), generator=g).to(torch.bfloat16).double().numpy()
    with threadpool_limits(1):
        kc, ks, _ = O.pack_fp4(ki, 0, 1.0)
        c, sc, rp = O.pack_fp4(kv, s.d_r, 1.0)
        rows = O.entry_kv(c, sc, rp, s.d_n, 1.0)
        t0 = time.perf_counter()
        for i in range(nseq):
            q = torch.randn((1, s.H, s.d), generator=g).to(torch.bfloat16).double().numpy()
            qI = torch.randn((1, s.H_I, s.d_I), generator=g).to(torch.bfloat16).double().numpy()
            w = (torch.randn((1, s.H_I), generator=g) * s.H_I ** -0.5).double().numpy()
            scr, ids = O.index_scores(qI, w, 1.0, kc, ks, 1.0, [s.T - 1], s.n_c, s.r)
            idx, _ = O.topk(scr, ids, s.k)
            O.attention(q, [s.T - 1], rows, idx, s.n_c, win, s.T - s.W, s.W, s.d ** -0.5)
        el = time.perf_counter() - t0
    return {"value": nseq / el, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{nseq} decode tokens of the same workload (one sequence each: index over {s.n_c} entries, "
                      f"top-{s.k}, attention over {s.k}+{s.W} keys; pack of the caches untimed), numpy fp64, 1 thread"}


def run_ours(args, rank, world):
    import compressed_sparse_attention_18_b200 as csa
    from compressed_sparse_attention_18_b200.layer import CSADecodeLayer, LayerShape
    from csa_workloads import CFG2, decode_inputs
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    s = CFG2
    ls = LayerShape(B=s.B, n_max=s.n_c, r=s.r, H=s.H, d=s.d, d_r=s.d_r, H_I=s.H_I, d_I=s.d_I, k=s.k, W=s.W)
    layers, inputs = [], []
    for li in range(LAYERS):
        L = CSADecodeLayer(ls, dev)
        inp = decode_inputs(s, seed=1000 * rank + li, device=dev)
        L.load_history(inp["kv_src"], inp["kI_src"], s.n_c)
        L.win.copy_(inp["win_kv"])
        del inp["kv_src"], inp["kI_src"]
        layers.append(L)
        inputs.append(inp)
        torch.cuda.synchronize()
    torch.cuda.empty_cache()

    stream = torch.cuda.Stream(dev)
    marks = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(LAYERS)]

    def run_layers(n, with_marks):
        for li in range(n):
            inp = inputs[li]
            layers[li].step(inp["C"], inp["Z"], inp["b_pos"], inp["W_IK"], inp["q"], inp["q_I"], inp["w"],
                            stream=stream, marks=marks[li] if with_marks else None)

    def set_early(flag):
        for L in layers:
            L.early = flag

    # eager warm-up (also sets kernel attributes before capture)
    with torch.cuda.stream(stream):
        run_layers(LAYERS, False)
    stream.synchronize()
    steps = StepGraphs(run_layers, set_early, stream, LAYERS)
    # every graph the warm-up, the timed loop and the stage replay use is captured, instantiated and
    # replayed once here, before timing starts; the timed region only replays
    steps.prepare(max(args.warmup, 3), args.steps)
    steps.prepare(LAYERS, with_marks=True)
    steps.freeze()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    # the warm-up steps run right before the timed region (after the sampler's start-up, which leaves the
    # GPU idle), then a synchronize and the barrier
    steps.run(max(args.warmup, 3))
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    steps.run(args.steps)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = clk.stop()
    ms = t0.elapsed_time(t1)
    # per-stage times: a second timed region replaying the same steps from a graph with an event at every
    # stage boundary.  The events serialise the stages, so this is the SERIALISED stage-by-stage plan
    # (no early-start overlap, each kernel's full launch and ramp inside its stage), not the headline's
    # schedule; the JSON line labels it so.
    steps.run(LAYERS, with_marks=True)
    stream.synchronize()
    steps.run(LAYERS, with_marks=True)
    stream.synchronize()
    stage = [[marks[li][j].elapsed_time(marks[li][j + 1]) for j in range(4)] for li in range(LAYERS)]
    score_ms = statistics.mean(st[1] for st in stage)
    ms = max_over_ranks(ms, world, dev)
    value = whole_job_rate(s.B * args.steps, world, ms)

    # ---- end to end through the public API: pinned host inputs in, result out, every step
    e2e = run_e2e(args, layers, inputs, stream, dev, world)

    if rank != 0:
        return
    hbm, kind = peaks()
    attn_ms = statistics.mean(st[3] for st in stage)
    abytes = attention_bytes(s, s.B)
    a_achieved = abytes / (attn_ms / 1e3) / 1e9
    bpl = score_kernel_bytes(s, s.B)
    achieved = bpl / (score_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp4-e2m1/bf16", "data": "synthetic", "config": config_dict(s),
        "gpu_launches": layers[0].kernels_per_step * args.steps,
        "clocks": clocks,
        "stages_ms": {"compress_pack": statistics.mean(st[0] for st in stage), "index_score": score_ms,
                      "topk": statistics.mean(st[2] for st in stage), "attention": attn_ms},
        "stages_plan": "the same launch plan replayed with an event at every stage boundary (stages serialised, "
                       "no overlap between kernels); value/ms_per_step time the overlapped schedule",
        # the dominant stage: tcgen05 attention over one 128-key tile per CTA plus the split merge
        "roofline": {"bound": "hbm", "kernel": "attn_tc_kernel + attn_merge_kernel (attention stage)",
                     "timed_on": "stage-serialised replay of the same launch plan",
                     "achieved": a_achieved, "peak": hbm, "peak_kind": kind, "unit": "GB/s",
                     "frac": a_achieved / hbm, "traffic": profiled_traffic(ATTN_PROFILE, ATTN_SRC),
                     "algorithmic_bytes_per_launch": abytes},
        # the streaming stage: every FP4 indexer key of every sequence
        "roofline_index": {"bound": "hbm", "kernel": "index_score_tc_kernel",
                           "timed_on": "stage-serialised replay of the same launch plan",
                           "achieved": achieved, "peak": hbm,
                           "peak_kind": kind, "unit": "GB/s", "frac": achieved / hbm,
                           "traffic": profiled_traffic(SCORE_PROFILE, INDEX_SRC), "algorithmic_bytes_per_launch": bpl},
        "step_hbm_gbs": 2682432 * s.B / (ms / args.steps / 1e3) / 1e9,
        "e2e": e2e,
    }
    if world == 1 or rank == 0:
        line["cpu_baseline"] = cpu_baseline(args.cpu_sample) if (world == 1 and args.cpu_sample > 0) else None
    if world == 1 and not args.no_configs:
        line["other_configs"] = other_configs()
    print(json.dumps(line), flush=True)


def run_e2e(args, layers, inputs, stream, dev, world):
    """The same metric through the public API with host buffers: every step copies its inputs (C, Z,
    q, q_I, w and the new token's window row) from pinned host memory to the device and reads the
    attention output back.  A step's inputs sit in one pinned host buffer and go over in one copy into one
    device buffer whose views are the step's input tensors (the window row is then moved into the layer's
    window inside the step's CUDA graph).  The copies run on their own streams (host-to-device and
    device-to-host, so both directions move at once) and events order copy -> step -> read-back per step,
    so the copies of one step overlap the kernels of its neighbours.  All copies of every step are inside
    the timed region."""
    s_layers = len(layers)
    keys = ("C", "Z", "q", "q_I", "w")
    staged = []
    for li in range(s_layers):
        inp, L = inputs[li], layers[li]
        parts = [(k, inp[k]) for k in keys] + [("win_row", L.win[:, -1:].contiguous())]
        offs, o = {}, 0
        for k, t in parts:
            offs[k] = o
            o = (o + t.numel() * t.element_size() + 255) // 256 * 256
        hbuf = torch.empty(o, dtype=torch.uint8).pin_memory()
        dbuf = torch.empty(o, dtype=torch.uint8, device=dev)
        dview = {}
        for k, t in parts:
            nb = t.numel() * t.element_size()
            hbuf[offs[k]:offs[k] + nb].copy_(t.reshape(-1).view(torch.uint8).cpu())
            dview[k] = dbuf[offs[k]:offs[k] + nb].view(t.dtype).view(t.shape)
        staged.append({"h": hbuf, "d": dbuf, "v": dview,
                       "out": torch.empty_like(L.out, device="cpu").pin_memory()})
    nbytes_in = sum(staged[0]["v"][k].numel() * staged[0]["v"][k].element_size() for k in keys + ("win_row",))
    nbytes_out = staged[0]["out"].numel() * staged[0]["out"].element_size()
    steps = max(args.e2e_steps, 8)
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)

    def compute(li):
        L, inp, v = layers[li], inputs[li], staged[li]["v"]
        L.win[:, -1:].copy_(v["win_row"])
        L.step(v["C"], v["Z"], inp["b_pos"], inp["W_IK"], v["q"], v["q_I"], v["w"], stream=stream)

    graphs = []
    for li in range(s_layers):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            compute(li)
        graphs.append(g)
    ev_in = [torch.cuda.Event() for _ in range(s_layers)]
    ev_done = [torch.cuda.Event() for _ in range(s_layers)]
    used = [False] * s_layers

    def one(i):
        li = i % s_layers
        st = staged[li]
        with torch.cuda.stream(h2d):
            if used[li]:
                h2d.wait_event(ev_done[li])                   # the previous step on this layer has read its inputs
            st["d"].copy_(st["h"], non_blocking=True)
            ev_in[li].record(h2d)
        stream.wait_event(ev_in[li])
        graphs[li].replay()
        ev_done[li].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done[li])
            st["out"].copy_(layers[li].out, non_blocking=True)
        used[li] = True

    with torch.cuda.stream(stream):
        for i in range(2 * s_layers):
            one(i)
    torch.cuda.synchronize()
    # the packed inputs are the step's inputs: layer 0 run from them selects the same entries as when run
    # from the original input tensors (the top-k writes its k ids in no fixed slot order, so they are
    # compared as sorted lists) and gives the same output up to the summation order that slot order sets
    got = staged[0]["out"].clone()
    got_idx = layers[0].idx.sort(dim=-1).values
    L0, i0 = layers[0], inputs[0]
    with torch.cuda.stream(stream):
        L0.step(i0["C"], i0["Z"], i0["b_pos"], i0["W_IK"], i0["q"], i0["q_I"], i0["w"], stream=stream)
    torch.cuda.synchronize()
    ref = L0.out.cpu().float()
    if not torch.equal(got_idx, L0.idx.sort(dim=-1).values) or \
            (got.float() - ref).abs().max().item() > 2.0 ** -6 * max(ref.abs().max().item(), 1.0):
        raise RuntimeError("end-to-end path: the packed inputs do not reproduce the step's result")
    if world > 1:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    stream.wait_event(t0)
    with torch.cuda.stream(stream):
        for i in range(steps):
            one(i)
    d2h.wait_event(ev_done[(steps - 1) % s_layers])
    t1.record(d2h)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    ms = max_over_ranks(ms, world, dev)
    B = layers[0].s.B
    return {"value": whole_job_rate(B * steps, world, ms), "unit": UNIT, "h2d_bytes_per_step": nbytes_in,
            "d2h_bytes_per_step": nbytes_out, "steps": steps,
            "note": "pinned host buffers: one host-to-device copy of the step's packed inputs and one read-back "
                    "per step, on two copy streams overlapped with the neighbouring steps' kernels (CUDA graph "
                    "per layer step)"}


def _graph_ms(fn, reps, states, warm=3):
    """Mean device time of fn(i): fn(0) .. fn(states - 1) (the rotated input states) captured in one CUDA
    graph after `warm` eager calls, the graph replayed `reps` times between CUDA events, so the host's
    launch overhead is not timed (as for the decode step)."""
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        for i in range(states):
            fn(i)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / (reps * states)


GRAPH_TIMED = "CUDA graph replay of the row's calls over its rotated states (host launch overhead not timed)"


def _tensor_peak(sustained=False):
    """bf16 dense peak: the burst figure for a kernel timed alone, the sustained one inside a long step."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        if sustained and "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"]), "measured"
        return float(d["bf16_tflops"]), "measured"
    return (1400.0 if sustained else 1590.0), "fallback"


def rows_measure(with_cpu=True):
    """The rows of the hot path that the decode step does not exercise, each timed with CUDA events on
    its own synthetic workload (caches rotated so they are read from HBM), against its roofline, with
    the oracle timed on one sequence beside it (with_cpu).  Returns one dict per row."""
    import compressed_sparse_attention_18_b200 as csa
    from csa_workloads import CFG4_HCA, CFG4_REUSE, CFG5, decode_inputs, gen, normal
    from threadpoolctl import threadpool_limits
    if with_cpu:
        from oracle import csa_oracle as O
    dev = torch.device("cuda", 0)
    hbm, hkind = peaks()
    tfl, tkind = _tensor_peak()

    def f64(x):
        return x.double().cpu().numpy()

    res = []

    def emit(d):
        if not with_cpu:
            d.pop("cpu_baseline", None)
        res.append(d)

    def cpu_time(fn):
        """seconds of one single-threaded oracle call (None when the oracle is not timed)"""
        if not with_cpu:
            return None
        with threadpool_limits(1):
            t0 = time.perf_counter()
            fn()
            return time.perf_counter() - t0

    # ---- a1 in HCA mode: 128x pooling of one 1,048,576-token sequence (C, Z read once: 2 GB)
    s = CFG4_HCA
    G = gen(3, dev)
    C = normal((1, s.T, s.d), 1.0, G, dev)
    Z = normal((1, s.T, s.d), 1.0, G, dev)
    b_pos = normal((s.r, s.d), 0.1, G, dev, torch.float32)
    c_out = torch.empty((1, s.T // s.r, s.d), dtype=torch.bfloat16, device=dev)
    ms = _graph_ms(lambda i: csa.compress(C=C, Z=Z, b_pos=b_pos, ratio=s.r, d_rope=s.d_r, rope_theta=10000.0,
                                          c_out=c_out), 10, 1)
    nbytes = 2 * s.T * s.d * 2 + (s.T // s.r) * s.d * 2
    cC, cZ, cb = f64(C[0, :64 * s.r]), f64(Z[0, :64 * s.r]), f64(b_pos)

    def pool64():
        for e in range(64):
            O.compress_pool(cC[e * s.r:(e + 1) * s.r], cZ[e * s.r:(e + 1) * s.r], cb, s.r, s.d_r, 10000.0, e * s.r)
    el = cpu_time(pool64)
    emit({"row": "a1 compress (HCA pooling, r=128)", "workload": "1 sequence x 1,048,576 tokens -> 8192 entries",
          "ms": ms, "timed": GRAPH_TIMED, "value": (s.T // s.r) / (ms / 1e3), "unit": "entries/s",
          "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm, "peak_kind": hkind,
                       "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / hbm, "algorithmic_bytes": nbytes},
          "cpu_baseline": {"value": 64 / el if el else None, "unit": "entries/s", "cores": 1, "kind": "oracle",
                           "sample": "64 entries of the same sequence"}})
    del C, Z, c_out
    torch.cuda.empty_cache()

    # ---- a6 HCA dense attention: 16 sequences over all 8192 entries + 128-token window; 4 cache copies
    R = 4
    states = []
    for li in range(R):
        inp = decode_inputs(s, seed=10 + li, device=dev, needles=0)
        cache = csa.PackedCache(s.B, s.n_c, s.d, s.d_r, dev)
        csa.pack_fp4(inp["kv_src"], cache)
        del inp["kv_src"], inp["kI_src"]
        inp["cache"] = cache
        inp["out"] = torch.empty((s.B, 1, s.H, s.d), dtype=torch.bfloat16, device=dev)
        inp["lse"] = torch.empty((s.B, 1, s.H), dtype=torch.float32, device=dev)
        states.append(inp)
    torch.cuda.synchronize()
    st0 = states[0]
    ws = torch.empty(csa.attn_workspace_size(st0["q"], st0["q_pos"], st0["cache"], st0["n_c"], None, st0["win_kv"],
                                             st0["win_pos0"], ratio=s.r, window=s.W, hca=True),
                     dtype=torch.uint8, device=dev)

    def hca(i):
        st = states[i % R]
        csa.hca_attn(st["q"], st["q_pos"], st["cache"], st["n_c"], st["win_kv"], st["win_pos0"], ratio=s.r,
                     out=st["out"], lse=st["lse"], ws=ws)
    ms = _graph_ms(hca, 10, R)
    flops = s.B * 4 * s.H * (s.n_c + s.W) * s.d
    nbytes = s.B * (s.n_c * (s.d_n // 2 + 16 + s.d_r * 2) + s.W * s.d * 2 + 2 * s.H * s.d * 2)
    el = None
    if with_cpu:
        rows = O.entry_kv(st0["cache"].codes[0].cpu().numpy(), st0["cache"].scales[0].cpu().numpy(),
                          f64(st0["cache"].rope[0]), s.d_n, 1.0)
        el = cpu_time(lambda: O.hca_attention(f64(st0["q"][0]), [s.T - 1], rows, s.n_c, s.r, f64(st0["win_kv"][0]),
                                              s.T - s.W, s.W, s.d ** -0.5))
    emit({"row": "a6 HCA dense attention", "workload": "16 sequences x (8192 entries + 128 window), 64 heads x 512",
          "ms": ms, "timed": GRAPH_TIMED, "value": s.B / (ms / 1e3), "unit": "tokens/s",
          "roofline": {"bound": "tensor", "achieved": flops / (ms / 1e3) / 1e12, "peak": tfl, "peak_kind": tkind,
                       "unit": "TFLOP/s", "frac": flops / (ms / 1e3) / 1e12 / tfl, "algorithmic_flops": flops,
                       "hbm_frac": nbytes / (ms / 1e3) / 1e9 / hbm, "algorithmic_bytes": nbytes},
          "cpu_baseline": {"value": 1 / el if el else None, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                           "sample": "1 sequence of the same workload"}})
    del states, ws, st0
    torch.cuda.empty_cache()

    # ---- a7 cross-layer reuse (layer 1 Full top-2048 over 262,144 entries, layer 2 Reindex -> top-512,
    # Reuse: attention over layer 2's ids) and hierarchical index (level 1 with a pool of 1024 x 8 blocks,
    # level 2 Reindex over the pool), 4 sequences each, 2 index-cache copies rotated
    for name, s in (("a7 reuse (Full -> Reindex -> attention)", CFG4_REUSE), ("a7 hierarchical index", CFG5)):
        B = 4
        sts = []
        for li in range(2):
            inp = decode_inputs(s, seed=20 + li, device=dev, B=B, needles=0, qnorm_student_t=(s is CFG5))
            ki = csa.PackedCache(B, s.n_c, s.d_I, 0, dev)
            csa.pack_fp4(inp["kI_src"], ki)
            inp["ki"] = ki
            if s is CFG4_REUSE:
                kv = csa.PackedCache(B, s.n_c, s.d, s.d_r, dev)
                csa.pack_fp4(inp["kv_src"], kv)
                inp["kv"] = kv
            del inp["kv_src"], inp["kI_src"]
            G2 = gen(77 + li, dev)
            inp["qI2"] = normal(inp["q_I"].shape, 1.0, G2, dev)
            inp["w2"] = normal(inp["w"].shape, 0.35, G2, dev, torch.float32)
            sts.append(inp)
        torch.cuda.synchronize()
        k2 = s.extra.get("k2", s.k)

        def step(i):
            st = sts[i % 2]
            if s is CFG5:
                _, _, pool = csa.index_topk(st["q_I"], st["w"], st["ki"], st["n_c"], st["q_pos"], ratio=s.r, k=s.k,
                                            pool_blocks=s.pool_blocks)
                csa.index_topk(st["qI2"], st["w2"], st["ki"], st["n_c"], st["q_pos"], ratio=s.r, k=s.k, cand=pool)
            else:
                idx1, _, _ = csa.index_topk(st["q_I"], st["w"], st["ki"], st["n_c"], st["q_pos"], ratio=s.r, k=s.k)
                idx2, _, _ = csa.index_topk(st["qI2"], st["w2"], st["ki"], st["n_c"], st["q_pos"], ratio=s.r, k=k2,
                                            cand=idx1)
                csa.sparse_attn(st["q"], st["q_pos"], st["kv"], st["n_c"], idx2, st["win_kv"], st["win_pos0"],
                                ratio=s.r)
        ms = _graph_ms(step, 10, 2)
        per_key = s.d_I // 2 + s.d_I // 32 + 4
        nbytes = B * (s.n_c * per_key + (s.pool_blocks * 8 if s is CFG5 else s.k) * per_key)
        if s is CFG4_REUSE:
            nbytes += B * (k2 * (s.d_n // 2 + 16 + s.d_r * 2) + s.W * s.d * 2 + 2 * s.H * s.d * 2)
        el = None
        if with_cpu:
            st = sts[0]
            codes, scales = st["ki"].codes[0].cpu().numpy(), st["ki"].scales[0].cpu().numpy()
            t = int(st["q_pos"][0, 0])

            def level1():
                sc, ids = O.index_scores(f64(st["q_I"][0, 0])[None], f64(st["w"][0, 0])[None], 1.0, codes, scales,
                                         1.0, [t], s.n_c, s.r)
                O.topk(sc, ids, s.k)
            el = cpu_time(level1)
        emit({"row": name, "workload": f"{B} sequences x {s.n_c} entries, top-{s.k}" +
              (f", pool {s.pool_blocks}x8" if s is CFG5 else f", Reindex -> top-{k2}, attention"),
              "ms": ms, "timed": GRAPH_TIMED, "value": B / (ms / 1e3), "unit": "tokens/s",
              "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm, "peak_kind": hkind,
                           "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / hbm, "algorithmic_bytes": nbytes},
              "cpu_baseline": {"value": 1 / el if el else None, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                               "sample": "level-1 index + top-k of 1 sequence (a lower bound on the oracle's time)"}})
        del sts
        torch.cuda.empty_cache()
    return res


def run_rows(args):
    for d in rows_measure(with_cpu=True):
        print(json.dumps(d), flush=True)


def run_flops(args):
    """Analytic weighted FLOPs per token (every layer mode) next to the measured decode step (a Full-mode
    CSA layer: compress, index, top-k, attention) at contexts 4K .. 1M, B = 8 sequences, L2 flushed
    before every timed step."""
    import compressed_sparse_attention_18_b200 as csa  # noqa: F401  (loads the library)
    from compressed_sparse_attention_18_b200.layer import CSADecodeLayer, LayerShape
    from csa_workloads import CFG2, decode_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B = 8
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)       # larger than the 126 MB L2
    stream = torch.cuda.Stream(dev)
    for T in (4096, 16384, 65536, 131072, 262144, 1048576):
        s = dataclasses.replace(CFG2, name=f"decode_{T // 1024}k", B=B, T=T)
        ls = LayerShape(B=B, n_max=s.n_c, r=s.r, H=s.H, d=s.d, d_r=s.d_r, H_I=s.H_I, d_I=s.d_I, k=s.k, W=s.W)
        L = CSADecodeLayer(ls, dev)
        inp = decode_inputs(s, seed=5, device=dev, B=B, needles=0)
        L.load_history(inp["kv_src"], inp["kI_src"], s.n_c)
        L.win.copy_(inp["win_kv"])
        del inp["kv_src"], inp["kI_src"]
        torch.cuda.synchronize()

        def step():
            L.step(inp["C"], inp["Z"], inp["b_pos"], inp["W_IK"], inp["q"], inp["q_I"], inp["w"], stream=stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                step()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            step()
        times = []
        for i in range(max(args.warmup, 3) + 30):
            with torch.cuda.stream(stream):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
            stream.synchronize()
            if i >= max(args.warmup, 3):
                times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        curve = {m: decode_flops(T, s, m) for m in ("full", "reindex", "reuse", "hca")}
        print(json.dumps({"row": "decode FLOP curve", "context_tokens": T, "entries": s.n_c, "B": B,
                          "weighted_mflop_per_token": {m: c["total"] / 1e6 for m, c in curve.items()},
                          "full_parts_mflop": {k: v / 1e6 for k, v in curve["full"]["parts"].items()},
                          "measured_full_layer": {"ms_per_step": ms, "us_per_token": ms * 1e3 / B,
                                                  "tokens_per_s": B / (ms / 1e3), "l2": "flushed before each step"}}),
              flush=True)
        del g, L, inp
        torch.cuda.empty_cache()


def run_spec(args):
    """Speculative multi-position decode: every sequence scores, selects and attends for 5 consecutive
    draft positions at once (one multi-query index pass reads each key once for all 5), B = 32 at 128K
    context, 4 cache states rotated, CUDA events around the timed steps."""
    import compressed_sparse_attention_18_b200 as csa
    from csa_workloads import CFG2, decode_inputs, gen, normal
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = CFG2
    B, Nq, R = s.B, 5, 4
    n = s.n_c
    t0 = 4 * n - 5
    Wn = s.W + Nq - 1
    states = []
    for li in range(R):
        inp = decode_inputs(s, seed=60 + li, device=dev, needles=0)
        G = gen(70 + li, dev)
        st = {"q_I": normal((B, Nq, s.H_I, s.d_I), 1.0, G, dev), "w": normal((B, Nq, s.H_I), s.H_I ** -0.5, G, dev,
                                                                          torch.float32),
              "q": normal((B, Nq, s.H, s.d), 1.0, G, dev), "win": normal((B, Wn, s.d), 1.0, G, dev)}
        st["ki"] = csa.PackedCache(B, n, s.d_I, 0, dev)
        csa.pack_fp4(inp["kI_src"], st["ki"])
        st["kv"] = csa.PackedCache(B, n, s.d, s.d_r, dev)
        csa.pack_fp4(inp["kv_src"], st["kv"])
        del inp
        states.append(st)
    q_pos = (t0 + torch.arange(Nq, device=dev)).view(1, Nq).repeat(B, 1).contiguous()
    win_pos0 = torch.full((B,), t0 - s.W + 1, dtype=torch.int64, device=dev)
    n_c = torch.full((B,), n, dtype=torch.int32, device=dev)
    st0 = states[0]
    idx = torch.empty((B, Nq, s.k), dtype=torch.int32, device=dev)
    out = torch.empty((B, Nq, s.H, s.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Nq, s.H), dtype=torch.float32, device=dev)
    ws_i = torch.empty(max(csa.index_topk_workspace_size(st0["q_I"], st0["w"], st0["ki"], n_c, q_pos, ratio=s.r,
                                                         k=s.k), 1), dtype=torch.uint8, device=dev)
    ws_a = torch.empty(max(csa.attn_workspace_size(st0["q"], q_pos, st0["kv"], n_c, idx, st0["win"], win_pos0,
                                                   ratio=s.r, window=s.W), 1), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def step(i):
        st = states[i % R]
        csa.index_topk(st["q_I"], st["w"], st["ki"], n_c, q_pos, ratio=s.r, k=s.k, idx_out=idx, ws=ws_i)
        csa.sparse_attn(st["q"], q_pos, st["kv"], n_c, idx, st["win"], win_pos0, ratio=s.r, window=s.W, out=out,
                        lse=lse, ws=ws_a)
    ms = _graph_ms(step, 10, R)
    print(json.dumps({"row": "speculative decode (5 draft positions per sequence)", "timed": GRAPH_TIMED, "B": B,
                      "positions": Nq,
                      "context_tokens": s.T, "entries": n, "top_k": s.k, "window": s.W, "ms_per_step": ms,
                      "value": B * Nq / (ms / 1e3), "unit": "tokens/s",
                      "note": "index + top-k + attention per step (compress of the drafts' groups not included); "
                              "4 cache states rotated (inputs larger than L2)"}), flush=True)


def cfg1_measure(reps=100):
    """The small layer (4096-token sequence, 8 heads x 128, indexer 4 x 64, top-64, 16 decode positions).
    One pass = the compressor in projection mode over the whole sequence (C = x W_kv and Z = x W_g on the
    tensor cores, gated pooling with RoPE, k_I, FP4 appends of the 1024 entries and their indexer keys),
    then index + top-64 and attention over the selected entries plus the 128-token window for the 16
    positions.  The pass is replayed from one CUDA graph; L2 is flushed (a 256 MB write) before every
    timed pass and each pass is bracketed by its own events.  Returns the row's dict."""
    import compressed_sparse_attention_18_b200 as csa
    from csa_workloads import CFG1, small_layer_inputs
    s = CFG1
    dev = torch.device("cuda", 0)
    inp = small_layer_inputs(s, seed=0, device=dev)
    n = s.n_c
    bf, i32, i64 = torch.bfloat16, torch.int32, torch.int64
    kv = csa.PackedCache(1, n, s.d, s.d_r, dev, s.g)
    ki = csa.PackedCache(1, n, s.d_I, 0, dev, s.g)
    C = torch.empty((1, s.T, s.d), dtype=bf, device=dev)
    Z = torch.empty((1, s.T, s.d), dtype=bf, device=dev)
    c_out = torch.empty((1, n, s.d), dtype=bf, device=dev)
    kI_out = torch.empty((1, n, s.d_I), dtype=bf, device=dev)
    row0 = torch.zeros((1,), dtype=i32, device=dev)
    pos0 = torch.zeros((1,), dtype=i64, device=dev)
    win_pos0 = torch.zeros((1,), dtype=i64, device=dev)
    n_c = torch.full((1,), n, dtype=i32, device=dev)
    idx = torch.empty((1, s.Nq, s.k), dtype=i32, device=dev)
    out = torch.empty((1, s.Nq, s.H, s.d), dtype=bf, device=dev)
    lse = torch.empty((1, s.Nq, s.H), dtype=torch.float32, device=dev)
    q_pos = inp["q_pos"]
    ws_i = torch.empty(max(csa.index_topk_workspace_size(inp["q_I"], inp["w"], ki, n_c, q_pos, ratio=s.r, k=s.k), 1),
                       dtype=torch.uint8, device=dev)
    ws_a = torch.empty(max(csa.attn_workspace_size(inp["q"], q_pos, kv, n_c, idx, C, win_pos0, ratio=s.r,
                                                   window=s.W), 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)

    def one_pass():
        csa.compress(x=inp["x"], W_kv=inp["W_kv"], W_g=inp["W_g"], b_pos=inp["b_pos"], ratio=s.r, d_rope=s.d_r,
                     rope_theta=10000.0, pos0=pos0, W_IK=inp["W_IK"], C=C, Z=Z, c_out=c_out, kI_out=kI_out,
                     kv_cache=kv, ki_cache=ki, row0=row0, stream=stream)
        csa.index_topk(inp["q_I"], inp["w"], ki, n_c, q_pos, ratio=s.r, k=s.k, idx_out=idx, ws=ws_i, stream=stream)
        csa.sparse_attn(inp["q"], q_pos, kv, n_c, idx, C, win_pos0, ratio=s.r, window=s.W, out=out, lse=lse,
                        ws=ws_a, stream=stream)

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        one_pass()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        one_pass()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            g.replay()
            b.record(stream)
    stream.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / reps
    hbm, kind = peaks()
    # dominant algorithmic bytes: x and both weights read, C and Z written once and read once by the pooling,
    # the two FP4 caches written; the 16 positions' index and attention reads are a few hundred KB more
    nbytes = (s.T * s.d_m * 2 + 2 * s.d_m * s.d * 2 + 2 * 2 * s.T * s.d * 2
              + n * (s.d_n // 2 + s.d_n // 32 + 2 * s.d_r) + n * (s.d_I // 2 + s.d_I // 32))
    return {"row": "cfg1 small layer (compress 4096 tokens + 16 decode positions)", "workload": s.name,
            "ms": ms, "value": s.Nq / (ms / 1e3), "unit": "query tokens/s",
            "tokens_compressed_per_s": s.T / (ms / 1e3), "l2": "flushed before every timed pass",
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm, "peak_kind": kind,
                         "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / hbm, "algorithmic_bytes": nbytes}}


def other_configs():
    """Every other workload of the hot path timed on the device in the default run (the oracle is timed
    only for the headline workload here; `--prefill` and `--rows` time it beside each row)."""
    res = [cfg1_measure(), prefill_measure(3, 3, with_cpu=False)]
    torch.cuda.empty_cache()
    res += rows_measure(with_cpu=False)
    return res


def prefill_work(s):
    """Algorithmic work of the whole chunked prefill of one sequence (s.T tokens): the compressor's two
    projections (bf16 FLOPs), the causal indexer's FP4 products (query t scores (t+1) // r entries), and
    attention over min(k, visible) entries plus min(W, t+1) window rows per query and head (two bf16
    products of d per key)."""
    t = torch.arange(s.T, dtype=torch.float64)
    n_vis = torch.div(t + 1, s.r, rounding_mode="floor")
    proj = 2.0 * 2 * s.T * s.d_m * s.d
    index = float(n_vis.sum()) * s.H_I * s.d_I * 2
    keys = torch.clamp(n_vis, max=s.k) + torch.clamp(t + 1, max=s.W)
    attn = float(keys.sum()) * s.H * s.d * 4
    return {"projection": proj, "index": index, "attention": attn}


def run_prefill(args):
    steps = max(args.steps if args.steps < 1000 else 10, 1)
    warm = max(args.warmup if args.warmup < 1000 else 3, 3)
    print(json.dumps(prefill_measure(steps, warm, with_cpu=True)), flush=True)


def prefill_measure(steps, warm, with_cpu=True):
    """Chunked causal prefill of one 32768-token sequence in 4096-token chunks (d_m = 4096, 64 heads x
    512, indexer 8 x 128 FP4, top-512, window 128).  Per chunk: the compressor (projection GEMM on the
    tensor cores, gated pooling, FP4 append of the chunk's 1024 entries and their indexer keys), the
    multi-query indexer over every entry so far with the causal mask, top-512 per query, attention over
    the selected entries plus the window.  One step = the 8 chunks, replayed from one CUDA graph; inputs
    (x 256 MB, q 2 GB) are larger than L2.  Returns the JSON line's dict (the oracle timed beside it when
    with_cpu)."""
    import compressed_sparse_attention_18_b200 as csa
    from csa_workloads import CFG3, gen, normal
    from threadpoolctl import threadpool_limits
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = CFG3
    Lc = s.extra["chunk"]
    nch, n = s.T // Lc, s.n_c
    epc = Lc // s.r
    G = gen(40, dev)
    x = normal((nch, Lc, s.d_m), 1.0, G, dev)
    W_kv = normal((s.d_m, s.d), s.d_m ** -0.5, G, dev)
    W_g = normal((s.d_m, s.d), s.d_m ** -0.5, G, dev)
    b_pos = normal((s.r, s.d), 0.1, G, dev, torch.float32)
    W_IK = normal((s.d, s.d_I), s.d ** -0.5, G, dev)
    q = normal((nch, Lc, s.H, s.d), 1.0, G, dev)
    q_I = normal((nch, Lc, s.H_I, s.d_I), 1.0, G, dev)
    w = normal((nch, Lc, s.H_I), s.H_I ** -0.5, G, dev, torch.float32)
    C = torch.zeros((1, s.T, s.d), dtype=torch.bfloat16, device=dev)     # every token's C: the window KV
    Z = torch.empty((1, Lc, s.d), dtype=torch.bfloat16, device=dev)
    c_out = torch.empty((1, epc, s.d), dtype=torch.bfloat16, device=dev)
    kI_out = torch.empty((1, epc, s.d_I), dtype=torch.bfloat16, device=dev)
    kv = csa.PackedCache(1, n, s.d, s.d_r, dev)
    ki = csa.PackedCache(1, n, s.d_I, 0, dev)
    row0 = [torch.tensor([epc * c], dtype=torch.int32, device=dev) for c in range(nch)]
    pos0 = [torch.tensor([Lc * c], dtype=torch.int64, device=dev) for c in range(nch)]
    n_c = [torch.tensor([epc * (c + 1)], dtype=torch.int32, device=dev) for c in range(nch)]
    q_pos = [(Lc * c + torch.arange(Lc, dtype=torch.int64, device=dev)).view(1, Lc) for c in range(nch)]
    win_pos0 = torch.zeros((1,), dtype=torch.int64, device=dev)
    idx = torch.empty((1, Lc, s.k), dtype=torch.int32, device=dev)
    out = torch.empty((1, Lc, s.H, s.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, Lc, s.H), dtype=torch.float32, device=dev)
    ws_i = torch.empty(max(csa.index_topk_workspace_size(q_I[:1], w[:1], ki, n_c[-1], q_pos[-1], ratio=s.r, k=s.k), 1),
                       dtype=torch.uint8, device=dev)
    ws_a = torch.empty(max(max(csa.attn_workspace_size(q[c:c + 1], q_pos[c], kv, n_c[c], idx, C, win_pos0, ratio=s.r,
                                                       window=s.W) for c in range(nch)), 1),
                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize()

    def chunk(c, marks=None):
        def mark(i):
            if marks is not None:
                marks[i].record(stream)
        mark(0)
        csa.compress(x=x[c:c + 1], W_kv=W_kv, W_g=W_g, b_pos=b_pos, ratio=s.r, d_rope=s.d_r, rope_theta=10000.0,
                     pos0=pos0[c], W_IK=W_IK, C=C[:, Lc * c:Lc * (c + 1)], Z=Z, c_out=c_out, kI_out=kI_out,
                     kv_cache=kv, ki_cache=ki, row0=row0[c], stream=stream)
        mark(1)
        csa.index_topk(q_I[c:c + 1], w[c:c + 1], ki, n_c[c], q_pos[c], ratio=s.r, k=s.k, idx_out=idx, ws=ws_i,
                       stream=stream)
        mark(2)
        csa.sparse_attn(q[c:c + 1], q_pos[c], kv, n_c[c], idx, C, win_pos0, ratio=s.r, window=s.W, out=out, lse=lse,
                        ws=ws_a, stream=stream)
        mark(3)

    def prefill(marks=None):
        for c in range(nch):
            chunk(c, marks[c] if marks is not None else None)

    with torch.cuda.stream(stream):
        prefill()                                       # eager warm-up (kernel attributes set)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        prefill()
    clk = ClockSampler(0)
    clk.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            g.replay()
    e1.record(stream)
    stream.synchronize()
    clocks = clk.stop()
    ms = e0.elapsed_time(e1) / steps
    # per-stage times: eager chunks with an event at every stage boundary (serialised stages)
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nch)]
    with torch.cuda.stream(stream):
        prefill(marks)
    stream.synchronize()
    stage = {name: sum(marks[c][i].elapsed_time(marks[c][i + 1]) for c in range(nch))
             for i, name in enumerate(("compress", "index_topk", "attention"))}
    work = prefill_work(s)
    tfl, tkind = _tensor_peak()
    tfl_s = _tensor_peak(sustained=True)[0]

    def tf(flops, ms_):
        return flops / (ms_ / 1e3) / 1e12

    el = None
    if with_cpu:
        # oracle on a bounded sample: the projection of 4 tokens, and index + top-k + attention of 2 queries
        # of the last chunk (over all 8192 entries), 1 thread
        from oracle import csa_oracle as O
        f64 = lambda t_: t_.double().cpu().numpy()  # noqa: E731
        codes, scales = kv.codes[0].cpu().numpy(), kv.scales[0].cpu().numpy()
        kcodes, kscales = ki.codes[0].cpu().numpy(), ki.scales[0].cpu().numpy()
        rows = O.entry_kv(codes, scales, f64(kv.rope[0]), s.d_n, 1.0)
        win = f64(C[0, s.T - Lc - s.W:])
        with threadpool_limits(1):
            t0 = time.perf_counter()
            O.project(f64(x[-1, :4]), f64(W_kv))
            O.project(f64(x[-1, :4]), f64(W_g))
            for qq in (Lc - 2, Lc - 1):
                t = s.T - Lc + qq
                sc, ids = O.index_scores(f64(q_I[-1, qq])[None], f64(w[-1, qq])[None], 1.0, kcodes, kscales, 1.0,
                                         [t], n, s.r)
                sel, _ = O.topk(sc, ids, s.k)
                O.attention(f64(q[-1, qq])[None], [t], rows, sel, n, win, s.T - Lc - s.W, s.W, s.d ** -0.5)
            el = time.perf_counter() - t0
    line = {"row": "cfg3 chunked causal prefill", "workload": s.name,
            "config": {"B": 1, "tokens": s.T, "chunk": Lc, "d_model": s.d_m, "heads": s.H, "head_dim": s.d,
                       "indexer": f"{s.H_I}x{s.d_I} fp4", "top_k": s.k, "window": s.W,
                       "l2": "inputs larger than L2 (x 256 MB, q 2 GB)", "cuda_graph": True},
            "steps": steps, "warmup": warm, "ms_per_step": ms, "value": s.T / (ms / 1e3), "unit": "tokens/s",
            "clocks": clocks,
            "stages_ms": stage, "stages_plan": "eager chunks with an event at every stage boundary",
            "tflops": {"projection": tf(work["projection"], stage["compress"]),
                       "index_fp4": tf(work["index"], stage["index_topk"]),
                       "attention": tf(work["attention"], stage["attention"])},
            "algorithmic_flops": work,
            "roofline": {"bound": "tensor", "kernel": "attention stage (attn_tc_kernel)",
                         "achieved": tf(work["attention"], stage["attention"]), "peak": tfl_s,
                         "peak_kind": tkind + " sustained", "unit": "TFLOP/s",
                         "frac": tf(work["attention"], stage["attention"]) / tfl_s},
            "cpu_baseline": {"value": 2 / el, "unit": "query tokens/s", "cores": 1, "kind": "oracle",
                             "sample": "projection of 4 tokens + index/top-k/attention of 2 queries of the last "
                                       "chunk, numpy fp64, 1 thread"} if el else None}
    if not with_cpu:
        line.pop("cpu_baseline")
    return line


def run_profile_prefill(args):
    """Profiling case of the chunked prefill: the compressor fills the caches chunk by chunk (8 launches
    of the projection and pooling), then the last chunk's indexer, top-k and attention run once, eagerly
    (about 20 launches in all, 2.5 GB on the device)."""
    import compressed_sparse_attention_18_b200 as csa
    from csa_workloads import CFG3, gen, normal
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = CFG3
    Lc = s.extra["chunk"]
    nch, n, epc = s.T // Lc, s.n_c, Lc // s.r
    G = gen(40, dev)
    x = normal((Lc, s.d_m), 1.0, G, dev).view(1, Lc, s.d_m)
    W_kv = normal((s.d_m, s.d), s.d_m ** -0.5, G, dev)
    W_g = normal((s.d_m, s.d), s.d_m ** -0.5, G, dev)
    b_pos = normal((s.r, s.d), 0.1, G, dev, torch.float32)
    W_IK = normal((s.d, s.d_I), s.d ** -0.5, G, dev)
    C = torch.zeros((1, s.T, s.d), dtype=torch.bfloat16, device=dev)
    Z = torch.empty((1, Lc, s.d), dtype=torch.bfloat16, device=dev)
    kv = csa.PackedCache(1, n, s.d, s.d_r, dev)
    ki = csa.PackedCache(1, n, s.d_I, 0, dev)
    for c in range(nch):
        csa.compress(x=x, W_kv=W_kv, W_g=W_g, b_pos=b_pos, ratio=s.r, d_rope=s.d_r, rope_theta=10000.0,
                     pos0=torch.tensor([Lc * c], dtype=torch.int64, device=dev), W_IK=W_IK,
                     C=C[:, Lc * c:Lc * (c + 1)], Z=Z, kv_cache=kv, ki_cache=ki,
                     row0=torch.tensor([epc * c], dtype=torch.int32, device=dev))
    q = normal((1, Lc, s.H, s.d), 1.0, G, dev)
    q_I = normal((1, Lc, s.H_I, s.d_I), 1.0, G, dev)
    w = normal((1, Lc, s.H_I), s.H_I ** -0.5, G, dev, torch.float32)
    n_c = torch.tensor([n], dtype=torch.int32, device=dev)
    q_pos = (s.T - Lc + torch.arange(Lc, dtype=torch.int64, device=dev)).view(1, Lc)
    idx, _, _ = csa.index_topk(q_I, w, ki, n_c, q_pos, ratio=s.r, k=s.k)
    csa.sparse_attn(q, q_pos, kv, n_c, idx, C, torch.zeros((1,), dtype=torch.int64, device=dev), ratio=s.r,
                    window=s.W)
    torch.cuda.synchronize()
    print(json.dumps({"profile": "ok", "workload": s.name, "chunk": nch - 1}), flush=True)


def run_profile(args):
    """One layer state, `--steps` eager decode steps: the small case ncu captures run on."""
    from compressed_sparse_attention_18_b200.layer import CSADecodeLayer, LayerShape
    from csa_workloads import CFG2, decode_inputs
    s = CFG2
    ls = LayerShape(B=s.B, n_max=s.n_c, r=s.r, H=s.H, d=s.d, d_r=s.d_r, H_I=s.H_I, d_I=s.d_I, k=s.k, W=s.W)
    L = CSADecodeLayer(ls, torch.device("cuda", 0))
    inp = decode_inputs(s, seed=1, device="cuda")
    L.load_history(inp["kv_src"], inp["kI_src"], s.n_c)
    L.win.copy_(inp["win_kv"])
    del inp["kv_src"], inp["kI_src"]
    for _ in range(max(args.steps, 1)):
        L.step(inp["C"], inp["Z"], inp["b_pos"], inp["W_IK"], inp["q"], inp["q_I"], inp["w"])
    torch.cuda.synchronize()
    print(json.dumps({"profile": "ok", "steps": max(args.steps, 1), "workload": s.name}), flush=True)


def main():
    args = parse()
    if args.profile:
        run_profile_prefill(args) if args.prefill else run_profile(args)
        return
    if args.rows:
        run_rows(args)
        return
    if args.flops:
        run_flops(args)
        return
    if args.spec:
        run_spec(args)
        return
    if args.prefill:
        run_prefill(args)
        return
    rank, world = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
