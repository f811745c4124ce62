#!/usr/bin/env python3
"""Benchmark of the compressed-KV sparse decode-attention step on B200.

One step = one pass of the whole decode path over a batch: for every layer, append the decode
token through the compressor (position L-1; idempotent across steps), score every compressed
entry and select the top-k (sparse layers), attend over the selected entries plus the window.
Inputs are resident in HBM; L2 is flushed before every timed step, outside the step's events:
a 256 MiB buffer is written, then another 256 MiB buffer is read, so that the flush's dirty lines
are written back before the step starts instead of during it. The metric is decode-attention
queries*layers per second over all ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ckv|reference]

The headline workload is the 1M-context CSA layer (batch 4, the largest configuration that fits
one GPU). At N = 1 the same line also carries `per_config`: every named configuration (4K fp32,
32K, 128K HCA, 1M, mixed 64 requests) measured the same way, each with the indexer's and the
attention's roofline and its own end-to-end figure.

For N > 1 launch one rank per GPU with torch.distributed.run; every rank runs its own batch of
the workload (data-parallel requests, no collective on the data path) and rank 0 prints one JSON
line. `--impl reference` times the CPU oracle on a bounded sample of the same workload.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synth import workloads as S  # noqa: E402

METRIC = "decode attention queries*layers/s"
UNIT = "queries*layers/s"
DEFAULT_WORKLOAD = "csa_b4_ctx1m"
CONFIGS = ("csa_b1_ctx4k_fp32", "csa_b8_ctx32k", "hca_b32_ctx128k", "csa_b4_ctx1m", "mixed_64req")
FLUSH_BYTES = 256 << 20
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------------------------------------
# algorithmic bytes (per step, per layer), from the stored formats
# ------------------------------------------------------------------------------------------------

def entry_bytes(ls: S.LayerSpec, d: int) -> int:
    return S.comp_code_bytes(ls.comp_dtype, d) + (d // 16 if ls.comp_dtype == "nvfp4" else 0)


def token_bytes(ls: S.LayerSpec, d: int) -> int:
    return S.win_code_bytes(ls.win_dtype, d) + (4 if ls.win_dtype == "fp8" else 0)


MH_HEADS, MH_DIM = 64, 128  # multi-head indexer: index heads x index dim


def layer_bytes(w: S.Workload, ls: S.LayerSpec, indexer: str = "avg") -> dict:
    """Bytes a step must move for one layer: the indexer reads every candidate once (its K=V
    entry for the head-averaged score; its FP8 index entry and scale for the multi-head score)
    and the block-table entry of each 256-token block; attention reads the selected entries, the
    window tokens, the query and writes the output; the
    append reads the unfinished group's ring and writes one entry and one window token (the
    multi-head form also appends the index key: its ring, one FP8 entry)."""
    d, h = w.head_dim, w.num_heads
    idx_b = att_b = app_b = 0
    for L in w.seq_lens:
        n_c = L // ls.ratio
        if ls.top_k is not None:
            if indexer == "mh":
                idx_b += n_c * (MH_DIM + 4) + 4 * math.ceil(L / 256) + 4 * MH_HEADS * (MH_DIM + 1)
                app_b += 4 * MH_DIM + 4 + (ls.ratio - 1) * (4 * MH_DIM + 4) + MH_DIM + 4
            else:
                idx_b += n_c * entry_bytes(ls, d) + 4 * math.ceil(L / 256)
            sel = min(ls.top_k, n_c)
        else:
            sel = n_c
        att_b += sel * entry_bytes(ls, d) + min(w.window, L) * token_bytes(ls, d) + 2 * 4 * h * d
        app_b += 4 * d + 4 + (ls.ratio - 1) * (4 * d + 4) + entry_bytes(ls, d) + token_bytes(ls, d)
    return {"indexer": idx_b, "attention": att_b, "append": app_b}


# ------------------------------------------------------------------------------------------------
# environment
# ------------------------------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device="cpu") -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: int, world: int, steps: int, max_total_ms: float) -> float:
    """Whole-job rate: the units every rank processed in `steps` steps over the slowest rank's time."""
    return units_per_rank_step * world * steps / (max_total_ms / 1e3)


def tensor_record(w: S.Workload, indexer: str, avg_ms: float) -> dict:
    """Tensor-core side of the multi-head score kernel: 2 H_I d_I flops per candidate (fp16
    operands), against the measured dense bf16 rate (fp16 runs at the same rate)."""
    n_c = sum(L // ls.ratio for ls in w.layers if ls.top_k is not None for L in w.seq_lens)
    flops = 2.0 * MH_HEADS * MH_DIM * n_c
    try:
        with open(PEAKS_FILE) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured bf16 burst"
    except Exception:
        peak, src = 1590.0, "fallback"
    ach = flops / (avg_ms / 1e3) / 1e12
    return {"flops_per_launch": flops, "achieved_tflops": ach, "peak_tflops": peak, "peak_source": src,
            "frac": ach / peak}


def measured_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,power.draw")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
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
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:6]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def traffic_record(kernel: str, workload: str):
    """dram bytes per launch of `kernel` from the committed ncu summary, if the kernel source
    has not changed since it was captured (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]+)", txt)
    src = re.search(r"source_file:\s*(\S+)", txt)
    if not (m and h and src):
        return None
    try:
        cur = hashlib.sha256(open(os.path.join(ROOT, src.group(1)), "rb").read()).hexdigest()
    except OSError:
        return None
    return float(m.group(1)) if cur == h.group(1) else None


# ------------------------------------------------------------------------------------------------
# CUDA arm
# ------------------------------------------------------------------------------------------------

class Step:
    """All layers of a workload on one GPU, with the step's inputs resident in HBM."""

    def __init__(self, ckv, w: S.Workload, seed_offset: int = 0, api: str = "fused", indexer: str = "avg"):
        self.ckv, self.w, self.api, self.indexer = ckv, w, api, indexer
        wseed = S.Workload(w.name, w.seq_lens, w.num_heads, w.head_dim, w.rope_dim, w.window,
                           w.layers, w.paged, w.from_scratch, w.seed + seed_offset, w.description)
        self.gen = S.generate(wseed, "cuda")
        self.seq = self.gen["seq_len"]
        self.prev = (self.seq - 1).to(torch.int32)
        self.layers = []
        self.index = []  # per layer: None, or the multi-head indexer's plane, inputs and workspace
        for li, (lay, ls) in enumerate(zip(self.gen["layers"], w.layers)):
            cfg = ckv.LayerConfig(w.num_heads, w.head_dim, w.rope_dim, ls.ratio, w.window,
                                  ls.comp_dtype, ls.win_dtype)
            cache = ckv.cache_from_tensors(cfg, w.batch, lay["comp_codes"], lay["comp_scales"],
                                           lay["win_codes"], lay["win_scales"], lay["comp_table"],
                                           lay["win_table"])
            dl = ckv.DecodeLayer(cfg, cache, w.batch, max(w.seq_lens), ls.top_k)
            cu = lay["cu_setup"]
            n = int((cu[1:] - cu[:-1]).max().item())
            if n > 0:  # the unfinished group before the decode token (setup, untimed)
                dl.append(lay["setup_start"].to(torch.int32), lay["kv_setup"], lay["logit_setup"],
                          cu_new=cu, max_new=n)
            mh = None
            if indexer == "mh" and ls.top_k is not None:
                ix = S.generate_index(wseed, self.gen, layer=li, heads=MH_HEADS, dim=MH_DIM, device="cuda")
                icfg = ckv.IndexConfig(MH_HEADS, MH_DIM)
                icache = ckv.IndexCache(ix["codes"], ix["scales"],
                                        torch.zeros((w.batch, ls.ratio, MH_DIM), device="cuda"),
                                        torch.zeros((w.batch, ls.ratio), device="cuda"))
                if n > 0:
                    ckv.kv_index_append(cfg, cache, icfg, icache, lay["setup_start"].to(torch.int32),
                                        ix["k_setup"], lay["logit_setup"], dl.status, cu_new=cu, max_new=n,
                                        max_seq_len=dl.max_seq_len)
                wsb = ckv.mh_indexer_workspace_bytes(cfg, icfg, w.batch, dl.max_seq_len, ls.top_k)
                mh = {"ix": ix, "icfg": icfg, "icache": icache,
                      "ws": torch.empty(wsb, dtype=torch.uint8, device="cuda")}
            self.layers.append((dl, lay))
            self.index.append(mh)
        torch.cuda.synchronize()

    def inputs(self, i):
        """The step's inputs of layer i: q, new token, its logit, and (multi-head) the index
        query, head weights and new index key."""
        lay, mh = self.layers[i][1], self.index[i]
        extra = [] if mh is None else [mh["ix"]["q_index"], mh["ix"]["weights"], mh["ix"]["k_new"]]
        return [lay["q"], lay["kv_new"], lay["logit_new"]] + extra

    def run_layer(self, i, seq, prev, ins):
        dl, mh = self.layers[i][0], self.index[i]
        q, kv, lg = ins[:3]
        if mh is not None:
            qi, wt, kn = ins[3:]
            dl.append(prev, kv, lg)
            self.ckv.kv_index_append(dl.cfg, dl.cache, mh["icfg"], mh["icache"], prev, kn, lg, dl.status,
                                     max_seq_len=dl.max_seq_len)
            self.ckv.sparse_mh_indexer_topk(dl.cfg, dl.cache, mh["icfg"], mh["icache"], seq, dl.max_seq_len, qi,
                                            wt, dl.top_k, dl.idx, dl.cnt, mh["ws"], dl.status)
            return dl.attend(seq, q)
        if self.api == "fused":
            return dl.fused_step(seq, q, kv, lg)
        return dl.step(seq, prev, q, kv, lg)

    def run(self, ins_list=None, seq=None, prev=None):
        seq = self.seq if seq is None else seq
        prev = self.prev if prev is None else prev
        return [self.run_layer(i, seq, prev, self.inputs(i) if ins_list is None else ins_list[i])
                for i in range(len(self.layers))]

    def status(self) -> int:
        return max(int(dl.status[0].item()) & 0xffffffff for dl, _ in self.layers)


def roofline_record(kind: str, bytes_per_launch: float, launch_ms: list, peak: float, peak_src: str,
                    workload: str, flops_per_launch: float | None = None, note: str = "") -> dict:
    """Achieved bandwidth of one kernel kind: algorithmic bytes per launch over the average
    CUDA-event duration of its launches, against the peak."""
    avg_ms = sum(launch_ms) / len(launch_ms)
    ach = bytes_per_launch / (avg_ms / 1e3) / 1e9
    rec = {"bound": "hbm", "kernel": kind, "achieved": ach, "peak": peak, "peak_source": peak_src,
           "unit": "GB/s", "frac": ach / peak, "frac_of_8TBps": ach / 8000.0,
           "avg_launch_us": avg_ms * 1e3, "algorithmic_bytes": bytes_per_launch,
           "launches_timed": len(launch_ms), "timed_in": note,
           "traffic": traffic_record(kind, workload)}
    if flops_per_launch is not None:
        try:
            with open(PEAKS_FILE) as f:
                tpk, tsrc = float(json.load(f)["bf16_tflops"]), "measured bf16 burst"
        except Exception:
            tpk, tsrc = 1590.0, "fallback"
        tf = flops_per_launch / (avg_ms / 1e3) / 1e12
        rec["tensor"] = {"flops_per_launch": flops_per_launch, "achieved_tflops": tf, "peak_tflops": tpk,
                         "peak_source": tsrc, "frac": tf / tpk}
    return rec


def attention_flops(w: S.Workload, ls: S.LayerSpec) -> float:
    """Algorithmic tensor work of one layer's attention: 2 H D flops per key for the logits and
    2 H D per key for the weighted sum."""
    keys = 0
    for L in w.seq_lens:
        n_c = L // ls.ratio
        keys += (min(ls.top_k, n_c) if ls.top_k is not None else n_c) + min(w.window, L)
    return 4.0 * w.num_heads * w.head_dim * keys


def measure(ckv, args, w: S.Workload, dev, ws: int, rank: int, cpu_leg: bool) -> dict:
    """Every timed figure of one workload on this rank (max over ranks where it matters)."""
    step = Step(ckv, w, seed_offset=rank, api=args.api, indexer=args.indexer)
    flush_w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    def barrier():
        torch.cuda.synchronize()
        if ws > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    sparse = any(ls.top_k is not None for ls in w.layers)
    score_name = "mh_score_kernel" if args.indexer == "mh" else "score_kernel"
    dominant = score_name if sparse else "attention_kernel"

    for _ in range(args.warmup):
        flush_l2()
        step.run()
    barrier()
    if step.status() != 0:
        raise RuntimeError(f"device status {step.status():#x} after warm-up ({w.name})")

    # ---- timed region: K steps with one event pair per step, the step replayed as one CUDA graph
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for pair in ev:  # CUDA events are created on first record
        for e in pair:
            e.record(stream)
    torch.cuda.synchronize()
    step_graph, step_launch = None, "eager"
    launches_per_step = None
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            l0 = ckv.launch_count()
            with torch.cuda.graph(g):
                step.run()
            launches_per_step = ckv.launch_count() - l0
            g.replay()
            torch.cuda.synchronize()
            step_graph, step_launch = g, "one CUDA graph per step"
        except RuntimeError as exc:   # capture refused: stay eager and say so
            step_launch = "eager (graph capture failed: %s)" % str(exc).splitlines()[0][:120]
            torch.cuda.synchronize()
    launches0 = ckv.launch_count()
    barrier()
    for i in range(args.steps):
        flush_l2()
        ev[i][0].record(stream)
        if step_graph is not None:
            step_graph.replay()
        else:
            step.run()
        ev[i][1].record(stream)
    barrier()
    launches = (launches_per_step * args.steps if step_graph is not None
                else ckv.launch_count() - launches0)
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)

    # ---- kernel passes: events between kernels end the programmatic launch overlap of the
    #      kernels they separate, so each kernel kind is timed in a pass of K steps of its own, with
    #      an event pair around every launch of that kind
    def kernel_pass(which, takes):
        pairs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for li in range(len(w.layers)) if takes(w.layers[li])] for _ in range(args.steps)]
        kst = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for pair in kst + [x for row in pairs for x in row]:  # CUDA events are created on first record
            for e in pair:
                e.record(stream)
        barrier()
        for i in range(args.steps):
            flush_l2()
            kst[i][0].record(stream)
            k = 0
            for li in range(len(w.layers)):
                if takes(w.layers[li]):
                    ckv.profile_events(which, pairs[i][k][0], pairs[i][k][1])
                    k += 1
                else:
                    ckv.profile_events(which)
                step.run_layer(li, step.seq, step.prev, step.inputs(li))
            kst[i][1].record(stream)
        barrier()
        ckv.profile_events(which)
        # per step: the summed duration of this kind's launches (one per layer of the kind)
        per_step = [sum(a.elapsed_time(b) for a, b in row) for row in pairs]
        step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in kst), dev) / args.steps
        return per_step, step_ms, len(pairs[0])

    peak, peak_src = measured_peak()
    lb = [layer_bytes(w, ls, args.indexer) for ls in w.layers]
    rooflines = {}
    if sparse:
        per_step, sms, n = kernel_pass(ckv.CKV_PROF_SCORE, lambda ls: ls.top_k is not None)
        idx_bytes = sum(b["indexer"] for b, ls in zip(lb, w.layers) if ls.top_k is not None)
        rooflines["indexer"] = roofline_record(
            score_name, idx_bytes, per_step, peak, peak_src, w.name,
            note=f"a pass of K steps with an event pair around each launch of the score kernel "
                 f"({n} per step; bytes and time summed over them; that pass: {sms * 1e3:.1f} us per step)")
        if args.indexer == "mh":
            rooflines["indexer"]["tensor"] = tensor_record(w, args.indexer, sum(per_step) / len(per_step))
    per_step, sms, n = kernel_pass(ckv.CKV_PROF_ATTENTION, lambda ls: True)
    att_bytes = sum(b["attention"] for b in lb)
    rooflines["attention"] = roofline_record(
        "attention_kernel", att_bytes, per_step, peak, peak_src, w.name,
        flops_per_launch=sum(attention_flops(w, ls) for ls in w.layers),
        note=f"a pass of K steps with an event pair around the attention kernel and its split merge "
             f"of every layer ({n} per step; bytes and time summed over them; that pass: "
             f"{sms * 1e3:.1f} us per step)")
    if step.status() != 0:
        raise RuntimeError(f"device status {step.status():#x} in the timed region ({w.name})")

    # ---- end to end through the public API: pinned host inputs -> device -> result on host
    ins_h = [[x.cpu().pin_memory() for x in step.inputs(i)] for i in range(len(step.layers))]
    seq_h = step.seq.cpu().pin_memory()
    out_h = [torch.empty_like(lay["q"], device="cpu").pin_memory() for _, lay in step.layers]
    ins_d = [[torch.empty_like(x, device=dev) for x in row] for row in ins_h]
    seq_d = torch.empty_like(seq_h, device=dev)
    h2d = sum(x.numel() * x.element_size() for row in ins_h for x in row) + seq_h.numel() * 4
    d2h = sum(x.numel() * x.element_size() for x in out_h)
    need_prev = step.api == "calls" or args.indexer == "mh"

    def e2e_step():
        seq_d.copy_(seq_h, non_blocking=True)
        for row_d, row_h in zip(ins_d, ins_h):
            for a, b in zip(row_d, row_h):
                a.copy_(b, non_blocking=True)
        prev_d = (seq_d - 1).to(torch.int32) if need_prev else None
        outs = step.run(ins_d, seq_d, prev_d)
        for o, oh in zip(outs, out_h):
            oh.copy_(o, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        flush_l2()
        e2e_step()
    barrier()
    run_e2e, graph_note = e2e_step, "eager"
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                e2e_step()
            graph.replay()
            torch.cuda.synchronize()
            run_e2e, graph_note = graph.replay, "one CUDA graph per step (copies and kernels)"
        except RuntimeError as exc:   # capture refused: stay eager and say so
            graph_note = "eager (graph capture failed: %s)" % str(exc).splitlines()[0][:120]
            torch.cuda.synchronize()
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for pair in eev:
        for e in pair:
            e.record(stream)
    barrier()
    for i in range(args.steps):
        flush_l2()
        eev[i][0].record(stream)
        run_e2e()
        eev[i][1].record(stream)
    barrier()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eev), dev)

    units = w.batch * len(w.layers)  # queries*layers per step on this rank
    step_bytes = sum(sum(b.values()) for b in lb)
    rec = {
        "value": job_throughput(units, ws, args.steps, total_ms), "ms_per_step": total_ms / args.steps,
        "config": {
            "workload": w.name, "batch_per_gpu": w.batch, "seq_lens": summarize_lens(w.seq_lens),
            "heads": w.num_heads, "head_dim": w.head_dim, "rope_dim": w.rope_dim,
            "window": w.window,
            "layers": [{"ratio": ls.ratio, "top_k": ls.top_k, "comp_cache": ls.comp_dtype,
                        "win_cache": ls.win_dtype} for ls in w.layers],
            "paged": w.paged, "parallelism": f"dp{ws} (independent requests per GPU)",
            "l2": "flushed before every step outside the step events: 256 MiB written, then another "
                  "256 MiB read (the written lines are evicted before the step)",
            "step": "append decode token + indexer/top-k + attention (+ split merge), per layer",
            "api": ("kv_compress_append + kv_index_append + sparse_mh_indexer_topk + "
                    "compressed_window_attention on sparse layers" if args.indexer == "mh"
                    else "ckv_decode_step, one call per layer" if args.api == "fused"
                    else "kv_compress_append + sparse_indexer_topk + compressed_window_attention"),
            "indexer": (f"multi-head: {MH_HEADS} index heads x {MH_DIM} dims, FP8 index entries and query"
                        if args.indexer == "mh" else "head-averaged MQA logits over the K=V entries"),
            "launch": step_launch,
        },
        "hbm": {"step_bytes": step_bytes,
                "step_GBps": step_bytes / (total_ms / args.steps / 1e3) / 1e9,
                "frac_of_measured": step_bytes / (total_ms / args.steps / 1e3) / 1e9 / peak,
                "frac_of_8TBps": step_bytes / (total_ms / args.steps / 1e3) / 1e9 / 8000.0},
        "roofline": dict(rooflines["indexer" if sparse else "attention"]),
        "roofline_indexer": rooflines.get("indexer"),
        "roofline_attention": rooflines["attention"],
        "e2e": {"value": job_throughput(units, ws, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "launch": graph_note,
                "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": launches,
    }
    assert rec["roofline"]["kernel"] == dominant
    if cpu_leg:
        rec["cpu_baseline"] = cpu_baseline(w, step, args.cpu_seconds)
    del step, step_graph, ev
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def run_cuda(args, w: S.Workload):
    import compressed_kv_sparse_compress_b200 as ckv
    ckv.load_library()
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    cpu_leg = rank == 0 and ws == 1 and not args.no_cpu_baseline
    head = measure(ckv, args, w, dev, ws, rank, cpu_leg)
    per_config = None
    if ws == 1 and not args.no_per_config:
        per_config = {}
        for name in CONFIGS:
            wc = S.WORKLOADS[name]()
            if wc.name == w.name:
                rec = dict(head)
                rec.pop("cpu_baseline", None)
            else:
                rec = measure(ckv, args, wc, dev, ws, rank, False)
            per_config[name] = {k: rec[k] for k in ("value", "ms_per_step", "roofline_indexer",
                                                    "roofline_attention", "e2e", "gpu_launches")}
            per_config[name]["workload"] = wc.name
            per_config[name]["hbm_step_frac_of_measured"] = rec["hbm"]["frac_of_measured"]
    clk = clocks.stop()
    result = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": head["config"], "hbm": head["hbm"], "roofline": head["roofline"],
        "roofline_indexer": head["roofline_indexer"], "roofline_attention": head["roofline_attention"],
        "tensor": (head["roofline_indexer"] or {}).get("tensor") if args.indexer == "mh" else None,
        "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": clk,
    }
    if "cpu_baseline" in head:
        result["cpu_baseline"] = head["cpu_baseline"]
    if per_config is not None:
        result["per_config"] = per_config
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return result if rank == 0 else None


def summarize_lens(lens):
    if len(set(lens)) == 1:
        return lens[0]
    return {"n": len(lens), "min": min(lens), "median": int(statistics.median(lens)), "max": max(lens),
            "sum": sum(lens)}


# ------------------------------------------------------------------------------------------------
# CPU oracle (the reported baseline, and the --impl reference arm)
# ------------------------------------------------------------------------------------------------

def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name as lscpu prints it (else /proc/cpuinfo's)."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_request(w, gen_host, li, b, O, ix_host=None):
    """The oracle's whole step for request b of layer li (append + select + attention); with
    ix_host (the multi-head indexer's inputs of that layer) the selection is the multi-head one."""
    ls = w.layers[li]
    lay = gen_host["layers"][li]
    cfg = O.LayerCfg(w.num_heads, w.head_dim, w.rope_dim, ls.ratio, w.window, ls.comp_dtype,
                     ls.win_dtype)
    cache = O.LayerCache(lay["comp_codes"], lay["comp_scales"], lay["win_codes"], lay["win_scales"],
                         lay["comp_table"], lay["win_table"], residue=[[] for _ in range(w.batch)])
    L = w.seq_lens[b]
    start = int(lay["setup_start"][b])
    cu = lay["cu_setup"]
    O.append_tokens(cfg, cache, b, start, lay["kv_setup"][cu[b]:cu[b + 1]], lay["logit_setup"][cu[b]:cu[b + 1]])
    O.append_tokens(cfg, cache, b, L - 1, lay["kv_new"][b:b + 1], lay["logit_new"][b:b + 1])
    if ix_host is None or ls.top_k is None:
        O.decode_layer(cfg, cache, b, lay["q"][b], L, ls.top_k)
        return
    ic = O.IndexCache(ix_host["codes"], ix_host["scales"], residue=[[] for _ in range(w.batch)])
    O.index_append_tokens(cfg, ic, lay["comp_table"], b, start, ix_host["k_setup"][cu[b]:cu[b + 1]],
                          lay["logit_setup"][cu[b]:cu[b + 1]])
    O.index_append_tokens(cfg, ic, lay["comp_table"], b, L - 1, ix_host["k_new"][b:b + 1],
                          lay["logit_new"][b:b + 1])
    s = O.mh_indexer_scores(cfg, ic, lay["comp_table"], b, ix_host["q_index"][b], ix_host["weights"][b], L)
    O.attention(cfg, cache, b, lay["q"][b], L, O.topk_select(s, ls.top_k))


def host_inputs(gen):
    out = {"layers": []}
    for lay in gen["layers"]:
        out["layers"].append({k: (v.cpu().numpy().copy() if torch.is_tensor(v) else v)
                              for k, v in lay.items()})
    return out


def index_host(ix):
    return None if ix is None else {k: v.cpu().numpy().copy() for k, v in ix.items()}


def cpu_baseline(w, step, seconds):
    """The oracle on the host cores, on a bounded sample of the workload's requests (the same
    seeded inputs): once limited to one thread, once with every thread numpy's pool has."""
    from threadpoolctl import threadpool_limits
    from oracle import ckv_oracle as O
    gen_host = host_inputs(step.gen)
    ix_host = [index_host(None if mh is None else mh["ix"]) for mh in step.index]

    def leg(budget):
        done = 0
        t0 = time.perf_counter()
        while True:
            for li in range(len(w.layers)):
                oracle_request(w, gen_host, li, done % w.batch, O, ix_host[li])
            done += 1
            if time.perf_counter() - t0 >= budget or done >= 64 * w.batch:
                break
        el = time.perf_counter() - t0
        return done * len(w.layers) / el, done, el

    with threadpool_limits(limits=1):
        v1, n1, t1 = leg(seconds / 2)
    threads = oracle_threads()
    vall, nall, tall = leg(seconds / 2)
    what = (f"requests x {len(w.layers)} layer(s) of {w.name} (same seeded inputs), each a full "
            f"append+select+attend in the fp64 numpy oracle"
            f"{' with the multi-head indexer' if step.indexer == 'mh' else ''}")
    return {"value": vall, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{nall} {what}; {tall:.1f} s on {threads} threads",
            "one_thread": {"value": v1, "unit": UNIT, "cores": 1, "sample": f"{n1} {what}; {t1:.1f} s"},
            "all_threads": {"value": vall, "unit": UNIT, "cores": threads,
                            "sample": f"{nall} {what}; {tall:.1f} s"},
            "nproc": os.cpu_count(), "cpu_model": cpu_model()}


def run_reference(args, w):
    ws, rank, local = dist_env()
    if rank != 0:
        return None
    from oracle import ckv_oracle as O
    gen = S.generate(w, "cpu")
    gen_host = host_inputs(gen)
    ix_host = [index_host(S.generate_index(w, gen, layer=li, heads=MH_HEADS, dim=MH_DIM, device="cpu"))
               if args.indexer == "mh" and ls.top_k is not None else None for li, ls in enumerate(w.layers)]
    per_step = w.batch if args.reference_requests <= 0 else min(w.batch, args.reference_requests)
    b = 0
    for _ in range(args.warmup):
        for li in range(len(w.layers)):
            oracle_request(w, gen_host, li, b % w.batch, O, ix_host[li])
        b += 1
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _r in range(per_step):
            for li in range(len(w.layers)):
                oracle_request(w, gen_host, li, b % w.batch, O, ix_host[li])
            b += 1
    el = time.perf_counter() - t0
    units = args.steps * per_step * len(w.layers)
    value = units / el
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "sample_requests_per_step": per_step, "indexer": args.indexer,
                   "note": "CPU oracle (fp64 numpy) on a bounded sample of the workload's requests"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"{per_step} request(s) x {len(w.layers)} layer(s) per step",
                         "nproc": os.cpu_count(), "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(S.WORKLOADS))
    ap.add_argument("--impl", default="ckv", choices=["ckv", "reference"])
    ap.add_argument("--api", default="fused", choices=["fused", "calls"],
                    help="fused: one ckv_decode_step per layer; calls: append, select, attend")
    ap.add_argument("--indexer", default="avg", choices=["avg", "mh"],
                    help="avg: head-averaged indexer over the K=V entries; mh: multi-head indexer "
                         f"({MH_HEADS} heads x {MH_DIM} dims) over its own FP8 index entries")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="steps launched eagerly, not as CUDA graphs")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure only --workload (by default N = 1 also measures every named config)")
    ap.add_argument("--reference-requests", type=int, default=1,
                    help="requests of the batch the reference arm runs per step (0: all)")
    args = ap.parse_args()
    w = S.WORKLOADS[args.workload]()
    res = run_reference(args, w) if args.impl == "reference" else run_cuda(args, w)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
