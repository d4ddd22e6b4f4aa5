#!/usr/bin/env python
"""Throughput of the approximate-attention prefill layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 128k] [--impl ours|reference]

One step = one pass of the whole path over one layer through the layer entry
point spava_prefill_attention: query-block scores (statistics + scoring
kernels), top-l selection fused with the passing-block gather, and the
approximate attention with the query-row merge, on inputs resident in HBM.
A second timed region runs the same layer as the four separate C-ABI steps
(spava_score -> spava_topk_select -> spava_pack_passing -> spava_attn) with
CUDA events between them, for the per-kernel split and the roofline of the
attention launch.  Prints one JSON line (rank 0).

Multi-GPU (torchrun, N > 1): the one layer is split over the ranks by the
ZigZag sequence parallelism (rank r holds physical hosts r*H/N .. (r+1)*H/N-1,
i.e. chunk pairs p and 2H-1-p), with NCCL all-gathers of the passing blocks
and the query partials -- strong scaling of the layer; the time is the
slowest rank's.  ``--impl reference`` times the fp64 CPU oracle on a bounded sample of
the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sequence_sparse_attention_b200.synth import WORKLOADS, chunk_offsets, make_inputs  # noqa: E402

METRIC = "approx-attn prefill tokens/s per layer on 1 B200; % BF16 tensor peak"
# The spec sheet's dense bf16 tensor figure for one B200 (its 2:4-sparse
# figure halved): context beside the measured peaks.
NOMINAL_BF16_DENSE_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Kernels one spava_prefill_attention call launches: the anchor rows and
# query partials (attention kernel), scoring fused with top-l and gather, the
# context rows (attention kernel), the query merge.
KERNELS_PER_STEP = 4
# The four separate steps: statistics + scores, top-l, gather, attention + merge.
KERNELS_PER_SPLIT_STEP = 6

# DRAM traffic of one attention launch on the 128K layer (dram__bytes_read.sum
# + dram__bytes_write.sum of a single-pass ncu capture); valid only while the
# sources that decide it hash to the value it was taken with (KERNEL_FILES).
PROFILED_TRAFFIC = {"kernel_sha256": "d74482952a1f6e0b8adfcf54662d3e6c85f4b0e170f3983994054cd57cafad9f",
                    "bytes_per_launch": 3090140672 + 1257348096, "workload": "128k"}
KERNEL_FILES = ("attn_kernel.cuh", "plan.cuh", "sm100.cuh")  # what decides the attention launch


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha() -> str:
    h = hashlib.sha256()
    for name in KERNEL_FILES:
        with open(os.path.join(ROOT, "sequence_sparse_attention_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def physical_gpu(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x for x in vis.split(",") if x.strip()]
    if local < len(ids) and ids[local].strip().isdigit():
        return int(ids[local])
    return local


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank value over all ranks (the job is as slow as its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step: int, steps: int, ms_rank: float, world: int) -> tuple:
    """Whole-job tokens/s: the layer's tokens per step, all ranks together (the
    ranks share one layer: strong scaling); the elapsed time is the slowest
    rank's.  Returns (tokens/s, ms per step)."""
    ms = max_over_ranks(ms_rank, world)
    return tokens_per_step * steps / (ms / 1e3), ms / steps


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------- oracle
def oracle_inputs(w, Q=None, K=None, V=None):
    """Host bf16 bit patterns of the layer's inputs (the given tensors, or a
    fresh CPU draw of the same workload)."""
    from sequence_sparse_attention_b200.synth import bf16_bits
    if Q is None:
        Q, K, V, _ = make_inputs(w)
    return bf16_bits(Q), bf16_bits(K), bf16_bits(V)


def oracle_sample(w, budget_s: float, inputs, seed: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload and extrapolate
    to one whole layer.  Returns (tokens/s, description, threads, seconds)."""
    import oracle
    Qb, Kb, Vb = inputs
    off = chunk_offsets(w)
    p = oracle.Problem(H=w.H, Hq=w.Hq, Hkv=w.Hkv, d=w.d, N=w.N, a=w.a, q=w.q, offsets=off,
                       l=w.l, local_pair_full=w.local_pair_full, score_norm=w.score_norm,
                       score_pool=w.score_pool)
    G = w.Hq // w.Hkv
    # (1) scores of chunk 0, KV head 0, and their selection
    t0 = time.perf_counter()
    S = oracle.chunk_scores(p, Qb, Kb, 0, 0)
    t_score = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.select_top_l(S, int(off[0]), w.l)
    t_select = time.perf_counter() - t0
    n0 = int(off[1] - off[0])
    scored_total = sum(int(off[u + 1] - off[u]) for u in range(2 * w.H - 1)) * w.Hkv
    # (2) attention rows of the heads of KV group 0, spread over the sequence
    idx = np.full((2 * w.H - 1, w.Hkv, w.l), -1, dtype=np.int32)
    for u in range(2 * w.H - 1):
        k = min(w.l, int(off[u + 1] - off[u]))
        idx[u, :, :k] = off[u] + np.arange(k)       # any valid selection costs the same
    rng = np.random.default_rng(seed)
    rows_all = rng.permutation(w.N)
    heads = list(range(G))
    done_rows, pairs, t_attn = 0, 0, 0.0
    remaining = max(1.0, budget_s - t_score - t_select)
    batch = 8
    while t_attn < remaining and done_rows < len(rows_all):
        rows = rows_all[done_rows:done_rows + batch]
        t0 = time.perf_counter()
        oracle.prefill_rows(p, Qb, Kb, Vb, idx, rows, heads)
        t_attn += time.perf_counter() - t0
        pairs += sum(len(oracle.key_set(p, idx, int(t), 0)) for t in rows) * G
        done_rows += len(rows)
        batch = min(64, batch * 2)
    total_pairs = sum(oracle.attended_pairs(p)) * w.Hq
    t_layer = (t_score * scored_total / n0 + t_select * (2 * w.H - 1) * w.Hkv
               + t_attn * total_pairs / pairs)
    desc = (f"scores of chunk 0 for KV head 0 ({n0} keys x {G * w.q} query rows) and its top-l; "
            f"attention of {done_rows} random rows x {G} heads ({pairs} pairs); extrapolated to the "
            f"layer by scored keys and attended pairs; {t_score + t_select + t_attn:.1f} s of CPU")
    return w.N / t_layer, desc, oracle.num_threads(), t_score + t_select + t_attn


def selected_workload(args):
    """The named layer, with the selection variant asked for (default: none)."""
    return dataclasses.replace(WORKLOADS[args.workload], score_norm=args.score_norm,
                               score_pool=args.score_pool)


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = selected_workload(args)
    values, cores, desc, spent = [], None, None, 0.0
    per_step = max(3.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    inputs = oracle_inputs(w)
    for s in range(args.warmup + args.steps):
        v, desc, cores, sp = oracle_sample(w, per_step, inputs, seed=s)
        spent += sp
        if s >= args.warmup:
            values.append(v)
    value = statistics.median(values)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.N / value, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def parallelism(world: int) -> str:
    return ("one GPU, all 2H ZigZag virtual hosts on it" if world == 1 else
            f"ZigZag sequence parallelism over {world} GPUs (H/{world} physical hosts each; "
            "NCCL all-gathers of passing blocks and query partials)")


def workload_config(w, world=1):
    return {"parallelism": parallelism(world),"workload": f"{w.name}: H={w.H} ({2 * w.H} ZigZag virtual hosts), {w.Hq} q / {w.Hkv} kv heads, "
                        f"d={w.d}, {w.N} tokens (anchor {w.a}, query block {w.q}), top-l={w.l}",
            "tokens": w.N, "H": w.H, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
            "anchor": w.a, "query_block": w.q, "top_l": w.l,
            "local_pair_full": w.local_pair_full, "score_norm": w.score_norm,
            "score_pool": w.score_pool,
            "inputs": "seeded synthetic video-shaped bf16 (frame-correlated keys"
                      + (", 5% heavy-hitter keys" if w.heavy_frac else "")
                      + (", +/-10% uneven chunks" if w.jitter else "") + ")",
            "l2": "no flush: inputs (Q+K+V) exceed the 126 MB L2"}


# ----------------------------------------------------------------------- ours
def run_ours(args, world, rank, local):
    from sequence_sparse_attention_b200.api import Layout, Spava, attended_pairs
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = selected_workload(args)
    Q, K, V, off = make_inputs(w, device)
    lay = Layout.from_workload(w)
    sp = Spava(lay, device)
    scores = torch.zeros((w.Hkv, lay.context), dtype=torch.float32, device=device)
    idx = torch.empty((2 * w.H - 1, w.Hkv, w.l), dtype=torch.int32, device=device)
    pk = torch.empty((w.Hkv, sp.L, w.d), dtype=torch.bfloat16, device=device)
    pv = torch.empty_like(pk)
    O = torch.empty_like(Q)
    lse = torch.empty((w.Hq, w.N), dtype=torch.float32, device=device)

    def layer():
        """One step: the layer entry point (what a user calls)."""
        sp.prefill_attention(Q, K, V, O, lse)

    def split_step(ev):
        """The same layer as the four separate C-ABI steps, events between."""
        ev[0].record()
        sp.score(Q, K, scores)
        ev[1].record()
        sp.topk_select(scores, idx)
        ev[2].record()
        sp.pack_passing(K, V, idx, pk, pv)
        ev[3].record()
        sp.attn(Q, K, V, pk, pv, O, lse)
        ev[4].record()

    for _ in range(args.warmup):
        layer()
    torch.cuda.synchronize()
    status = sp.device_status()
    if status:
        raise RuntimeError(f"kernel status {status} during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(physical_gpu(local))
    with sampler:
        time.sleep(0.3)
        # (A) the headline: K calls of the layer entry point
        barrier(world)
        torch.cuda.synchronize()
        start.record()
        for _ in range(args.steps):
            layer()
        end.record()
        torch.cuda.synchronize()
        barrier(world)
        # (B) the per-kernel split, same layer, same inputs
        for _ in range(2):
            split_step([torch.cuda.Event(enable_timing=True) for _ in range(5)])
        torch.cuda.synchronize()
        barrier(world)
        for s_ in range(args.steps):
            split_step(evs[s_])
        torch.cuda.synchronize()
        barrier(world)
    clocks = sampler.summary()
    if sp.device_status():
        raise RuntimeError("kernel status set during the timed region")
    tokens_per_s, ms_step = job_throughput(w.N, args.steps, start.elapsed_time(end), world)
    names = ["score", "topk", "pack", "attn"]
    per = {n: statistics.mean(evs[s_][i].elapsed_time(evs[s_][i + 1]) for s_ in range(args.steps))
           for i, n in enumerate(names)}
    split_ms = sum(per.values())

    # ---- roofline of the dominant kernel (approximate attention)
    pk_, pe = peaks()
    pairs = sum(attended_pairs(lay)[0])
    flops = 4.0 * w.d * w.Hq * pairs
    achieved = flops / (per["attn"] / 1e3) / 1e12
    # Primary denominator: the burst bf16 GEMM figure.  This kernel runs at
    # ~1.7 GHz under the power cap, close to the burst GEMM's clock; the
    # sustained GEMM figure was taken at ~1.33 GHz and would flatter it.
    peak = pk_.get("bf16_tflops")
    sustained = pk_.get("bf16_tflops_sustained") or peak
    traffic = None
    if PROFILED_TRAFFIC["kernel_sha256"] == kernel_sha() and PROFILED_TRAFFIC["workload"] == w.name:
        traffic = PROFILED_TRAFFIC["bytes_per_launch"]
    sm_mhz = clocks.get("sm_mhz")
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    # tensor-pipe issue rate of dense bf16 MMA: 8192 FLOP per SM per clock
    pipe_at_clock = n_sm * 8192 * sm_mhz * 1e6 / 1e12 if sm_mhz else None
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": "attn_kernel<128> + query merge (spava_attn)",
                "peak_kind": f"{pe} bf16 dense GEMM, burst",
                "frac_of_sustained_peak": achieved / sustained,
                "frac_of_nominal_dense_peak": achieved / NOMINAL_BF16_DENSE_TFLOPS,
                "tflops_per_ghz": achieved / (sm_mhz / 1e3) if sm_mhz else None,
                "frac_of_tensor_pipe_at_sampled_clock": achieved / pipe_at_clock if pipe_at_clock else None,
                "launch_ms": per["attn"],
                "algorithmic_flops_per_launch": flops, "attended_pairs_per_head": pairs}

    # ---- the selection phase against HBM (each operand touched once)
    hbm = pk_.get("hbm_gbs")
    n_sel = sum(min(w.l, int(off[u + 1] - off[u])) for u in range(2 * w.H - 1))
    packed_rows = w.Hkv * (w.a + n_sel)
    scored = int(off[2 * w.H - 1]) - w.a    # keys of the producing chunks
    sel_bytes = {
        # K of the scored chunks read twice (statistics, scores), the query
        # block's Q rows, the scores written
        "score": 2 * scored * w.Hkv * w.d * 2 + w.q * w.Hq * w.d * 2 + 4 * w.Hkv * scored,
        # scores read, indices written
        "topk": 4 * w.Hkv * scored + 4 * (2 * w.H - 1) * w.Hkv * w.l,
        # K and V rows read and written
        "pack": 2 * 2 * packed_rows * w.d * 2,
    }
    selection = {k: {"bytes": b, "GB/s": b / (per[k] / 1e3) / 1e9,
                     "frac_of_hbm": b / (per[k] / 1e3) / 1e9 / hbm}
                 for k, b in sel_bytes.items()}
    phase_bytes = sum(sel_bytes.values())
    phase_ms = per["score"] + per["topk"] + per["pack"]
    # Scoring is a contraction with one exponential per (query row, head, key),
    # done twice (the statistics pass, then the scores): its TFLOP/s and
    # exponentials per second, the latter against the MUFU rate at the sampled
    # clock (16 per SM per clock; a quarter of the scoring pass's exponentials
    # run on the FMA pipe instead, so the fraction can pass 1).
    triples = w.Hq * w.q * scored
    score_s = per["score"] / 1e3
    selection["score"]["TFLOP/s"] = 2 * 2 * w.d * triples / score_s / 1e12
    selection["score"]["exp/s"] = 2 * triples / score_s
    selection["score"]["frac_of_mufu_at_sampled_clock"] = (
        2 * triples / score_s / (n_sm * 16 * sm_mhz * 1e6) if sm_mhz else None)
    selection["phase"] = {"bytes": phase_bytes, "ms": phase_ms,
                          "GB/s": phase_bytes / (phase_ms / 1e3) / 1e9,
                          "frac_of_hbm": phase_bytes / (phase_ms / 1e3) / 1e9 / hbm}
    selection["peak_GBps"] = hbm
    selection["note"] = ("pack (the gather) is the HBM-bound step; scoring is tensor/exp-bound "
                         "(one exponential per 4*d flops) and top-l latency-bound, so their GB/s "
                         "fractions are reported, not targeted")

    # ---- end to end through the host-buffer entry point
    qh = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)
    kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
    vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
    qh.copy_(Q)
    kh.copy_(K)
    vh.copy_(V)
    oh = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 5))
    copy_stream = torch.cuda.Stream()

    def time_host_calls(cs):
        sp.prefill_attention_host(qh, kh, vh, oh, None, Q, K, V, O, None, copy_stream=cs)  # warm
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e2e_steps):
            sp.prefill_attention_host(qh, kh, vh, oh, None, Q, K, V, O, None, copy_stream=cs)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps

    e2e_ms = time_host_calls(copy_stream)       # copies overlapped with the kernels
    serial_ms = time_host_calls(None)           # everything on one stream
    h2d = (Q.numel() + K.numel() + V.numel()) * 2
    d2h = O.numel() * 2
    e2e = {"value": world * w.N / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "api": "spava_prefill_attention_host (pinned host buffers in/out, copy stream "
                  "overlapping the copies with the kernels)",
           "one_stream_ms_per_step": serial_ms}

    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(w, world),
        "roofline": roofline,
        "selection_hbm": selection,
        "kernel_ms": per,
        "split_ms_per_step": split_ms,
        "tensor_peak_frac": {"of_burst": achieved / peak, "of_sustained": achieved / sustained,
                             "of_nominal_2250": achieved / 2250.0},
        "e2e": e2e, "gpu_launches": KERNELS_PER_STEP * args.steps,
        "gpu_launches_split_region": KERNELS_PER_SPLIT_STEP * args.steps, "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores, _ = oracle_sample(w, args.cpu_budget, oracle_inputs(w, Q, K, V))
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_sharded(args, world, rank, local):
    """N > 1: the one layer split over the ranks (ZigZag sequence parallelism).
    Each rank holds [anchor | its chunks | query block]; the passing blocks and
    the query partials are NCCL all-gathers on a second stream, overlapped with
    the rank's local attention.  ``--shard-on-one`` runs this path as world 1
    (the gathers are copies) to check it on a single GPU."""
    from sequence_sparse_attention_b200.api import Layout, SpavaShard, attended_pairs
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = selected_workload(args)
    lay = Layout.from_workload(w)
    sh = SpavaShard(lay, rank, world, device)
    Q, K, V, off = make_inputs(w, device)
    pos = torch.from_numpy(sh.positions).to(device)
    q, k, v = Q[pos].contiguous(), K[pos].contiguous(), V[pos].contiguous()
    del Q, K, V
    torch.cuda.empty_cache()
    o, lse = sh.new_outputs()
    if world > 1:
        import torch.distributed as dist

        def all_gather(out, inp):
            dist.all_gather_into_tensor(out, inp)
    else:
        def all_gather(out, inp):
            out.copy_(inp)
    cs = torch.cuda.Stream(device)

    def layer():
        sh.layer(q, k, v, o, lse, all_gather, comm_stream=cs)

    for _ in range(args.warmup):
        layer()
    torch.cuda.synchronize()
    if int(sh.ws[:4].view(torch.int32).item()):
        raise RuntimeError("kernel status set during warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_ev = 5
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu(local))
    with sampler:
        time.sleep(0.3)
        barrier(world)
        torch.cuda.synchronize()
        start.record()
        for _ in range(args.steps):
            layer()
        end.record()
        torch.cuda.synchronize()
        barrier(world)
        # per-call split on the compute stream, the gathers done in place
        for s_ in range(args.steps):
            ev = evs[s_]
            ev[0].record()
            sh.front(q, k, v)
            ev[1].record()
            sh.local_attn(q, k, v, o, lse)
            all_gather(sh.pass_all, sh.pass_send)
            all_gather(sh.part_all, sh.part_send)
            ev[2].record()
            sh.context_attn(q, k, v, o, lse)
            ev[3].record()
            sh.merge(o, lse)
            ev[4].record()
        torch.cuda.synchronize()
        barrier(world)
    clocks = sampler.summary()
    if int(sh.ws[:4].view(torch.int32).item()):
        raise RuntimeError("kernel status set during the timed region")
    tokens_per_s, ms_step = job_throughput(w.N, args.steps, start.elapsed_time(end), world)
    names = ["front", "local_attn_and_gathers", "context_attn", "merge"]
    per = {n: statistics.mean(evs[s_][i].elapsed_time(evs[s_][i + 1]) for s_ in range(args.steps))
           for i, n in enumerate(names)}

    # roofline: the context-row attention launch of this rank
    pk_, pe = peaks()
    _, per_host = attended_pairs(lay)
    m = w.H // world
    ctx_pairs = sum(per_host[rank * m:(rank + 1) * m])
    flops = 4.0 * w.d * w.Hq * ctx_pairs
    achieved = flops / (per["context_attn"] / 1e3) / 1e12
    peak = pk_.get("bf16_tflops")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None,
                "kernel": "attn_kernel<128>, context rows of this rank's chunks (spava_shard_context_attn)",
                "peak_kind": f"{pe} bf16 dense GEMM, burst", "rank": rank,
                "algorithmic_flops_per_launch": flops}

    # end to end: pinned host buffers of this rank's rows in, its O rows out
    qh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    kh = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    vh = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    qh.copy_(q)
    kh.copy_(k)
    vh.copy_(v)
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        q.copy_(qh, non_blocking=True)
        k.copy_(kh, non_blocking=True)
        v.copy_(vh, non_blocking=True)
        layer()
        oh.copy_(o, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    e2e = {"value": w.N / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * 2,
           "d2h_bytes_per_step": o.numel() * 2, "ms_per_step": e2e_ms,
           "api": "SpavaShard.layer per rank: pinned host copies of the rank's rows in, its O rows out"}
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(w, world),
        "roofline": roofline, "kernel_ms_rank": per, "e2e": e2e,
        "gpu_launches": args.steps * 10, "clocks": clocks,
        "messages_bytes": {"pass_per_rank": sh.pass_send.numel(), "part_per_rank": sh.part_send.numel()},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="128k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--score-norm", type=int, default=0, choices=[0, 1],
                    help="selection variant: 1 = row-normalised scores")
    ap.add_argument("--score-pool", type=int, default=0,
                    help="selection variant: odd window w >= 3 = pooled ranking")
    ap.add_argument("--shard-on-one", action="store_true",
                    help="run the sharded (multi-GPU) path as one rank")
    args = ap.parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if world > 1 or args.shard_on_one:
            run_sharded(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
