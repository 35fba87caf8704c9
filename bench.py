"""Throughput of the ISD step on B200: committed tokens/s and roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload qwen3_8b_b64|qwen3_8b_b1|tiny]

One step = one isd_step over the whole batch: assemble the block, 36
decoder layers (QKV / attention / O / MLP), LM head, verify-resample-
propose and page bookkeeping, all in libisd.so's kernels. Weights are
random-init (bf16 N(0, 0.02)) of the named shape, prompts uniform random
tokens with seeded lengths, physical pages randomly permuted, KV filled by
isd_prefill before timing. Accept-test uniforms are acceptance-controlled
(each draft passes with probability 0.9, the pages' operating point) so the
committed tokens per forward match a trained model's regime; the run with
natural uniforms is reported beside it.

The K timed steps are captured once into a CUDA graph (before timing) and
replayed once inside the timed region; the same number of steps launched
one by one is reported as "eager" (--no-graph times those instead).

Multi-GPU (torchrun): the method shards by request, so every rank runs an
independent replica with its own batch (weak scaling, no collective in the
step); time is the max over ranks, value the sum of all ranks' tokens.

--impl reference times the CPU oracle (fp64 numpy) on a bounded sample of
the same workload on rank 0 and extrapolates to the same metric.

--component gemm:MxNxKxS | gemm1:MxNxK | attention:WORKLOAD times one kernel
of the step through its C-ABI component entry (isd_gemm_bf16: Y = X W^T with
M tokens, N outputs, K inputs, S K-splits; isd_gemm_bf16_single: the same as
one slice, stream-K when the tiles overfill a wave; isd_paged_attention on
the workload's block rows and KV lengths), one launch per step with an L2 flush between,
and prints its duration and throughput. It is the command the kernel
profiles are taken with.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOADS = {
    # Qwen3-8B shape, batch 64, stride 4, prompt lengths U[512, 4096]
    "qwen3_8b_b64": dict(shape=synth.QWEN3_8B, batch=64, stride=4, len_lo=512, len_hi=4096),
    # Qwen3-8B shape, batch 1, stride 4, prompt 2048
    "qwen3_8b_b1": dict(shape=synth.QWEN3_8B, batch=1, stride=4, len_lo=2048, len_hi=2048),
    "tiny": dict(shape=synth.TINY, batch=1, stride=2, len_lo=32, len_hi=32),
    # the headline configuration with sampled proposals (full q rows kept per request)
    "qwen3_8b_b64_sample": dict(shape=synth.QWEN3_8B, batch=64, stride=4, len_lo=512, len_hi=4096,
                                sample=True),
    # R-ISD: Qwen3-8B shape + rank-128 gated LoRA on MASK rows, batch 32, N=4, prompts 2048
    "risd_8b_b32": dict(shape=synth.QWEN3_8B, batch=32, stride=4, len_lo=2048, len_hi=2048,
                        lora_rank=128),
    # the headline configuration cut to two layers (same batch, prompts, pages): the
    # per-layer kernels at the headline shapes in a few GB, for ncu captures
    "qwen3_8b_b64_l2": dict(shape=synth.QWEN3_8B_2L, batch=64, stride=4, len_lo=512, len_hi=4096),
    # Qwen3-32B shape (64 layers, hidden 5120, 64/8 heads), batch 64, N=4, prompts U[1024, 8192]
    "qwen3_32b_b64": dict(shape=synth.QWEN3_32B, batch=64, stride=4, len_lo=1024, len_hi=8192),
}
ACCEPT_RATE = 0.9
MODEL_NAMES = {synth.QWEN3_8B: "qwen3-8b-shape (random init)",
               synth.QWEN3_8B_2L: "qwen3-8b-shape, 2 layers (random init)",
               synth.QWEN3_32B: "qwen3-32b-shape (random init)"}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), for the CPU baseline."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


FALLBACK_PEAKS = dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0)
NOMINAL_HBM_GBS = 8000.0      # B200 HBM3e nominal, beside the measured copy peak


def load_peaks(path=None):
    """Roofline denominators: the measured copy bandwidth (GB/s) and bf16
    GEMM rates (TFLOP/s, burst and sustained) from MEASURED_PEAKS.json when
    it is there, each figure that is missing or not a plain positive number
    taken from the fallback; `source` says which."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    keys = dict(hbm="hbm_gbs", bf16="bf16_tflops", bf16_sus="bf16_tflops_sustained")
    try:
        with open(path) as f:
            p = json.load(f)
    except (OSError, ValueError):
        p = None
    if not isinstance(p, dict):
        return dict(FALLBACK_PEAKS, source="fallback")
    out, used = {}, []
    for k, name in keys.items():
        v = p.get(name)
        if isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0:
            out[k] = float(v)
            used.append(k)
        else:
            out[k] = FALLBACK_PEAKS[k]
    out["source"] = ("measured" if len(used) == len(keys) else
                     "fallback" if not used else "measured " + ", ".join(used) + "; fallback for the rest")
    return out


class ClockSampler:
    """nvidia-smi samples (200 ms) while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def reduce_over_ranks(times_ms, tokens, ws, device):
    """Whole-job figures from every rank's own: each time is the max over the
    ranks (the job ends with its slowest replica), each token count the sum.
    Every rank calls it with the same number of values."""
    import torch
    vals = torch.tensor(list(times_ms), device=device, dtype=torch.float64)
    toks = torch.tensor(list(tokens), device=device, dtype=torch.float64)
    if ws > 1:
        import torch.distributed as dist
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(toks, op=dist.ReduceOp.SUM)
    return vals.tolist(), toks.tolist()


def setup_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------ algorithmic ---

def step_w_params(shape):
    """Weights a step streams: every layer's projections and the LM head."""
    return shape.n_layers * shape.params_per_layer() + shape.vocab * shape.hidden


def step_bytes_flops(shape, lens_now, B, N):
    """Algorithmic bytes / flops of one step (weights once, KV once, logits once)."""
    R = 2 * N - 1
    w_params = step_w_params(shape)
    kv = sum(int(L) + R for L in lens_now) * shape.kv_bytes_per_token()
    logits = B * R * shape.vocab * 4
    flops = 2.0 * B * R * w_params
    return 2 * w_params, kv, logits, flops


# ---------------------------------------------------------------- CUDA arm ---

def metric_name(workload: str) -> str:
    """The JSON line's `metric` (both arms print the same one)."""
    if workload == "qwen3_8b_b64":
        return "committed tokens/s (ISD step, Qwen3-8B shape, batch 64, N=4)"
    return f"committed tokens/s ({workload})"


def workload_config(workload: str, ws: int) -> dict:
    """The JSON line's `config` (both arms print the same one): the workload
    with its sizes, and how it spreads over ws ranks."""
    wl = WORKLOADS[workload]
    shape, B, N = wl["shape"], wl["batch"], wl["stride"]
    wbytes = 2 * step_w_params(shape)
    return {"workload": workload, "shape": MODEL_NAMES.get(shape, "tiny"), "batch_per_gpu": B,
            "global_batch": B * ws, "stride_n": N, "rows_per_step": B * (2 * N - 1),
            "prompt_len": [wl["len_lo"], wl["len_hi"]], "page_size": shape.page_size,
            "parallelism": f"replicas x{ws} (request-sharded, no collective)",
            "uniforms": f"acceptance-controlled a={ACCEPT_RATE}",
            "l2": (f"inputs larger than L2 (weights {wbytes / 1e9:.0f} GB + KV > 126 MB)"
                   if wbytes > 126e6 else
                   f"inputs smaller than L2 (weights {wbytes / 1e6:.1f} MB): a test workload")}


def run_cuda(args, ws, rank, local):
    import torch
    import torch.distributed as dist
    from strided_verify_propose_b200 import binding as Bd

    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    wl = WORKLOADS[args.workload]
    shape, B, N = wl["shape"], wl["batch"], wl["stride"]
    R, P, V = 2 * N - 1, shape.page_size, shape.vocab
    seed = 1000 + rank
    total_steps = args.warmup + 6 * args.steps + 4   # every step run below grows the sequences
    lens = synth.prompt_lengths(B, wl["len_lo"], wl["len_hi"], seed)
    prompts = synth.prompts(shape, lens, seed)
    maxp = -(-(int(lens.max()) + total_steps * N + R + 1) // P) + 1
    need = [-(-(int(L) - 1 + R) // P) for L in lens]
    num_pages = int(sum(need)) + B * (-(-total_steps * N // P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, seed)

    t0 = time.time()
    weights = Bd.random_device_weights(shape, seed=seed)
    G = shape.n_q_heads // shape.n_kv_heads
    # 64 rows per request per prefill pass (several attention query tiles)
    model = Bd.Model(shape, weights, max_batch=B, max_rows=max(B * R, B * 64),
                     max_position=maxp * P)
    lora_rank = wl.get("lora_rank", 0)
    flags = 0
    if lora_rank:
        model.load_lora(Bd.random_device_lora(shape, lora_rank, seed=seed, std=0.01), rank=lora_rank)
        flags = Bd.USE_LORA
    kv = Bd.KVCache(shape, num_pages, table, free)
    if wl.get("sample"):
        flags |= Bd.PROPOSE_SAMPLE
    st = Bd.StepState(B, N, V, sample=bool(wl.get("sample")))
    torch.cuda.synchronize()
    t_setup = time.time() - t0
    t0 = time.time()
    Bd.prefill(model, kv, st, prompts)
    torch.cuda.synchronize()
    t_prefill = time.time() - t0
    if int(st.status.item()) != 0:
        raise RuntimeError(f"prefill status {int(st.status.item())}")

    unif = np.stack([synth.controlled_uniforms(B, N, ACCEPT_RATE, seed, s) for s in range(total_steps)])
    unif_nat = np.stack([synth.uniforms(B, R, seed + 77, s) for s in range(args.steps)])
    unif_d = torch.from_numpy(unif).cuda()
    unif_nat_d = torch.from_numpy(unif_nat).cuda()
    hist = torch.zeros(args.steps, B, device="cuda", dtype=torch.int32)
    step_i = 0

    def one(u, fl=None):
        Bd.step(model, kv, st, u, flags if fl is None else fl)

    for _ in range(args.warmup):
        one(unif_d[step_i]); step_i += 1
    torch.cuda.synchronize()
    lens_before = st.seq_len.cpu().numpy().copy()

    def barrier():
        if ws > 1:
            dist.barrier()

    # ---- timed region: K steps, inputs resident in HBM. By default the K
    # steps are one CUDA graph (captured here, before timing) replayed once;
    # the same K steps launched one by one are timed next as "eager".
    stream = torch.cuda.current_stream()
    graph = None
    if not args.no_graph:
        graph = Bd.StepGraph(model, kv, st, args.steps, flags)
        torch.cuda.synchronize()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("isd_timed")
        if graph is not None:
            u_g = unif_d[step_i:step_i + args.steps].clone()
            step_i += args.steps
            e_start.record(stream)
            graph.replay(u_g)
            e_stop.record(stream)
        else:
            e_start.record(stream)
            for i in range(args.steps):
                one(unif_d[step_i]); step_i += 1
                hist[i].copy_(st.accepted)
            e_stop.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    barrier()
    ms = e_start.elapsed_time(e_stop)
    if graph is not None:
        hist.copy_(graph.accepted)
        del graph
    launches_per_step = model.launches()
    committed = int((hist.long() + 1).sum().item())
    if int(st.status.item()) != 0:
        raise RuntimeError(f"step status {int(st.status.item())}")

    # ---- the same number of steps launched one by one
    eager_ms, eager_committed, step_ms = None, 0, None
    if not args.no_graph:
        # an event between consecutive steps: the per-step spread
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        h_start, h_stop = marks[0], marks[-1]
        eager_hist = torch.zeros(args.steps, B, device="cuda", dtype=torch.int32)
        torch.cuda.synchronize()
        h_start.record(stream)
        for i in range(args.steps):
            one(unif_d[step_i]); step_i += 1
            eager_hist[i].copy_(st.accepted)
            marks[i + 1].record(stream)
        torch.cuda.synchronize()
        eager_ms = h_start.elapsed_time(h_stop)
        step_ms = np.array([marks[i].elapsed_time(marks[i + 1]) for i in range(args.steps)])
        eager_committed = int((eager_hist.long() + 1).sum().item())

    lens_after_timed = st.seq_len.cpu().numpy().copy()   # (after the eager steps too)

    # ---- profiled region: same steps with per-kernel-class CUDA events; the
    # lengths each profiled step starts from price its attention bytes
    lens_prof = torch.zeros(args.steps, B, device="cuda", dtype=torch.int32)
    model.profile(True)
    for i in range(args.steps):
        lens_prof[i].copy_(st.seq_len)
        one(unif_d[step_i]); step_i += 1
    prof = model.profile_read()
    model.profile(False)
    lens_prof = lens_prof.cpu().numpy()

    # ---- the same steps without the adapter: R-ISD overhead alpha
    base_ms = None
    if lora_rank:
        torch.cuda.synchronize()
        b_start, b_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b_start.record(stream)
        for i in range(args.steps):
            one(unif_d[step_i % total_steps], 0); step_i += 1
        b_stop.record(stream)
        torch.cuda.synchronize()
        base_ms = b_start.elapsed_time(b_stop)

    # ---- natural uniforms (acceptance ~ 0 with random weights)
    torch.cuda.synchronize()
    n_start, n_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nat_hist = torch.zeros(args.steps, B, device="cuda", dtype=torch.int32)
    n_start.record(stream)
    for i in range(args.steps):
        one(unif_nat_d[i])
        nat_hist[i].copy_(st.accepted)
    n_stop.record(stream)
    torch.cuda.synchronize()
    nat_ms = n_start.elapsed_time(n_stop)
    nat_committed = int((nat_hist.long() + 1).sum().item())

    # ---- end to end through the C ABI with host buffers
    pin_u = torch.from_numpy(unif[step_i:step_i + args.steps].copy()).pin_memory()
    pin_acc = torch.zeros(args.steps, B, dtype=torch.int32).pin_memory()
    pin_com = torch.zeros(args.steps, B, N, dtype=torch.int32).pin_memory()
    u_dev = torch.empty(B, R, device="cuda", dtype=torch.float32)
    torch.cuda.synchronize()
    barrier()
    x_start, x_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x_start.record(stream)
    for i in range(args.steps):
        u_dev.copy_(pin_u[i], non_blocking=True)
        one(u_dev)
        pin_acc[i].copy_(st.accepted, non_blocking=True)
        pin_com[i].copy_(st.committed, non_blocking=True)
        stream.synchronize()            # the host reads this step's committed tokens
    x_stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = x_start.elapsed_time(x_stop)
    e2e_committed = int((pin_acc.long() + 1).sum().item())

    # ---- the other single-GPU configurations of the same model (one GPU only)
    extras = None
    if ws == 1 and not args.no_extras and shape is synth.QWEN3_8B and not lora_rank \
            and not wl.get("sample"):
        extras = extra_configs(model, shape, args, seed)

    # ---- reduce over ranks: max time, summed tokens
    (ms, e2e_ms, nat_ms, eager_ms_all), (committed, e2e_committed, nat_committed, eager_committed) = \
        reduce_over_ranks([ms, e2e_ms, nat_ms, eager_ms or 0.0],
                          [committed, e2e_committed, nat_committed, eager_committed], ws, "cuda")

    result = None
    if rank == 0:
        peaks = load_peaks()
        ms_step = ms / args.steps
        # the timed steps start from lens_before and grow by about a step's
        # commit each: price them at the mean length of the timed region
        lens_timed = lens_before + (lens_after_timed - lens_before) * (
            0.5 * args.steps / (2 * args.steps if eager_ms is not None else args.steps))
        wbytes, kvbytes, lbytes, flops = step_bytes_flops(shape, lens_timed, B, N)
        step_bytes = wbytes + kvbytes
        hbm_frac_step = (step_bytes / (ms_step * 1e-3)) / (peaks["hbm"] * 1e9)
        # ceiling: GEMMs at the tensor peak plus attention KV at HBM peak
        t_floor = flops / (peaks["bf16"] * 1e12) + kvbytes / (peaks["hbm"] * 1e9)
        ceiling = (step_bytes / (peaks["hbm"] * 1e9)) / t_floor
        roof = roofline_entry(prof, shape, B, N, lens_prof, args.steps, peaks)
        result = {
            "metric": metric_name(args.workload),
            "value": committed / (ms * 1e-3),
            "unit": "tokens/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (random-init weights, uniform random prompts, seeded)",
            "config": workload_config(args.workload, ws),
            "tokens_per_forward": committed / (args.steps * B * ws),
            "hbm_roofline_fraction_step": hbm_frac_step,
            "hbm_fraction_step_of_nominal": (step_bytes / (ms_step * 1e-3)) / (NOMINAL_HBM_GBS * 1e9),
            "hbm_roofline_ceiling_step": ceiling,
            "step_algorithmic_bytes": step_bytes,
            "risd_overhead_alpha": (ms / base_ms) if base_ms else None,
            "natural_uniforms": {"value": nat_committed / (nat_ms * 1e-3), "unit": "tokens/s",
                                 "tokens_per_forward": nat_committed / (args.steps * B * ws)},
            "timed_as": "one CUDA graph of the K steps, replayed once" if eager_ms is not None
            else "K steps launched one by one",
            "eager": None if eager_ms is None else {
                "value": eager_committed / (eager_ms_all * 1e-3), "unit": "tokens/s",
                "ms_per_step": eager_ms_all / args.steps,
                "step_ms_p10_median_p90": [round(float(np.percentile(step_ms, q)), 4)
                                           for q in (10, 50, 90)],
                "note": "the same number of steps launched one by one (per-step spread on rank 0)"},
            "prefill_s": t_prefill, "setup_s": t_setup,
            "gpu_launches": launches_per_step * args.steps,
            "launches_per_step": launches_per_step,
            "roofline": roof,
            "kernel_ms_per_step": {k: v[0] / args.steps for k, v in sorted(prof.items())},
            "clocks": clk.summary(),
            "e2e": {"value": e2e_committed / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": B * R * 4, "d2h_bytes_per_step": B * 4 + B * N * 4},
            "peaks": peaks,
        }
        if extras is not None:
            ex = dict(extras)
            for key in ("qwen3_8b_b1", "qwen3_8b_b64_sample"):
                e = ex[key]
                e["hbm_roofline_fraction"] = e["step_bytes"] / (e["ms_per_step"] * 1e-3) / (
                    peaks["hbm"] * 1e9)
            result["other_configs"] = ex
            result["risd_overhead_alpha"] = ex["risd_8b_b32"]["alpha"]
    del model
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def extra_configs(model, shape, args, seed):
    """The model's other single-GPU configurations, on the same weights:
    batch 1 with a 2048-token prompt; the headline batch (64, prompts
    U[512, 4096]) with sampled proposals and full q rows; and R-ISD (a
    rank-128 gated LoRA, A, B ~ N(0, 0.01), on the MASK rows) at batch 32
    with 2048-token prompts, timed against the same steps without the
    adapter. Each runs args.warmup eager steps, then args.steps steps
    between CUDA events (acceptance-controlled uniforms, inputs resident)."""
    import torch
    from strided_verify_propose_b200 import binding as Bd
    N = 4
    R, P, V = 2 * N - 1, shape.page_size, shape.vocab
    stream = torch.cuda.current_stream()
    out = {}

    def make(B, plen, s0, sample=False, lens=None):
        lens = np.full(B, plen, np.int64) if lens is None else lens
        prompts = synth.prompts(shape, lens, s0)
        steps = args.warmup + 3 * args.steps + 2
        maxp = -(-(int(lens.max()) + steps * N + R + 1) // P) + 1
        need = [-(-(int(L) - 1 + R) // P) for L in lens]
        num_pages = int(sum(need)) + B * (-(-steps * N // P) + 2)
        table, free = synth.page_layout(need, num_pages, maxp, s0)
        kv = Bd.KVCache(shape, num_pages, table, free)
        st = Bd.StepState(B, N, V, sample=sample)
        Bd.prefill(model, kv, st, prompts)
        torch.cuda.synchronize()
        if int(st.status.item()) != 0:
            raise RuntimeError("prefill status")
        return kv, st

    def timed(kv, st, B, flags, s0, first):
        for i in range(args.warmup):
            Bd.step(model, kv, st, torch.from_numpy(
                synth.controlled_uniforms(B, N, ACCEPT_RATE, s0, first + i)).cuda(), flags)
        u = torch.from_numpy(np.stack([synth.controlled_uniforms(B, N, ACCEPT_RATE, s0, first + 100 + i)
                                       for i in range(args.steps)])).cuda()
        acc = torch.zeros(args.steps, B, device="cuda", dtype=torch.int32)
        lens0 = st.seq_len.cpu().numpy().copy()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            Bd.step(model, kv, st, u[i], flags)
            acc[i].copy_(st.accepted)
        e1.record(stream)
        torch.cuda.synchronize()
        if int(st.status.item()) != 0:
            raise RuntimeError("step status")
        return e0.elapsed_time(e1), int((acc.long() + 1).sum().item()), lens0

    # batch 1, prompt 2048: every projection streams its weights for 7 rows
    kv, st = make(1, 2048, seed + 11)
    ms1, com1, lens1 = timed(kv, st, 1, 0, seed + 11, 0)
    w, kvb, _, _ = step_bytes_flops(shape, lens1, 1, N)
    out["qwen3_8b_b1"] = {"ms_per_step": ms1 / args.steps, "value": com1 / (ms1 * 1e-3),
                          "unit": "tokens/s", "step_bytes": w + kvb, "steps": args.steps}
    del kv, st
    # the headline batch with sampled proposals: every step writes the next
    # drafts' full q rows and the accept tests read them
    lens64 = synth.prompt_lengths(64, 512, 4096, seed)     # the headline workload's lengths
    kv, st = make(64, 0, seed + 13, sample=True, lens=lens64)
    ms_s, com_s, lens_s = timed(kv, st, 64, Bd.PROPOSE_SAMPLE, seed + 13, 2000)
    w, kvb, _, _ = step_bytes_flops(shape, lens_s, 64, N)
    qbytes = 2 * 64 * (N - 1) * V * 4        # q rows read and written per step
    out["qwen3_8b_b64_sample"] = {"ms_per_step": ms_s / args.steps, "value": com_s / (ms_s * 1e-3),
                                  "unit": "tokens/s", "step_bytes": w + kvb + qbytes,
                                  "steps": args.steps, "q_rows": "fp32, [64][3][151936]"}
    del kv, st
    # R-ISD at batch 32: the same steps with and without the adapter
    model.load_lora(Bd.random_device_lora(shape, 128, seed=seed, std=0.01), rank=128)
    kv, st = make(32, 2048, seed + 12)
    ms_b, _, _ = timed(kv, st, 32, 0, seed + 12, 0)
    ms_l, com_l, _ = timed(kv, st, 32, Bd.USE_LORA, seed + 12, 1000)
    out["risd_8b_b32"] = {"ms_per_step": ms_l / args.steps, "value": com_l / (ms_l * 1e-3),
                          "unit": "tokens/s", "base_ms_per_step": ms_b / args.steps,
                          "alpha": ms_l / ms_b, "steps": args.steps,
                          "adapter": "rank 128, A, B ~ N(0, 0.01), q/k/v/o/gate/up/down"}
    del kv, st
    torch.cuda.synchronize()
    return out


# DRAM bytes (read + write) of the tcgen05 attention kernel per byte of the
# layer's K+V, from one ncu capture of the same launch in the two-layer
# headline workload (549.6 MB for 527.9 MB of K+V; batch 64, prompts
# U[512, 4096]); the roofline's `traffic` scales it to this run's launch.
ATTN_DRAM_PER_KV_BYTE = 549.625 / 527.933


def roofline_entry(prof, shape, B, N, lens_steps, steps, peaks):
    """Roofline of the kernel class with the largest device time (lens_steps:
    the request lengths each profiled step started from, [steps][B])."""
    if not prof:
        return None
    R = 2 * N - 1
    top = max(prof, key=lambda k: prof[k][0])
    tot_ms, cnt = prof[top]
    avg_s = tot_ms / cnt * 1e-3
    M = B * R
    h, I, V = shape.hidden, shape.intermediate, shape.vocab
    gemm_flops = {"gemm_qkv": 2 * M * h * shape.qkv_dim, "gemm_o": 2 * M * shape.q_dim * h,
                  "gemm_gate_up_silu": 2 * M * h * 2 * I, "gemm_down": 2 * M * I * h,
                  "gemm_lm_head": 2 * M * h * V}
    if top in gemm_flops:
        # M rows do 2M flops per 2-byte weight: below the ridge (peak flops /
        # peak bytes, ~250 on B200) the projection streams weights (HBM-bound)
        ridge = peaks["bf16_sus"] * 1e12 / (peaks["hbm"] * 1e9)
        if M < ridge:
            wbytes = gemm_flops[top] / M   # 2 * in * out weight bytes
            achieved = wbytes / avg_s / 1e9
            peak = peaks["hbm"]
            return {"kernel": top, "bound": "hbm", "achieved": achieved, "peak": peak,
                    "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                    "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                    "peak_kind": f"{peaks['source']} HBM copy (weight streaming, {M} rows)",
                    "avg_launch_ms": avg_s * 1e3, "launches": cnt}
        achieved = gemm_flops[top] / avg_s / 1e12
        peak = peaks["bf16_sus"]
        return {"kernel": top, "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                "peak_kind": f"{peaks['source']} sustained bf16",
                "avg_launch_ms": avg_s * 1e3, "launches": cnt}
    if top.startswith("attention"):
        # one layer's K+V, averaged over the profiled steps
        kv = float(np.mean([sum(int(L) + R for L in ls) for ls in lens_steps])) * shape.kv_dim * 2 * 2
        algo = kv
        tc = (top == "attention" and shape.head_dim == 128 and shape.page_size == 64
              and R * (shape.n_q_heads // shape.n_kv_heads) <= 64)
        if tc:
            # the timed class also covers the layer's QKV reduction (its own
            # kernel, launched just before the attention): the QKV
            # projection's fp32 output read once, q and the block's K/V rows
            # written in bf16
            algo += M * shape.qkv_dim * 4 + M * (shape.q_dim + 2 * shape.kv_dim) * 2
        achieved = algo / avg_s / 1e9
        peak = peaks["hbm"]
        traffic = ATTN_DRAM_PER_KV_BYTE * kv if tc else None
        return {"kernel": top, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "algorithmic_bytes": algo,
                "kv_bytes": kv, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                "traffic_note": "ncu dram read+write of the tcgen05 attention kernel in one "
                                "capture of the same launch, scaled by this launch's K+V bytes "
                                "(the QKV reduction's own traffic is not in it)",
                "peak_kind": f"{peaks['source']} HBM copy",
                "avg_launch_ms": avg_s * 1e3, "launches": cnt}
    return {"kernel": top, "bound": "hbm", "achieved": None, "peak": peaks["hbm"], "unit": "GB/s",
            "frac": None, "traffic": None, "avg_launch_ms": avg_s * 1e3, "launches": cnt}


# ------------------------------------------------------------ oracle arm ---

def oracle_sample(args, n_reps: int, workload: str):
    """Time the oracle on a bounded sample of the workload and extrapolate.

    Sample: one decoder layer at the workload's widths and one 1/16 slice of
    the LM head, run by the oracle's own block forward for one request's
    2N-1 rows against a random KV prefix of the batch's mean length, plus
    the oracle's decide() on the full-vocabulary logits of that request.
    Full step time = batch x (layers x t_layer + 16 x t_lm_slice + t_decide).
    """
    from oracle import isd as oi
    from oracle import model as om
    wl = WORKLOADS[workload]
    shape, B, N = wl["shape"], wl["batch"], wl["stride"]
    R = 2 * N - 1
    slice_v = max(shape.vocab // 16, 128)
    one = dataclasses.replace(shape, n_layers=1, vocab=slice_v)
    w = synth.decoder_weights(one, seed=5)
    dec = om.Decoder(one, w)
    L = int(np.mean(synth.prompt_lengths(B, wl["len_lo"], wl["len_hi"], 1000)))
    kv = om.DenseKV(one)
    kv.k[0] = synth.normal((L, one.n_kv_heads, one.head_dim), 3, 1).astype(np.float64)
    kv.v[0] = synth.normal((L, one.n_kv_heads, one.head_dim), 3, 2).astype(np.float64)
    kv.n = L
    z_full = synth.synthetic_logits(R, shape.vocab, 4, boost=7.5).astype(np.float64)
    times, committed = [], 0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    for rep in range(n_reps):
        u = synth.controlled_uniforms(1, N, ACCEPT_RATE, 9, rep)[0]
        drafts = [int(np.argmax(z_full[j])) for j in range(N - 1)]
        # the sliced model's vocabulary holds the block's tokens
        toks = [1] + [t % slice_v for t in drafts] + [one.mask_token_id] * (R - N)
        t0 = time.perf_counter()
        om.block_forward(dec, kv, toks, L + np.arange(R))
        t1 = time.perf_counter()
        d = oi.decide(z_full, drafts, None, N, u)
        t2 = time.perf_counter()
        t_fwd = t1 - t0
        # the forward above = 1 layer + embedding + LM-head slice; time the slice alone too
        t3 = time.perf_counter()
        x = np.ones((R, shape.hidden))
        _ = om.rms_norm(x, dec.final_norm, shape.rms_eps) @ dec.lm_head.T
        t_lm = time.perf_counter() - t3
        t_layer = max(t_fwd - t_lm, 1e-9)
        t_step = B * (shape.n_layers * t_layer + (shape.vocab / slice_v) * t_lm + (t2 - t1))
        times.append(t_step)
        committed += B * (d.accepted + 1)
    per_step = float(np.mean(times))
    value = (committed / n_reps) / per_step
    sample = (f"{n_reps} reps of: 1 decoder layer at {workload} widths + 1/{shape.vocab // slice_v} "
              f"LM-head slice for one request's {R} rows against a random KV prefix of {L} "
              f"positions, plus decide() on full-vocab logits; extrapolated x{shape.n_layers} "
              f"layers, full LM head, batch {B}")
    return value, threads, sample, per_step


def run_reference(args, ws, rank):
    if rank != 0:
        return None
    reps = max(1, args.steps)
    for _ in range(min(args.warmup, 1)):
        oracle_sample(args, 1, args.workload)
    t0 = time.time()
    value, threads, sample, per_step = oracle_sample(args, reps, args.workload)
    return {"metric": metric_name(args.workload),
            "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args.workload, ws),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample, "wall_s": time.time() - t0,
                             "cpu_model": cpu_model(), "host_cpus": os.cpu_count()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_component(args):
    """Average device time of one component kernel over args.steps launches."""
    import torch
    from strided_verify_propose_b200 import binding as Bd

    torch.cuda.set_device(0)
    torch.manual_seed(0)
    kind, _, spec = args.component.partition(":")
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    if kind == "gemm":
        m, n, k, split = (int(v) for v in spec.split("x"))
        w = (torch.randn(n, k, device="cuda") * 0.02).to(torch.bfloat16)
        x = torch.randn(m, k, device="cuda").to(torch.bfloat16)

        def fn():
            Bd.gemm_bf16(w, x, split, status=st)
        work = {"flops": 2.0 * m * n * k,
                "bytes": 2.0 * n * k + 2.0 * m * k + 4.0 * split * m * n}
    elif kind == "gemm1":
        # one output slice, planned like the step's gate/up and LM head (stream-K)
        m, n, k = (int(v) for v in spec.split("x"))
        w = (torch.randn(n, k, device="cuda") * 0.02).to(torch.bfloat16)
        x = torch.randn(m, k, device="cuda").to(torch.bfloat16)
        wsp = Bd.gemm_workspace(m, n, k)

        def fn():
            Bd.gemm_bf16_single(w, x, wsp, status=st)
        work = {"flops": 2.0 * m * n * k, "bytes": 2.0 * n * k + 2.0 * m * k + 4.0 * m * n}
    elif kind == "attention":
        wl = WORKLOADS[spec]
        shape, Bn, N = wl["shape"], wl["batch"], wl["stride"]
        R, P, hd = 2 * N - 1, shape.page_size, shape.head_dim
        lens = synth.prompt_lengths(Bn, wl["len_lo"], wl["len_hi"], 7)
        need = [-(-(int(L) + R) // P) for L in lens]
        maxp = max(need) + 1
        num_pages = int(sum(need)) + 4
        table, _ = synth.page_layout(need, num_pages, maxp, 7)
        pool = (1, num_pages, shape.n_kv_heads, P, hd)
        kp = torch.randn(pool, device="cuda").to(torch.bfloat16)
        vp = torch.randn(pool, device="cuda").to(torch.bfloat16)
        q = torch.randn(Bn * R, shape.n_q_heads, hd, device="cuda").to(torch.bfloat16)
        pos = torch.tensor([int(L) + r for L in lens for r in range(R)], dtype=torch.int32,
                           device="cuda")
        tab = torch.from_numpy(table).cuda()

        def fn():
            Bd.paged_attention(q, pos, kp, vp, tab, R, 0, status=st)
        keys = float(sum(int(L) + R for L in lens))
        work = {"flops": 4.0 * keys * R * shape.n_q_heads * hd,
                "bytes": keys * shape.n_kv_heads * hd * 2 * 2 + 2.0 * q.numel() * 2}
    else:
        raise SystemExit(f"unknown component {args.component!r}")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        total += e0.elapsed_time(e1)
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())}")
    us = total / args.steps * 1e3
    return {"component": args.component, "avg_us": us, "launches": args.steps,
            "tflops": work["flops"] / us * 1e-6, "gbs": work["bytes"] / us * 1e-3,
            "l2": "256 MB flush between launches"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="qwen3_8b_b64", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the batch-1 and R-ISD runs reported beside the headline")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the steps launched one by one instead of replaying a CUDA graph")
    ap.add_argument("--component", default=None,
                    help="gemm:MxNxKxS, gemm1:MxNxK or attention:WORKLOAD (one kernel, for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.component:
        print(json.dumps(run_component(args)), flush=True)
        return
    ws, rank, local = setup_dist()
    if args.impl == "reference":
        res = run_reference(args, ws, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    res = run_cuda(args, ws, rank, local)
    if res is not None:
        if ws == 1 and not args.no_cpu_baseline:
            v, threads, sample, _ = oracle_sample(args, 2, args.workload)
            res["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                   "sample": sample, "cpu_model": cpu_model(),
                                   "host_cpus": os.cpu_count()}
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
