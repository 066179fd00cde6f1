"""Benchmark: KDA chunk forward tokens/s and decode steps/s on B200, with the
roofline fraction of the chunk forward and the CPU oracle beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]

One timed step = one `chunk_kda` forward over the varlen workload (4 packed
sequences of 4096/8192/12288/7168 tokens, H = 96, d_k = d_v = 128, bf16
inputs, fp32 states, lower bound -5, per-sequence initial states, final
states out). The decode step workload (64 sequences x 96 heads x 128 x 128
fp32 state, bf16 token vectors, one fresh token per step) is timed in the
same run, K' = 256 steps per timed pass, and reported under "decode"; so is the
serving decode token (conv window 4 + SiLU, the recurrent step and the output
gate fused, same geometry) under "decode_token", the chunk_kda backward on the
B1 T8192 H16 d128 chunk workload under "backward" (and at the 300M layer's geometry under
"backward_small"), and the other chunk workloads
(twin B4 T2048 H8 d32 with states, B1 T8192 H16 d128 lb -5, one layer of the
300M model: B128 T2048 H8 d_k 32 d_v 64 with the in-kernel gate) under
"chunk_workloads", each timed launch by launch with L2 flushed in between.
Inputs are resident in HBM and larger than L2 (3.9 GB chunk inputs, 384 MiB
decode state), so no L2 flush runs between iterations.

The chunk forward is one `kda_chunk_fwd` call that launches four kernels (set-up,
the intra-chunk pass, the exact-record pass for steep gates, the state pass);
its roofline entry divides the operator's algorithmic bytes by the time of the
whole call, and `traffic` is the DRAM traffic of those four launches.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own replica of
the workload (no data-path collective; weak scaling); the timed region is
bracketed by barriers and the slowest rank's device time is reported.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only); the main arm's `cpu_baseline` times the
same sample once, with the chunkwise oracle (form C) timed beside it.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
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

METRIC = "chunk_kda fwd tokens/s & decode steps/s on 1 B200; % of tensor/HBM roofline"
CHUNK_WL = 4
DECODE_WL = 3
DECODE_STEPS_PER_PASS = 256
# kernels one chunk forward launches on the bench workload (set-up, intra-chunk
# records, exact records, state pass) and the sources they are built from
CHUNK_SOURCES = ("kda_chunk_2pass.cu", "kda_tc_util.cuh", "kda_sm100.cuh", "kda_common.cuh", "kda_record.cuh")
# the other chunk workloads, timed one launch at a time with L2 flushed in between
EXTRA_CHUNK_WLS = (1, 2, 5)
L2_FLUSH_BYTES = 256 << 20
# heads of the varlen workload in the CPU oracle's sample (all four sequences)
CPU_SAMPLE_HEADS = 16


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def chunk_algorithmic(wl):
    """Algorithmic bytes and flops of one chunk forward launch.

    Per token-head: q, k, v, g, o (5 x 128 x 2 B) + beta (2 B) = 1282 B; plus
    one read of the initial and one write of the final fp32 state per
    (sequence, head). Flops per token-head (triangles exploited): A_kk, A_qk,
    W, U, A_qk.Delta = 3 C d_k + 2 C d_v, state terms W.S, Q.S, K^T.Delta =
    6 d_k d_v.
    """
    th = wl.tokens * wl.H
    esz = 2
    per_th = (3 * wl.Dk + 2 * wl.Dv) * esz + esz
    states = wl.n_seqs * wl.H * wl.Dk * wl.Dv * 4 * (int(wl.init_state) + int(wl.final_state))
    C = wl.chunk_size
    flops = th * (3 * C * wl.Dk + 2 * C * wl.Dv + 6 * wl.Dk * wl.Dv)
    return th * per_th + states, flops


def chunk_options(wl, inp):
    """chunk_kda keyword arguments of a chunk workload: L2 norm in the kernel,
    its lower bound, chunk size, in-kernel gate and beta form."""
    kw = dict(use_qk_l2norm_in_kernel=True, lower_bound=wl.lower_bound, chunk_size=wl.chunk_size)
    if wl.gate_in_kernel:
        kw.update(use_gate_in_kernel=True, A_log=inp["A_log"], dt_bias=inp["dt_bias"],
                  safe_gate=wl.lower_bound is not None)
    if wl.beta_prob:
        kw["use_beta_sigmoid_in_kernel"] = False
    return kw


# serving decode token (conv + SiLU, recurrent step, output gate): the production
# layer (H 96, d 128, conv window 4, lower bound -5) for 64 sequences
TOKEN_WL = dict(N=64, H=96, D=128, K=4, distinct_steps=32)


def token_algorithmic(N, H, D, K):
    """Bytes of one decode token: fp32 state read + write, fp32 conv windows read +
    write (3 D channels x K per head), the bf16 token vectors (x of 3 D channels, g,
    g_out, o) and one beta per head, plus one read of the shared conv weights."""
    heads = N * H
    per_head = 2 * D * D * 4 + 2 * 3 * D * K * 4 + (3 * D + 3 * D) * 2 + 2
    return heads * per_head + H * 3 * D * K * 4


# chunk_kda backward: the B1 T8192 H16 d128 lb-5 chunk workload with an output and a
# final-state cotangent (its 16 (sequence, head) chains run in segment form)
BWD_WL = 2


def bwd_small_workload(KI):
    """The backward at the 300M layer's geometry (B128 T2048 H8, d_k 32, d_v 64) with the
    log-decay gate and a lower bound of -5 (the autograd route takes the log gate): the
    micro-chunk backward."""
    return dataclasses.replace(KI.CHUNK_WORKLOADS[5], name="300M layer geometry B128 T2048 H8 dk32 dv64 lb-5",
                               gate_in_kernel=False, beta_prob=False, lower_bound=-5.0, seed=55)


def bwd_algorithmic(wl):
    """Flops and bytes of one chunk_kda backward call on workload wl (d_k = d_v = d),
    in the chunk form the library runs for it (bf16, d = 128, lower bound >= -5).

    Flops per token-head, as for the forward (2 per multiply-add, triangles
    exploited, C the chunk): the recompute of what the backward needs from the
    forward (A_kk, A_qk, W, U: 4 C d; W S and Khat^T D: 4 d^2), the cotangent chain
    (A_qk^T dO: C d; Khat dS, Qtil^T dO, W^T dD: 6 d^2) and the chunk-local terms
    (dO S^T, dD S^T, D dS^T: 6 d^2; dA_qk, dT' (two), dV, dKtil, A_kk again and the
    four gated products: 10 C d; the inverse's three C x C x C products, C^2) --
    15 C d + 16 d^2 + C^2 in all. Bytes: q, k, v, g, do, beta read, dq, dk, dv, dg,
    dbeta written, the final-state cotangent read and the initial-state gradient
    written.
    """
    th = wl.tokens * wl.H
    esz = 2
    per_th = 2 * (3 * wl.Dk + 2 * wl.Dv) * esz + 2 * esz
    states = 2 * wl.n_seqs * wl.H * wl.Dk * wl.Dv * 4
    C, d = wl.chunk_size, wl.Dk
    return th * (15 * C * d + 16 * d * d + C * C), th * per_th + states


def decode_algorithmic(wl):
    """Bytes and flops of one decode step: fp32 state read + write, q/k/g/v/o
    vectors and one beta per head; 7 d_k d_v flops per head."""
    heads = wl.N * wl.H
    per_head = 2 * wl.Dk * wl.Dv * 4 + (3 * wl.Dk + 2 * wl.Dv) * 2 + 2
    return heads * per_head, heads * 7 * wl.Dk * wl.Dv


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, log_dir=None):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(log_dir or tempfile.gettempdir(), f"kda_clocks_rank{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "kimi_delta_attention_20_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(key, sha):
    """DRAM bytes per launch recorded from an ncu capture of this exact kernel
    source (profiles/ncu_traffic.json), else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f)[key]
        return rec["bytes_per_launch"] if rec.get("source_sha") == sha else None
    except Exception:
        return None


def launches():
    """Kernel launches libkda.so has queued so far (its own counter)."""
    from kimi_delta_attention_20_b200 import _abi
    return int(_abi.load().kda_launch_count())


def bench_config(world):
    """The `config` object of the JSON line (both arms)."""
    return {
        "workload": "chunk_kda fwd: varlen 4096/8192/12288/7168 (T=31744), H=96, d_k=d_v=128, "
                    "bf16, lower_bound=-5, chunk 64, initial+final states; decode: N=64, H=96, "
                    "d=128, fp32 state, 256 steps per pass",
        "tokens_per_step": 31744, "heads": 96, "d_k": 128, "d_v": 128,
        "chunk_size": 64, "parallelism": f"replica per GPU x{world} (no collective)",
        "l2": "inputs larger than L2 (3.9 GB chunk inputs, 384 MiB decode state); no flush "
              "(the smaller chunk workloads flush L2 before every timed launch)",
    }


# --------------------------------------------------------------------------- ranks

def rank_barrier(world):
    """Barrier across ranks (no-op for a single process)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks_value(x, world, device):
    """Slowest rank's value: an all-reduce MAX of one float (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, units_per_rank, ms_max):
    """Weak scaling: every rank processes `units_per_rank`; the job takes the slowest
    rank's time, so the whole-job rate is world * units / that time."""
    return world * units_per_rank / (ms_max * 1e-3)


# --------------------------------------------------------------------------- GPU arm

def run_kda(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import kda_inputs as KI
    import kimi_delta_attention_20_b200 as kda
    from kimi_delta_attention_20_b200 import _abi

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, peak_kind = load_peaks()

    wl = KI.CHUNK_WORKLOADS[args.workload if (args.only and args.workload is not None) else CHUNK_WL]
    if args.only == "chunk" and args.chunk_heads:  # fewer heads for profiler captures
        wl = dataclasses.replace(wl, H=args.chunk_heads, name=f"{wl.name} (H{args.chunk_heads})")
    if args.only in (None, "chunk"):  # the single-leg profiler runs allocate only their own leg
        inp = KI.chunk_inputs(wl, device=dev)
        q, k, v, g, beta = (inp[n] for n in ("q", "k", "v", "g", "beta"))
        S0, cu = inp["initial_state"], inp["cu_seqlens"]
        cu_cpu = cu.cpu() if cu is not None else None  # host copy: no blocking read per call
        o = torch.empty_like(v)
        S_out = torch.empty(wl.n_seqs, wl.H, wl.Dk, wl.Dv, dtype=torch.float32, device=dev) \
            if wl.final_state else None
        opts = chunk_options(wl, inp)
        ws_bytes = kda.chunk_workspace_bytes(wl.B, wl.T, wl.H, wl.Dk, wl.Dv, N=wl.n_seqs,
                                             varlen=wl.seqlens is not None)
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)

    def chunk_step():
        kda.chunk_kda(q, k, v, g, beta, initial_state=S0, output_final_state=wl.final_state,
                      cu_seqlens=cu, cu_seqlens_cpu=cu_cpu, out=o, final_state_out=S_out,
                      workspace=ws, **opts)

    dwl = KI.DECODE_WORKLOADS[DECODE_WL]
    if args.only in (None, "token"):
        tk = KI.draw_token(TOKEN_WL["N"], TOKEN_WL["H"], TOKEN_WL["D"], TOKEN_WL["D"], TOKEN_WL["K"],
                           TOKEN_WL["distinct_steps"], dtype=torch.bfloat16, seed=9, device=dev)
        tk_o = torch.empty(TOKEN_WL["N"], TOKEN_WL["H"], TOKEN_WL["D"], dtype=torch.bfloat16, device=dev)

    def token_step(t):
        i = t % TOKEN_WL["distinct_steps"]
        kda.decode_token(tk["x"][i], tk["w"], tk["cs"], tk["g"][i], tk["beta"][i], tk["S0"],
                         g_out=tk["g_out"][i], lower_bound=-5.0, out=tk_o)

    bwl = KI.CHUNK_WORKLOADS[BWD_WL]
    BWD_SMALL = bwd_small_workload(KI)
    if args.only == "bwd" and args.bwd_tokens:  # shorter sequence for profiler captures
        bwl = dataclasses.replace(bwl, T=args.bwd_tokens, name=f"{bwl.name} T{args.bwd_tokens}")
    if args.only in (None, "bwd"):
        binp = KI.chunk_inputs(bwl, device=dev)
        bgen = torch.Generator(device=dev)
        bgen.manual_seed(bwl.seed + 1000)
        b_do = torch.randn(binp["v"].shape, generator=bgen, device=dev).to(bwl.dtype)
        b_dSf = torch.randn(bwl.n_seqs, bwl.H, bwl.Dk, bwl.Dv, generator=bgen, device=dev) * 0.5
        b_ws = torch.empty(kda.chunk_bwd_workspace_bytes(bwl.B, bwl.T, bwl.H, bwl.Dk, bwl.Dv, N=bwl.n_seqs),
                           dtype=torch.uint8, device=dev)

    if args.only is None:
        sinp = KI.chunk_inputs(BWD_SMALL, device=dev)
        sgen = torch.Generator(device=dev)
        sgen.manual_seed(BWD_SMALL.seed + 1000)
        s_do = torch.randn(sinp["v"].shape, generator=sgen, device=dev).to(BWD_SMALL.dtype)

    def bwd_small_step():
        return kda.chunk_kda_bwd(sinp["q"], sinp["k"], sinp["v"], sinp["g"], sinp["beta"], s_do,
                                 use_qk_l2norm_in_kernel=True, lower_bound=BWD_SMALL.lower_bound)

    def bwd_step():
        return kda.chunk_kda_bwd(binp["q"], binp["k"], binp["v"], binp["g"], binp["beta"], b_do,
                                 dfinal_state=b_dSf, use_qk_l2norm_in_kernel=True,
                                 lower_bound=bwl.lower_bound, workspace=b_ws)

    if args.only in (None, "decode"):
        dinp = KI.decode_inputs(dwl, device=dev)
        state = dinp["state"].clone()
        od = torch.empty(dwl.N, dwl.H, dwl.Dv, dtype=dwl.dtype, device=dev)

    def decode_step(t):
        kda.recurrent_step(dinp["q"][t], dinp["k"][t], dinp["v"][t], dinp["g"][t],
                           dinp["beta"][t], state, out=od)

    def barrier():
        rank_barrier(world)

    def max_over_ranks(x):
        return max_over_ranks_value(x, world, dev)

    stream = torch.cuda.current_stream(dev)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local_rank

    if args.only:
        # one kernel, few launches: the shape profiler captures use
        one = {"chunk": chunk_step, "decode": lambda: decode_step(0), "token": lambda: token_step(0),
               "bwd": bwd_step}[args.only]
        for _ in range(args.warmup):
            one()
        torch.cuda.synchronize(dev)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            one()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        ms = a0.elapsed_time(a1) / args.steps
        out = {"only": args.only, "ms_per_launch": ms, "launches": args.steps}
        if args.only == "chunk":
            nbytes, nflops = chunk_algorithmic(wl)
            gbs = nbytes / (ms * 1e-3) / 1e9
            out.update({"workload": wl.name, "tokens_per_s": wl.tokens / (ms * 1e-3),
                        "algorithmic_bytes_per_launch": nbytes, "achieved_gbs": gbs,
                        "hbm_frac": gbs / hbm_peak, "peak_kind": peak_kind,
                        "achieved_tflops": nflops / (ms * 1e-3) / 1e12})
        return out

    def capture_pass(step_fn):
        """One pass of DECODE_STEPS_PER_PASS decode steps as a CUDA graph, the way a serving
        engine launches its decode steps: the same kernels, without the launch gaps.
        Returns the graph and the number of library kernels it holds."""
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step_fn(0)
        torch.cuda.current_stream(dev).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        n0 = launches()
        with torch.cuda.graph(graph):
            for t in range(DECODE_STEPS_PER_PASS):
                step_fn(t)
        torch.cuda.synchronize(dev)
        return graph, launches() - n0

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if args.only is None else None

    def time_chunk_workload(idx):
        """One of the smaller chunk workloads: K launches, each timed by its own events
        with L2 flushed (a 256 MiB write) before it, the flush outside the events."""
        xwl = KI.CHUNK_WORKLOADS[idx]
        xin = KI.chunk_inputs(xwl, device=dev)
        xo = torch.empty_like(xin["v"])
        xS = torch.empty(xwl.n_seqs, xwl.H, xwl.Dk, xwl.Dv, dtype=torch.float32, device=dev) \
            if xwl.final_state else None
        xopts = chunk_options(xwl, xin)
        xcu = xin["cu_seqlens"]
        xcu_cpu = xcu.cpu() if xcu is not None else None
        xws = torch.empty(max(kda.chunk_workspace_bytes(xwl.B, xwl.T, xwl.H, xwl.Dk, xwl.Dv, N=xwl.n_seqs,
                                                        varlen=xwl.seqlens is not None), 1),
                          dtype=torch.uint8, device=dev)

        def step():
            kda.chunk_kda(xin["q"], xin["k"], xin["v"], xin["g"], xin["beta"], initial_state=xin["initial_state"],
                          output_final_state=xwl.final_state, cu_seqlens=xcu, cu_seqlens_cpu=xcu_cpu, out=xo,
                          final_state_out=xS, workspace=xws, **xopts)

        for _ in range(args.warmup):
            step()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        barrier(); torch.cuda.synchronize(dev)
        n0 = launches()
        for a0, a1 in evs:
            flush.zero_()
            a0.record(stream)
            step()
            a1.record(stream)
        torch.cuda.synchronize(dev); barrier()
        n_launch = launches() - n0
        ms = max_over_ranks(sum(a0.elapsed_time(a1) for a0, a1 in evs)) / args.steps
        nbytes, nflops = chunk_algorithmic(xwl)
        gbs = nbytes / (ms * 1e-3) / 1e9
        tflops = nflops / (ms * 1e-3) / 1e12
        leg = {
            "workload": xwl.name, "value": whole_job_rate(world, xwl.tokens, ms), "unit": "tokens/s",
            "ms_per_step": ms, "steps_timed": args.steps, "launches_per_step": n_launch / args.steps,
            "l2": "flushed before every timed launch",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": nbytes,
                         "tensor": {"achieved_tflops": tflops, "peak_tflops": tc_peak,
                                    "frac": tflops / tc_peak}},
        }
        del xin, xo, xS, xws
        return leg, n_launch

    # warm-up (untimed)
    for _ in range(args.warmup):
        chunk_step()
    for t in range(min(args.warmup, dwl.steps)):
        decode_step(t)
    dec_graph, dec_graph_launches = capture_pass(lambda t: decode_step(t % dwl.steps))
    tok_graph, tok_graph_launches = capture_pass(token_step)
    dec_graph.replay()
    tok_graph.replay()
    torch.cuda.synchronize(dev)

    with ClockSampler(gpu_index, args.clocks_log) as clocks:
        # chunk forward: K timed steps
        barrier(); torch.cuda.synchronize(dev)
        n0 = launches()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            chunk_step()
        e1.record(stream)
        torch.cuda.synchronize(dev); barrier()
        chunk_launches = launches() - n0
        chunk_ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps

        # decode: K passes of 256 steps each
        state.copy_(dinp["state"])
        barrier(); torch.cuda.synchronize(dev)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(args.steps):
            dec_graph.replay()
        d1.record(stream)
        nsteps = args.steps * DECODE_STEPS_PER_PASS
        torch.cuda.synchronize(dev); barrier()
        dec_ms = max_over_ranks(d0.elapsed_time(d1)) / nsteps
        # serving decode token: K passes of 256 tokens (cycling over the drawn inputs)
        barrier(); torch.cuda.synchronize(dev)
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        for _ in range(args.steps):
            tok_graph.replay()
        k1.record(stream)
        ntok = args.steps * DECODE_STEPS_PER_PASS
        torch.cuda.synchronize(dev); barrier()
        tok_ms = max_over_ranks(k0.elapsed_time(k1)) / ntok
        # chunk_kda backward: K timed calls
        for _ in range(args.warmup):
            bwd_step()
        barrier(); torch.cuda.synchronize(dev)
        n0 = launches()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.steps):
            bwd_step()
        b1.record(stream)
        torch.cuda.synchronize(dev); barrier()
        bwd_launches = launches() - n0
        bwd_ms = max_over_ranks(b0.elapsed_time(b1)) / args.steps
        # the small-head backward: K timed calls
        for _ in range(args.warmup):
            bwd_small_step()
        barrier(); torch.cuda.synchronize(dev)
        n0 = launches()
        b0.record(stream)
        for _ in range(args.steps):
            bwd_small_step()
        b1.record(stream)
        torch.cuda.synchronize(dev); barrier()
        bwd_small_launches = launches() - n0
        bwd_small_ms = max_over_ranks(b0.elapsed_time(b1)) / args.steps
        # the smaller chunk workloads
        extra_legs, extra_launches = {}, 0
        for idx in EXTRA_CHUNK_WLS:
            leg, n_launch = time_chunk_workload(idx)
            extra_legs[str(idx)] = leg
            extra_launches += n_launch
    clk = clocks.summary()

    # end to end through the public API with host buffers: every step copies its inputs
    # in from pinned host memory, runs the chunk forward and copies o and the final
    # states back. Steps are pipelined over three streams with two device buffer sets,
    # so step i's inputs cross PCIe while step i-1 computes and its outputs come back.
    host = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v", "g", "beta", "initial_state")}
    cu_host = cu.cpu()
    h_o = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    h_S = [torch.empty(S_out.shape, dtype=S_out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + cu_host.numel() * 4
    d2h = o.numel() * o.element_size() + S_out.numel() * 4
    dbuf = [{n: torch.empty_like(inp[n]) for n in host} for _ in range(2)]
    cu_dev = [torch.empty_like(cu) for _ in range(2)]
    dout = [(torch.empty_like(o), torch.empty_like(S_out)) for _ in range(2)]
    s_in, s_c, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in, ev_done, ev_read = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])  # step i - 2 has consumed these input buffers
            for n in host:
                dbuf[b][n].copy_(host[n], non_blocking=True)
            cu_dev[b].copy_(cu_host, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(ev_in[b])
            if i >= 2:
                s_c.wait_event(ev_read[b])  # step i - 2's outputs have been copied back
            kda.chunk_kda(dbuf[b]["q"], dbuf[b]["k"], dbuf[b]["v"], dbuf[b]["g"], dbuf[b]["beta"],
                          initial_state=dbuf[b]["initial_state"], output_final_state=True,
                          cu_seqlens=cu_dev[b], cu_seqlens_cpu=cu_host, out=dout[b][0],
                          final_state_out=dout[b][1], workspace=ws, **opts)
            ev_done[b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            h_o[b].copy_(dout[b][0], non_blocking=True)
            h_S[b].copy_(dout[b][1], non_blocking=True)
            ev_read[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e2e_steps = max(3, min(args.steps, 6))
    barrier(); torch.cuda.synchronize(dev)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for st_ in (s_in, s_c, s_out):
        st_.wait_event(x0)
    for i in range(e2e_steps):
        e2e_step(i)
    x1.record(s_out)  # the last device-to-host copy is the last work of the pipeline
    torch.cuda.synchronize(dev); barrier()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1)) / e2e_steps

    chunk_bytes, chunk_flops = chunk_algorithmic(wl)
    dec_bytes, dec_flops = decode_algorithmic(dwl)
    chunk_gbs = chunk_bytes / (chunk_ms * 1e-3) / 1e9
    chunk_tflops = chunk_flops / (chunk_ms * 1e-3) / 1e12
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9
    tok_bytes = token_algorithmic(TOKEN_WL["N"], TOKEN_WL["H"], TOKEN_WL["D"], TOKEN_WL["K"])
    tok_gbs = tok_bytes / (tok_ms * 1e-3) / 1e9
    bwd_flops, bwd_bytes = bwd_algorithmic(bwl)
    # bytes of the small-head backward (no final-state cotangent, no initial state), all bf16:
    # q, k, g, v, do, beta in; dq, dk, dg, dv, dbeta out
    bwd_small_bytes = BWD_SMALL.tokens * BWD_SMALL.H * ((6 * BWD_SMALL.Dk + 3 * BWD_SMALL.Dv) * 2 + 2 * 2)
    chunk_sha = source_sha(*CHUNK_SOURCES)
    result = {
        "metric": METRIC,
        "value": whole_job_rate(world, wl.tokens, chunk_ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": chunk_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the varlen chunk and decode workloads)",
        "config": bench_config(world),
        "roofline": {
            "bound": "hbm", "achieved": chunk_gbs, "peak": hbm_peak, "unit": "GB/s",
            "frac": chunk_gbs / hbm_peak, "peak_kind": peak_kind,
            "algorithmic_bytes_per_launch": chunk_bytes,
            "traffic": ncu_traffic("chunk", chunk_sha),
            "tensor": {"achieved_tflops": chunk_tflops, "peak_tflops": tc_peak,
                       "frac": chunk_tflops / tc_peak},
        },
        "decode": {
            "value": whole_job_rate(world, 1, dec_ms), "unit": "steps/s",
            "tokens_per_s": whole_job_rate(world, dwl.N, dec_ms), "ms_per_step": dec_ms,
            "steps_timed": nsteps, "launch": "CUDA graph of 256 steps per pass",
            "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": dec_gbs / hbm_peak, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": dec_bytes,
                         "traffic": ncu_traffic("decode", source_sha("kda_decode.cu",
                                                                     "kda_common.cuh"))},
        },
        "decode_token": {
            "value": whole_job_rate(world, 1, tok_ms), "unit": "steps/s",
            "tokens_per_s": whole_job_rate(world, TOKEN_WL["N"], tok_ms), "ms_per_step": tok_ms,
            "steps_timed": ntok, "launch": "CUDA graph of 256 steps per pass",
            "workload": "serving decode token: conv window 4 + SiLU, recurrent step, output gate; "
                        "N=64, H=96, d=128, bf16 vectors, fp32 state and windows, lower_bound=-5",
            "roofline": {"bound": "hbm", "achieved": tok_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": tok_gbs / hbm_peak, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": tok_bytes},
        },
        "backward": {
            "value": whole_job_rate(world, bwl.tokens, bwd_ms), "unit": "tokens/s", "ms_per_step": bwd_ms,
            "steps_timed": args.steps,
            "workload": "chunk_kda backward: B1 T8192 H16 d128, bf16, lower_bound=-5, output and "
                        "final-state cotangents, initial-state gradient out",
            "form": "chunked: forward with state saves, cotangent chain on tcgen05 over segments, "
                    "chunk-local gradients on warp-level MMAs",
            "roofline": {"bound": "tensor", "achieved": bwd_flops / (bwd_ms * 1e-3) / 1e12,
                         "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": bwd_flops / (bwd_ms * 1e-3) / 1e12 / tc_peak,
                         "peak_kind": peak_kind,
                         "algorithmic_flops_per_launch": bwd_flops,
                         "hbm": {"algorithmic_bytes_per_launch": bwd_bytes,
                                 "achieved_gbs": bwd_bytes / (bwd_ms * 1e-3) / 1e9}},
        },
        "backward_small": {
            "value": whole_job_rate(world, BWD_SMALL.tokens, bwd_small_ms), "unit": "tokens/s",
            "ms_per_step": bwd_small_ms, "steps_timed": args.steps,
            "workload": "chunk_kda backward at the 300M layer's geometry: B128 T2048 H8, d_k 32, d_v 64, "
                        "bf16, log-decay gate with lower_bound=-5, output cotangent",
            "form": "micro-chunk: the d_k = 32 forward saving each 16-token micro-chunk's state, then one "
                    "warp per (sequence, head) on warp-level MMAs",
            "roofline": {"bound": "hbm", "achieved": bwd_small_bytes / (bwd_small_ms * 1e-3) / 1e9,
                         "peak": hbm_peak, "unit": "GB/s",
                         "frac": bwd_small_bytes / (bwd_small_ms * 1e-3) / 1e9 / hbm_peak,
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": bwd_small_bytes},
        },
        "e2e": {"value": whole_job_rate(world, wl.tokens, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipelined": "copy-in, compute and copy-back of consecutive steps on three streams"},
        "chunk_workloads": extra_legs,
        "gpu_launches": chunk_launches + args.steps * (dec_graph_launches + tok_graph_launches)
        + bwd_launches + bwd_small_launches + extra_launches,
        "gpu_launches_by_leg": {"chunk": chunk_launches, "decode": args.steps * dec_graph_launches,
                                "decode_token": args.steps * tok_graph_launches, "backward": bwd_launches,
                                "backward_small": bwd_small_launches,
                                "chunk_workloads": extra_launches,
                                "counted_by": "libkda.so's own launch counter (kda_launch_count); graph "
                                              "replays count the kernels captured in the graph"},
        "clocks": clk,
        "library": os.path.relpath(_abi.LIB_PATH, ROOT),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl)
    return result


# --------------------------------------------------------------------------- CPU oracle

def cpu_sample(wl, heads=CPU_SAMPLE_HEADS):
    """The CPU oracle's sample of the varlen chunk workload: the same recipe (lengths,
    dims, dtype, distributions, seed) drawn on the host for the first `heads` heads."""
    import kda_inputs as KI
    return KI.draw_chunk(1, wl.T, heads, wl.Dk, wl.Dv, dtype=wl.dtype, seed=wl.seed,
                         seqlens=wl.seqlens, init_state=wl.init_state)


def time_oracle(inp, wl, form):
    """Seconds the fp64 oracle (as it stands) takes for the sample, on all host cores."""
    import oracle
    fn = {"R": oracle.recurrent, "C": oracle.chunkwise}[form]
    t0 = time.perf_counter()
    fn(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], inp["beta"][0],
       initial_state=inp["initial_state"], cu_seqlens=inp["cu_seqlens"], lower_bound=wl.lower_bound,
       nthreads=os.cpu_count() or 1)
    return time.perf_counter() - t0


def sample_rate(wl, heads, seconds):
    """tokens/s of the whole workload implied by the sample: it holds `heads` of wl.H heads."""
    return wl.tokens * heads / wl.H / seconds


def cpu_baseline(wl, heads=CPU_SAMPLE_HEADS):
    """The oracle timed on the sample: form R (the definition, the baseline) and form C
    (the chunkwise oracle) beside it."""
    inp = cpu_sample(wl, heads)
    tR = time_oracle(inp, wl, "R")
    tC = time_oracle(inp, wl, "C")
    return {"value": sample_rate(wl, heads, tR), "unit": "tokens/s", "cores": os.cpu_count() or 1,
            "kind": "oracle",
            "sample": f"fp64 form R (token recurrence) on all {wl.n_seqs} sequences ({wl.tokens} tokens) x "
                      f"{heads} of {wl.H} heads in {tR:.2f} s, scaled to tokens of all {wl.H} heads",
            "form_c": {"value": sample_rate(wl, heads, tC), "unit": "tokens/s", "seconds": tC,
                       "kind": "oracle (chunkwise form, chunk 64)"}}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, each step one run of form R over the
    sample. ms_per_step is the measured wall time of that run; `value` is the rate of
    the whole workload that it implies."""
    import kda_inputs as KI
    wl = KI.CHUNK_WORKLOADS[CHUNK_WL]
    heads = CPU_SAMPLE_HEADS
    inp = cpu_sample(wl, heads)
    for _ in range(args.warmup):
        pass  # the oracle keeps no state between runs: warm-up steps are no-ops
    secs = [time_oracle(inp, wl, "R") for _ in range(args.steps)]
    per_step = statistics.mean(secs)
    v = sample_rate(wl, heads, per_step)
    tC = time_oracle(inp, wl, "C")
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": bench_config(1),
        "step": f"form R over all {wl.n_seqs} sequences x {heads} of {wl.H} heads; the whole workload "
                f"would take {per_step * wl.H / heads * 1e3:.0f} ms",
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count() or 1, "kind": "oracle",
                         "sample": f"fp64 form R on all {wl.n_seqs} sequences ({wl.tokens} tokens) x {heads} "
                                   f"of {wl.H} heads per step, {per_step:.2f} s per step",
                         "form_c": {"value": sample_rate(wl, heads, tC), "unit": "tokens/s", "seconds": tC,
                                    "kind": "oracle (chunkwise form, chunk 64)"}},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["chunk", "decode", "token", "bwd"], default=None,
                    help="run one leg only and print its timing (for profiler captures)")
    ap.add_argument("--bwd-tokens", type=int, default=None,
                    help="with --only bwd: sequence length of the backward workload (default 8192)")
    ap.add_argument("--workload", type=int, default=None,
                    help="with --only chunk: chunk workload index (default: the varlen H=96 one)")
    ap.add_argument("--chunk-heads", type=int, default=None,
                    help="with --only chunk: number of heads of the chunk workload (default: its own)")
    ap.add_argument("--clocks-log", default=None,
                    help="directory for the nvidia-smi clock samples (default: the temp directory)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "kda":
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_kda(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
