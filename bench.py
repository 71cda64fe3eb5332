#!/usr/bin/env python
"""Benchmark of the channel-wise gated delta-rule hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  gdelta_state_init (S <- 0)  ->  gdelta_fwd_chunked over the batch
  (S_in = S_out = S)  ->  one gdelta_decode_step continuing every head.
Workload (per GPU): B=4, T=4096, H=16, d_k=d_v=128, chunk 64, bf16 tokens,
fp32 log-decay and state -- the Muir 1.34B-scale layer (the Muir review's
d=2048 model: 16 heads of 128; 4096-token training length), synthetic data
from ``synth``.  The inputs (680 MB) are larger than the 126 MB L2, so no L2
flush is needed between steps.

A second measurement times the decode step alone on batch 64 x 16 heads (fp32
state of 67 MB, which fits in L2), flushing L2 between steps.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
N > 1 is launched with torchrun (one process per GPU); every rank runs its own
batch (independent heads, no collective on the data path) and rank 0 prints
one JSON line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
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

METRIC = ("gated-delta chunked fwd tokens/s (H=16,dk=dv=128); decode-step state HBM GB/s")
WORKLOAD = "muir1b3_bf16"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--path", choices=["auto", "simt", "tc"], default="auto")
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stream-tokens", type=int, default=0,
                    help="also serve one long stream (B1 H16) of this many tokens: forward calls of "
                         "16384 tokens carrying the state, then decode steps (0 = off)")
    ap.add_argument("--bwd-calls", type=int, default=2,
                    help="timed gdelta_bwd calls on the workload (0 = skip the backward measurement)")
    ap.add_argument("--no-forms", action="store_true",
                    help="skip the forward timings of the reduced gate forms")
    ap.add_argument("--no-gate-proj", action="store_true",
                    help="skip the five-gate projection timing")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the forward timings of the other full-size workloads (350M layer, 32k tokens)")
    # profiling aid: a smaller case of the same workload (fewer batch rows) for
    # ncu captures that must stay small; the bench line itself uses the default
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch rows (for profiler captures only)")
    return ap.parse_args()


# ---------------------------------------------------------------- plumbing

def dist_init(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, local, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms from before the
    warm-up until after the last GPU measurement (the timed loops are too short
    for the sampling period on their own; the GPU is under load throughout)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # wait (at most 5 s) until the first sample is written, so that sampling is live
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        # samples taken while kernels ran (the window also holds host-only work,
        # such as generating the other workloads' inputs); all of them if none
        n_all = len(rows)
        loaded = [r for r in rows if (num(r[9]) or 0.0) >= 50.0]
        rows = loaded or rows
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": n_all, "samples_under_load": len(loaded), "reasons": reasons}


def fwd_bytes(B, T, H, dk, dv, tok_bytes, z=True, beta=False, decay_tok=False):
    """Algorithmic HBM bytes of one chunked-forward launch: q,k,z,b (d_k) and
    v,w,g (d_v) tokens, fp32 log-decay, y, the fp32 state read and written.
    Reduced gate forms: no z; one beta per token and head in place of the b
    and w rows; one fp32 log-decay per token and head."""
    n_dk = 2 + (1 if z else 0) + (0 if beta else 1)          # q, k [, z] [, b]
    n_dv = 2 + (0 if beta else 1)                            # v, g [, w]
    per_token_head = (n_dk * dk + n_dv * dv + dv) * tok_bytes + (4 if decay_tok else 4 * dk)
    if beta:
        per_token_head += tok_bytes
    return B * T * H * per_token_head + 2 * B * H * dk * dv * 4 + H * dk * 4


def decode_bytes(B, H, dk, dv, tok_bytes):
    """Algorithmic bytes of one decode step: state read + write, the token
    vectors, the fp32 log-decay and y."""
    return B * H * (2 * dk * dv * 4 + 4 * dk * tok_bytes + 3 * dv * tok_bytes + 4 * dk
                    + dv * tok_bytes) + H * dk * 4


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file: str):
    """Per-launch DRAM bytes recorded from an ncu capture of the current
    source of ``kernel_file`` (profiles/traffic.json), else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel_file)
        if rec and rec.get("source_sha") == source_digest([kernel_file]):
            return float(rec["bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, local, world):
    import channel_gated_delta_b200 as gd
    import synth

    dev = torch.device("cuda", local)
    shape = synth.CONFIGS[WORKLOAD]
    if args.batch > 0:
        shape = dataclasses.replace(shape, B=args.batch)
    B, T, H, dk, dv, C = shape.B, shape.T, shape.H, shape.dk, shape.dv, shape.chunk
    host = synth.generate(shape, seed=shape.seed + 1000 * rank)
    d = {k: v.to(dev) for k, v in host.items()}
    S = torch.empty(B, H, dk, dv, device=dev)
    y = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=dev)
    step_tok = synth.decode_step_inputs(0, seed=77 + rank, B=B, H=H, dk=dk, dv=dv)
    dtok = {k: v.to(dev) for k, v in step_tok.items()}
    y_dec = torch.empty(B, H, dv, dtype=torch.bfloat16, device=dev)
    path = gd.gdelta_fwd_selected_path(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                       d["log_alpha"], chunk=C, path=args.path)
    ws_bytes = gd.gdelta_fwd_workspace_bytes(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                             d["log_alpha"], chunk=C, path=args.path)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev) if ws_bytes else None
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        gd.gdelta_state_init(S, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                              gamma_stat=d["gamma_stat"], S_in=S, S_out=S, y=y, chunk=C,
                              path=args.path, workspace=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        gd.gdelta_decode_step(dtok["q"], dtok["k"], dtok["v"], dtok["b"], dtok["w"], dtok["z"],
                              dtok["g"], dtok["log_alpha"], S, gamma_stat=d["gamma_stat"], y=y_dec,
                              stream=stream)
        if ev is not None:
            ev[3].record(stream)

    clocks = ClockSampler(dev.index if world == 1 else local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if gd.gdelta_get_last_device_error(stream) != 0:
        raise RuntimeError("device status word set during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = start.elapsed_time(end)
    fwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    ms_step = max_over_ranks(total_ms / args.steps, world)
    fwd_avg_ms = max_over_ranks(sum(fwd_ms) / len(fwd_ms), world)

    tok_per_step = B * T + B                       # prefill tokens + one decode token per row
    value = tok_per_step * world / (ms_step * 1e-3)
    hbm, peak_kind = peaks()
    fb = fwd_bytes(B, T, H, dk, dv, 2)
    achieved = fb / (fwd_avg_ms * 1e-3) / 1e9
    kernel_file = ("channel_gated_delta_b200/csrc/fwd_tc.cu" if path == "tc"
                   else "channel_gated_delta_b200/csrc/fwd_simt.cu")
    traffic = recorded_traffic(kernel_file)

    # ---- decode-only measurement (batch 64 x 16 heads, L2 flushed between steps)
    dec = run_decode(args, dev, stream, rank, world) if args.decode_steps > 0 else None

    # ---- forward alone on the reduced gate forms (same workload shape)
    forms = None if args.no_forms else run_forms(args, gd, d, shape, dev, stream, ws, world)

    # ---- forward alone on the other full-size workloads
    configs = None if (args.no_configs or args.batch > 0) else run_configs(args, gd, dev, stream, rank, world)

    # ---- the five-gate projection that produces the gates of this layer
    gproj = None if args.no_gate_proj else run_gate_proj(args, gd, shape, dev, stream, rank, world)

    # ---- backward pass on the same workload
    bwd = run_bwd(args, gd, d, shape, dev, stream, world) if args.bwd_calls > 0 else None

    # ---- one long stream: consecutive forward calls, then decode (opt-in)
    stream_res = run_stream(args, gd, d, shape, dev, stream, world) if args.stream_tokens > 0 else None

    # ---- end to end through the public API with host buffers
    e2e = None if args.no_e2e else run_e2e(args, gd, host, dev, stream, shape, world, path)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    clk["window"] = "from before the warm-up to the end of the last GPU measurement"

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(host, shape)

    line = {
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
        "dtype": "f32" if path == "simt" else "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"{WORKLOAD}: B{B} T{T} H{H} dk=dv={dk} chunk {C}, bf16 tokens, fp32 log-decay and state",
            "step": "state_init + fwd_chunked + 1 decode step (all heads)",
            "kernels_per_step": 4 if path == "tc" else 3,
            "tokens_per_step_per_gpu": tok_per_step,
            "kernel_path": path,
            "workspace_bytes": ws_bytes,
            "l2": "inputs (680 MB per GPU) larger than the 126 MB L2; no flush",
            "parallelism": f"dp{world} (independent batches per GPU, no collective)",
        },
        "roofline": {
            "bound": "hbm",
            # the timed unit is one gdelta_fwd_chunked call: on the tensor-core path
            # the intra-chunk kernel followed by the chain kernel
            "kernel": ("gdelta_fwd_chunked = gdn2_chunk_intra_tc_kernel + gdn2_fwd_tc_kernel" if path == "tc"
                       else "gdn2_fwd_simt_kernel"),
            "achieved": achieved,
            "peak": hbm,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6650 GB/s",
            "unit": "GB/s",
            "frac": achieved / hbm,
            "traffic": traffic,
            "algorithmic_bytes_per_launch": fb,
            "launch_ms": fwd_avg_ms,
        },
        "cpu_baseline": cpu,
        "e2e": e2e,
        # state init + decode + forward (the tensor-core forward is two kernels)
        "gpu_launches": (4 if path == "tc" else 3) * args.steps,
        "clocks": clk,
        "decode": dec,
        "forms": forms,
        "configs": configs,
        "gate_proj": gproj,
        "stream": stream_res,
        "backward": bwd,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_decode(args, dev, stream, rank, world):
    import channel_gated_delta_b200 as gd
    import synth
    D = synth.DECODE
    B, H, dk, dv = D["B"], D["H"], D["dk"], D["dv"]
    gen = torch.Generator(device="cpu").manual_seed(5 + rank)
    S = (torch.randn(B, H, dk, dv, generator=gen) * 0.05).to(dev)
    gamma = synth.decode_gamma().to(dev)
    pool = [{k: v.to(dev) for k, v in synth.decode_step_inputs(i, B=B, H=H, dk=dk, dv=dv).items()}
            for i in range(8)]
    y = torch.empty(B, H, dv, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    # Written, the flush buffer would leave up to the whole L2 dirty, and its
    # write-back would land in the next timed step; reading a second buffer
    # larger than L2 afterwards writes those lines back before the step.
    flush_read = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    def one(i):
        t = pool[i % len(pool)]
        gd.gdelta_decode_step(t["q"], t["k"], t["v"], t["b"], t["w"], t["z"], t["g"], t["log_alpha"],
                              S, gamma_stat=gamma, y=y, stream=stream)

    for i in range(5):
        one(i)
    n = args.decode_steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    barrier(world)
    for i in range(n):
        flush.zero_()                                   # evict the state from L2 (untimed)
        flush_read.sum()                                # and leave L2 clean (untimed)
        evs[i][0].record(stream)
        one(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = sorted(a.elapsed_time(b) for a, b in evs)
    med = max_over_ranks(statistics.median(ms), world)
    mean = max_over_ranks(sum(ms) / n, world)
    nb = decode_bytes(B, H, dk, dv, 2)
    hbm, kind = peaks()
    gbs = nb / (med * 1e-3) / 1e9
    return {
        "workload": f"decode B{B} H{H} dk=dv={dk}, fp32 state {B * H * dk * dv * 4 / 1e6:.1f} MB, bf16 tokens",
        "value": gbs * world,
        "unit": "GB/s",
        "per_gpu_gbs": gbs,
        "steps_per_s": 1e3 / med,
        "tokens_per_s": B * world * 1e3 / med,
        "ms_per_step_median": med,
        "ms_per_step_mean": mean,
        "timed_steps": n,
        "bytes_per_step": nb,
        "roofline": {"bound": "hbm", "kernel": "gdn2_decode_kernel", "achieved": gbs, "peak": hbm,
                     "unit": "GB/s", "frac": gbs / hbm,
                     "traffic": recorded_traffic("channel_gated_delta_b200/csrc/decode.cu")},
        "l2": "between timed steps a 256 MB buffer is written (state evicted), then a second 256 MB "
              "buffer is read (the first buffer's dirty lines written back before the step)",
        "state_init": "random N(0, 0.05^2) state (timing does not depend on values)",
    }


FORMS = {
    # Muir readout with the static profile only (no dynamic z)
    "static_gain": dict(z=False, beta=False, decay_tok=False),
    # KDA: one beta for erase and write, per-channel decay
    "kda": dict(z=True, beta=True, decay_tok=False),
    # Gated DeltaNet: one beta and one scalar decay per token, no z
    "gdn": dict(z=False, beta=True, decay_tok=True),
    # per-channel gates on pre-activation q and k: SiLU and l2 norm in the kernels
    "raw_qk": dict(z=True, beta=False, decay_tok=False, qk_raw=True),
}


def run_forms(args, gd, d, shape, dev, stream, ws, world):
    """Times gdelta_fwd_chunked alone on each reduced gate form, inputs made
    from the workload's tensors (beta = channel 0 of w, the scalar log-decay =
    channel 0 of log_alpha).  Inputs stay larger than L2 for every form."""
    B, T, H, dk, dv, C = shape.B, shape.T, shape.H, shape.dk, shape.dv, shape.chunk
    S = torch.empty(B, H, dk, dv, device=dev)
    y = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=dev)
    hbm, _ = peaks()
    out = {}
    for name, f in FORMS.items():
        z = d["z"] if f["z"] else None
        beta = d["w"][..., 0].contiguous() if f["beta"] else None
        b, w = (None, None) if f["beta"] else (d["b"], d["w"])
        la = d["log_alpha"][..., 0].contiguous() if f["decay_tok"] else d["log_alpha"]
        raw = f.get("qk_raw", False)

        def call():
            gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], b, w, z, d["g"], la, gamma_stat=d["gamma_stat"],
                                  S_in=S, S_out=S, y=y, chunk=C, path=args.path, workspace=ws,
                                  stream=stream, beta=beta, decay_per_token=f["decay_tok"], qk_raw=raw)

        for _ in range(5):
            gd.gdelta_state_init(S, stream=stream)
            call()
        torch.cuda.synchronize(dev)
        if gd.gdelta_get_last_device_error(stream) != 0:
            raise RuntimeError(f"device status word set during the {name} warm-up")
        n = max(20, args.steps)                              # median of at least 20 calls
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        barrier(world)
        for i in range(n):
            gd.gdelta_state_init(S, stream=stream)
            evs[i][0].record(stream)
            call()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(statistics.median(a.elapsed_time(c) for a, c in evs), world)
        nb = fwd_bytes(B, T, H, dk, dv, 2, z=f["z"], beta=f["beta"], decay_tok=f["decay_tok"])
        gbs = nb / (ms * 1e-3) / 1e9
        out[name] = {"fwd_ms_median": ms, "tokens_per_s": B * T * world / (ms * 1e-3),
                     "algorithmic_bytes": nb, "achieved_gbs": gbs, "frac": gbs / hbm, "timed_calls": n}
        if raw:
            # for comparison: the same preprocessing as separate PyTorch ops, then the plain forward
            import torch.nn.functional as F
            qn = torch.empty_like(d["q"])
            kn = torch.empty_like(d["k"])
            ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            for i in range(n):
                gd.gdelta_state_init(S, stream=stream)
                ev2[i][0].record(stream)
                with torch.cuda.stream(stream):
                    qn.copy_(F.normalize(F.silu(d["q"].float()), dim=-1))
                    kn.copy_(F.normalize(F.silu(d["k"].float()), dim=-1))
                gd.gdelta_fwd_chunked(qn, kn, d["v"], b, w, z, d["g"], la, gamma_stat=d["gamma_stat"],
                                      S_in=S, S_out=S, y=y, chunk=C, path=args.path, workspace=ws,
                                      stream=stream)
                ev2[i][1].record(stream)
            torch.cuda.synchronize(dev)
            out[name]["torch_preprocess_then_fwd_ms_median"] = max_over_ranks(
                statistics.median(a.elapsed_time(c) for a, c in ev2), world)
    return out


OTHER_CONFIGS = ("layer350m_bf16", "long32k_bf16")


def run_configs(args, gd, dev, stream, rank, world):
    """gdelta_fwd_chunked alone on the 350M-scale layer (B8 T4096 H8) and the
    32768-token sequence (B1 T32768 H16), each with its own inputs from
    ``synth`` (the generators of the parity tests), CUDA events around every
    call.  Inputs are larger than L2 in both, so no flush."""
    import synth
    hbm, kind = peaks()
    out = {}
    for name in OTHER_CONFIGS:
        shape = synth.CONFIGS[name]
        B, T, H, dk, dv, C = shape.B, shape.T, shape.H, shape.dk, shape.dv, shape.chunk
        host = synth.generate(shape, seed=shape.seed + 1000 * rank)
        d = {k: v.to(dev) for k, v in host.items()}
        del host
        S = torch.empty(B, H, dk, dv, device=dev)
        y = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=dev)
        nws = gd.gdelta_fwd_workspace_bytes(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                            d["log_alpha"], chunk=C, path=args.path)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)

        def call():
            gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                                  gamma_stat=d["gamma_stat"], S_in=None, S_out=S, y=y, chunk=C,
                                  path=args.path, workspace=ws, stream=stream)

        for _ in range(5):
            call()
        torch.cuda.synchronize(dev)
        if gd.gdelta_get_last_device_error(stream) != 0:
            raise RuntimeError(f"device status word set during the {name} warm-up")
        n = max(20, min(args.steps, 40))                     # median of at least 20 calls
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        barrier(world)
        for a, c in evs:
            a.record(stream)
            call()
            c.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(statistics.median(a.elapsed_time(c) for a, c in evs), world)
        nb = fwd_bytes(B, T, H, dk, dv, 2)
        gbs = nb / (ms * 1e-3) / 1e9
        out[name] = {
            "workload": f"{name}: B{B} T{T} H{H} dk=dv={dk} chunk {C}, bf16 tokens, fp32 log-decay and state, "
                        "S_in = 0",
            "fwd_ms_median": ms, "tokens_per_s": B * T * world / (ms * 1e-3), "timed_calls": n,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_source": kind, "algorithmic_bytes_per_launch": nb, "launch_ms": ms},
            "l2": "inputs larger than the 126 MB L2; no flush",
        }
        if B == 1 and T >= 16384 and T % (4 * C) == 0:
            out[name]["segment_scan"] = run_segment_scan(gd, d, shape, y, dev, stream, world, args, 4)
        del d, S, y, ws
        torch.cuda.empty_cache()
    return out


def run_segment_scan(gd, d, shape, y_direct, dev, stream, world, args, P):
    """One sequence (B = 1) as P segments on one GPU: the segments' affine state
    maps (gdelta_segment_map: two forward calls over the P segments as batch
    rows), their composition into each segment's starting state
    (gdelta_state_affine), and the forward over the segments from those states.
    Timed against the direct call above; y compared with it."""
    T, H, dk, dv, C = shape.T, shape.H, shape.dk, shape.dv, shape.chunk
    Ts = T // P
    seg = {k: d[k].view(P, Ts, *d[k].shape[2:]) for k in ("q", "k", "v", "b", "w", "z", "g", "log_alpha")}
    S_start = torch.zeros(P, H, dk, dv, device=dev)
    S_end = torch.empty(P, H, dk, dv, device=dev)
    ys = torch.empty(P, Ts, H, dv, dtype=torch.bfloat16, device=dev)

    def call():
        A, D = gd.gdelta_segment_map(seg["q"], seg["k"], seg["v"], seg["b"], seg["w"], seg["z"], seg["g"],
                                     seg["log_alpha"], chunk=C, path=args.path, stream=stream)
        for j in range(1, P):
            gd.gdelta_state_affine(A[j - 1:j], S_start[j - 1:j], D[j - 1:j], S_out=S_start[j:j + 1], stream=stream)
        gd.gdelta_fwd_chunked(seg["q"], seg["k"], seg["v"], seg["b"], seg["w"], seg["z"], seg["g"],
                              seg["log_alpha"], gamma_stat=d["gamma_stat"], S_in=S_start, S_out=S_end, y=ys,
                              chunk=C, path=args.path, stream=stream)

    for _ in range(2):
        call()
    torch.cuda.synchronize(dev)
    if gd.gdelta_get_last_device_error(stream) != 0:
        raise RuntimeError("device status word set during the segment scan")
    n = max(3, min(args.steps, 5))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    barrier(world)
    for a, c in evs:
        a.record(stream)
        call()
        c.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(statistics.median(a.elapsed_time(c) for a, c in evs), world)
    ref = y_direct.float().view(-1)
    diff = float((ys.float().view(-1) - ref).abs().max() / ref.pow(2).mean().sqrt())
    return {"segments": P, "ms_median": ms, "tokens_per_s": T * world / (ms * 1e-3),
            "y_max_abs_diff_over_rms_vs_direct": diff,
            "note": "three forward calls over T/P tokens in P rows (the map's two, then the final one) "
                    "against the direct call's one over T: on one GPU the chain already has 128 CTAs' "
                    "worth of work at P = 4"}


def run_gate_proj(args, gd, shape, dev, stream, rank, world):
    """gdelta_gate_proj on the Muir 1.34B-scale layer's tokens: N = B*T rows of
    d = H*128, ranks (64, 64, 128, 128, 128), synthetic weights.  Algorithmic
    bytes: x and the weights read once, the five gates written once (four bf16,
    log-decay fp32); FLOPs 4 N d R."""
    import synth
    B, T, H, dk = shape.B, shape.T, shape.H, shape.dk
    N, d = B * T, H * dk
    ranks = synth.GATE_RANKS
    R = sum(ranks)
    inp = {k: v.to(dev) for k, v in synth.gate_proj_inputs(N, d, seed=4 + rank).items()}
    out = {"log_alpha": torch.empty(N, d, device=dev)}
    out.update({n: torch.empty(N, d, dtype=torch.bfloat16, device=dev) for n in ("b", "g", "w", "z")})
    ws = torch.empty(N * 2 * R * 2 + 256, dtype=torch.uint8, device=dev)     # the codes as two bf16 parts

    def call():
        gd.gdelta_gate_proj(inp["x"], inp["w_down"], inp["w_up"], inp["bias"], ranks=ranks, out=out,
                            workspace=ws, stream=stream)

    for _ in range(5):
        call()
    torch.cuda.synchronize(dev)
    if gd.gdelta_get_last_device_error(stream) != 0:
        raise RuntimeError("device status word set during the gate projection warm-up")
    n = max(20, min(args.steps, 40))                         # median of at least 20 calls
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    barrier(world)
    for a, c in evs:
        a.record(stream)
        call()
        c.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(statistics.median(a.elapsed_time(c) for a, c in evs), world)
    nbytes = N * d * 2 + 2 * d * R * 2 + 5 * d * 4 + N * d * (4 * 2 + 4)
    flops = 4.0 * N * d * R
    hbm, kind = peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {
        "workload": f"x [{N}, {d}] bf16 (the B{B} T{T} H{H} layer's tokens), ranks {list(ranks)}, synthetic weights",
        "kernel": "gate_proj_kernel (down: codes = x w_down; up: five grouped products, bias, activations)",
        "ms_median": ms, "tokens_per_s": N * world / (ms * 1e-3), "timed_calls": n,
        "algorithmic_bytes": nbytes, "flops": flops, "tflops": flops / (ms * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_source": kind,
                     "traffic": recorded_traffic("channel_gated_delta_b200/csrc/gate_proj.cu"),
                     "note": "4 N d R flops at the measured bf16 peak would take less time than the bytes"},
    }


def bwd_bytes(B, T, H, dk, dv, tok_bytes):
    """Algorithmic HBM bytes of one backward call: the forward's inputs (q, k,
    z, b, v, w, g, log_alpha) and dL/dy read once, the eight fp32 token
    gradients written, the states S_in and dL/dS_out read and dL/dS_in written."""
    per = 4 * dk * tok_bytes + 3 * dv * tok_bytes + 4 * dk + 4 * dv + 4 * (5 * dk + 3 * dv)
    return B * T * H * per + 3 * B * H * dk * dv * 4 + 2 * H * dk * 4


def run_bwd(args, gd, d, shape, dev, stream, world):
    """gdelta_bwd on the workload (dL/dy random, dL/dS_T zero), CUDA events."""
    B, T, H, dk, dv = shape.B, shape.T, shape.H, shape.dk, shape.dv
    gen = torch.Generator(device="cpu").manual_seed(13)
    dy = torch.randn(B, T, H, dv, generator=gen).to(dev)
    S0 = torch.zeros(B, H, dk, dv, device=dev)

    def call():
        # outputs and workspace come from torch's caching allocator (no cudaMalloc after the warm-up)
        return gd.gdelta_bwd(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], dy,
                             gamma_stat=d["gamma_stat"], S_in=S0, stream=stream)

    call()                                                # warm-up
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.bwd_calls)]
    barrier(world)
    for a, c in evs:
        a.record(stream)
        call()
        c.record(stream)
    torch.cuda.synchronize(dev)
    if gd.gdelta_get_last_device_error(stream) != 0:
        raise RuntimeError("device status word set during the backward")
    ms = max_over_ranks(statistics.median(a.elapsed_time(c) for a, c in evs), world)
    nb = bwd_bytes(B, T, H, dk, dv, 2)
    hbm, _ = peaks()
    gbs = nb / (ms * 1e-3) / 1e9
    return {"kernel": "gdn2_bwd_kernel (+ gdn2_bwd_dgamma_kernel)", "ms_per_call": ms,
            "tokens_per_s": B * T * world / (ms * 1e-3), "algorithmic_bytes": nb,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm},
            "timed_calls": args.bwd_calls,
            "note": f"a two-CTA cluster per head (value halves) walks the tokens in order: latency-bound, {2 * B * H} CTAs"}


def run_stream(args, gd, d, shape, dev, stream, world, decode_steps=256):
    """One sequence served for ``args.stream_tokens`` tokens: the workload's
    [B,T,H,d] tensors read as one [1, B*T, H, d] segment (B-major layout makes
    that a view), forward calls over that segment repeated with the state
    carried in place, then single-token decode steps on the same state."""
    import synth
    B, T, H, dk, dv, C = shape.B, shape.T, shape.H, shape.dk, shape.dv, shape.chunk
    seg = B * T
    v1 = {k: (t.view(1, seg, H, t.shape[-1]) if t.dim() == 4 else t) for k, t in d.items()}
    S = torch.zeros(1, H, dk, dv, device=dev)
    y = torch.empty(1, seg, H, dv, dtype=torch.bfloat16, device=dev)
    ws_bytes = gd.gdelta_fwd_workspace_bytes(v1["q"], v1["k"], v1["v"], v1["b"], v1["w"], v1["z"], v1["g"],
                                             v1["log_alpha"], chunk=C, path=args.path)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    n_calls = max(1, -(-args.stream_tokens // seg))
    dec = [{k: t.to(dev) for k, t in synth.decode_step_inputs(i, seed=91, B=1, H=H, dk=dk, dv=dv).items()}
           for i in range(4)]
    y1 = torch.empty(1, H, dv, dtype=torch.bfloat16, device=dev)

    def call():
        gd.gdelta_fwd_chunked(v1["q"], v1["k"], v1["v"], v1["b"], v1["w"], v1["z"], v1["g"], v1["log_alpha"],
                              gamma_stat=d["gamma_stat"], S_in=S, S_out=S, y=y, chunk=C, path=args.path,
                              workspace=ws, stream=stream)

    def step(i):
        t = dec[i % len(dec)]
        gd.gdelta_decode_step(t["q"], t["k"], t["v"], t["b"], t["w"], t["z"], t["g"], t["log_alpha"], S,
                              gamma_stat=d["gamma_stat"], y=y1, stream=stream)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    S.zero_()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    barrier(world)
    ev[0].record(stream)
    for _ in range(n_calls):
        call()
    ev[1].record(stream)
    for i in range(decode_steps):
        step(i)
    ev[2].record(stream)
    torch.cuda.synchronize(dev)
    if gd.gdelta_get_last_device_error(stream) != 0:
        raise RuntimeError("device status word set during the stream")
    pre_ms = max_over_ranks(ev[0].elapsed_time(ev[1]), world)
    dec_ms = max_over_ranks(ev[1].elapsed_time(ev[2]), world)

    # the pieces a rank of a sequence-sharded forward adds: the segment map
    # (two forward calls) and one affine composition of the state
    A, D = gd.gdelta_segment_map(v1["q"], v1["k"], v1["v"], v1["b"], v1["w"], v1["z"], v1["g"], v1["log_alpha"],
                                 chunk=C, path=args.path, stream=stream)
    S2 = torch.empty_like(S)
    sm = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    sm[0].record(stream)
    gd.gdelta_segment_map(v1["q"], v1["k"], v1["v"], v1["b"], v1["w"], v1["z"], v1["g"], v1["log_alpha"],
                          chunk=C, path=args.path, stream=stream)
    sm[1].record(stream)
    gd.gdelta_state_affine(A, S_in=S, D=D, S_out=S2, stream=stream)
    sm[2].record(stream)
    torch.cuda.synchronize(dev)
    map_ms = max_over_ranks(sm[0].elapsed_time(sm[1]), world)
    aff_ms = max_over_ranks(sm[1].elapsed_time(sm[2]), world)
    return {
        "workload": f"one stream per GPU, B1 H{H} dk=dv={dk}: {n_calls * seg} tokens in {n_calls} forward calls "
                    f"of {seg} tokens (the workload's tensors read as one sequence, repeated), state carried "
                    f"in place, then {decode_steps} decode steps",
        "tokens": n_calls * seg,
        "prefill_tokens_per_s": n_calls * seg * world / (pre_ms * 1e-3),
        "prefill_ms_per_call": pre_ms / n_calls,
        "decode_us_per_step": dec_ms * 1e3 / decode_steps,
        "segment_map_ms": map_ms,
        "state_affine_us": aff_ms * 1e3,
        "state_bytes": H * dk * dv * 4,
        "finite": bool(torch.isfinite(S).all().item()),
    }


def run_e2e(args, gd, host, dev, stream, shape, world, path):
    """Same step through the public API, inputs copied from pinned host memory
    every step and y / S read back, all inside the timed region.  Steps are
    pipelined as a streaming user would run them: inputs and outputs are
    double-buffered on the device, the copies in, the compute and the copies
    out run on three streams ordered by events, so step i's results go back
    over PCIe while step i+1's inputs come in.  The timed region runs from the
    first copy in to the last copy out."""
    B, T, H, dk, dv, C = shape.B, shape.T, shape.H, shape.dk, shape.dv, shape.chunk
    keys = ("q", "k", "v", "b", "w", "z", "g", "log_alpha", "gamma_stat")
    hp = {k: host[k].pin_memory() for k in keys}
    dd = [{k: torch.empty_like(host[k], device=dev) for k in keys} for _ in range(2)]
    S = [torch.empty(B, H, dk, dv, device=dev) for _ in range(2)]
    y = [torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    y_h = [torch.empty(B, T, H, dv, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    S_h = [torch.empty(B, H, dk, dv).pin_memory() for _ in range(2)]
    ws_bytes = gd.gdelta_fwd_workspace_bytes(dd[0]["q"], dd[0]["k"], dd[0]["v"], dd[0]["b"], dd[0]["w"],
                                             dd[0]["z"], dd[0]["g"], dd[0]["log_alpha"], chunk=C, path=args.path)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    h2d = sum(hp[k].numel() * hp[k].element_size() for k in keys)
    d2h = y_h[0].numel() * 2 + S_h[0].numel() * 4
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(i):
        x = i % 2
        if used[x]:
            s_in.wait_event(comp_done[x])                     # the forward of step i-2 has read dd[x]
        with torch.cuda.stream(s_in):
            for k in keys:
                dd[x][k].copy_(hp[k], non_blocking=True)
        in_done[x].record(s_in)
        stream.wait_event(in_done[x])
        if used[x]:
            stream.wait_event(out_done[x])                    # y[x], S[x] of step i-2 have been read back
        gd.gdelta_state_init(S[x], stream=stream)
        gd.gdelta_fwd_chunked(dd[x]["q"], dd[x]["k"], dd[x]["v"], dd[x]["b"], dd[x]["w"], dd[x]["z"],
                              dd[x]["g"], dd[x]["log_alpha"], gamma_stat=dd[x]["gamma_stat"], S_in=S[x],
                              S_out=S[x], y=y[x], chunk=C, path=args.path, workspace=ws, stream=stream)
        comp_done[x].record(stream)
        s_out.wait_event(comp_done[x])
        with torch.cuda.stream(s_out):
            y_h[x].copy_(y[x], non_blocking=True)
            S_h[x].copy_(S[x], non_blocking=True)
        out_done[x].record(s_out)
        used[x] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(2, min(args.steps, 6))
    barrier(world)
    a.record(s_in)
    for i in range(n):
        step(i)
    b.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(a.elapsed_time(b) / n, world)
    return {"value": B * T * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "api": "channel_gated_delta_b200.gdelta_state_init + gdelta_fwd_chunked (pinned host copies; "
                   "copies in, compute and copies out on three streams, device buffers doubled)"}


# ---------------------------------------------------------------- oracle arm

def cpu_baseline(host, shape, heads=None):
    """The float64 oracle as it stands, on this host's cores."""
    import oracle
    H, T = shape.H, shape.T
    heads = heads if heads is not None else [(b, h) for b in range(shape.B) for h in range(H)]
    sub = {k: v for k, v in host.items()}
    t0 = time.perf_counter()
    r = oracle.forward(sub, heads=heads)
    dt = time.perf_counter() - t0
    token_heads = len(heads) * T
    return {"value": token_heads / H / dt, "unit": "tokens/s", "cores": r["threads"], "kind": "oracle",
            "sample": f"{len(heads)} of {shape.B * H} heads x {T} tokens of the same workload "
                      f"({token_heads} token-heads; tokens/s = token-heads/s / H), float64 C recurrence",
            "seconds": dt}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import synth
    shape = synth.CONFIGS[WORKLOAD]
    host = synth.generate(shape)
    heads = [(0, h) for h in range(4)]
    T = 1024
    sub = {k: (v[:, :T] if v.dim() == 4 else v) for k, v in host.items()}
    import oracle
    for _ in range(args.warmup):
        oracle.forward(sub, heads=heads)
    t0 = time.perf_counter()
    threads = 0
    for _ in range(args.steps):
        threads = oracle.forward(sub, heads=heads)["threads"]
    dt = (time.perf_counter() - t0) / args.steps
    value = len(heads) * T / shape.H / dt
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: B4 T4096 H16 dk=dv=128 chunk 64 (bounded sample per step)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: {len(heads)} heads x {T} tokens of the workload, "
                                   "float64 C recurrence on the host cores"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, local, world = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            if not torch.cuda.is_available():
                raise RuntimeError("bench.py --impl ours needs a CUDA device")
            run_ours(args, rank, local, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
