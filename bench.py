#!/usr/bin/env python
"""GDN forward benchmark on B200: tokens/s per layer on the minute-scale SANA-WM layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload minute|block|clip241|sessions]

Default workload (minute): B = 1, H = 20, d_k = d_v = 112, T = 106,480 tokens
(121 latent frames of 880 tokens), chunk 64, bf16 q/k/v/out, float32 logits and
state, seeded synthetic inputs; one step = 20 layer calls back to back (one
buffer set of 1.9 GB, larger than the 126 MB L2, so no call finds its inputs in
L2).  The other workloads: block (one 3-frame streaming block, T = 2,640, state
in and out; 20 calls per step rotating over 8 buffer sets, 396 MB in all, so
that no call finds its inputs in L2), clip241 (T = 27,280, zero initial state,
20 layers per step) and sessions (4 independent sessions, 40 successive
3-frame blocks per step through gdn_state_step with the state carried in
place; every block its own inputs, 7.9 GB in all).

Multi-GPU: one process per GPU (torchrun); the layer's (batch, head) chains are
independent, so every rank runs the same per-GPU workload with no collective
on the data path ("weak" scaling); the step time is the max over ranks.

Prints ONE JSON line from rank 0.  ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload instead (rank 0 only).
"""

import argparse
import datetime
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN fwd tokens/s per layer (20 heads x d112) on 1 B200; % of roofline"
UNIT = "tokens/s"
BYTES_PER_TOKEN_HEAD = 900          # q, k, v in + out (bf16, d = 112) + beta logit (f32)
CHUNKED_FLOPS_PER_TOKEN_HEAD = 146944   # 10 C d + 6 d^2 at C = 64, d = 112
KERNEL_SOURCES = ["hybrid_linear_attention_frame_b200/csrc/gdn_seq.cu",
                  "hybrid_linear_attention_frame_b200/csrc/gdn_ring.cu",
                  "hybrid_linear_attention_frame_b200/csrc/gdn_tc.cu",
                  "hybrid_linear_attention_frame_b200/csrc/gdn_ffma.cu",
                  "hybrid_linear_attention_frame_b200/csrc/gdn_common.cuh",
                  "hybrid_linear_attention_frame_b200/csrc/gdn_sm100.cuh"]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=None, help="layer calls per step (default 20)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target wall time of the oracle sample")
    ap.add_argument("--profile-tokens", type=int, default=0,
                    help="profiling case: two layer calls on the layer's first T tokens, no timing")
    ap.add_argument("--gate-mode", choices=["token", "frame"], default="token",
                    help="token: a frame's gate at each of its tokens (gdn_forward*); frame: once, at "
                         "the frame's first token (gdn_forward_gated, gate_mode 1)")
    ap.add_argument("--path", choices=["ws", "plain"], default="plain",
                    help="plain: gdn_forward / gdn_state_step (sequence-parallel kernel, no workspace); "
                         "ws: gdn_forward_ws / gdn_state_step_ws (shared prep through a workspace ring)")
    ap.add_argument("--workload", choices=["minute", "block", "clip241", "sessions"], default="minute",
                    help="minute: the minute-scale layer (default); block: one streaming block with state in "
                         "and out; clip241: the 241-frame clip layer; sessions: 4 sessions x 40 blocks "
                         "through gdn_state_step")
    ap.add_argument("--layer", choices=["gdn", "softmax"], default="gdn",
                    help="gdn: the GDN layer; softmax: the chunk-causal softmax attention layer "
                         "(gdn_softmax_attention, blocks of 3 frames, 2 cached blocks, 1 sink frame)")
    ap.add_argument("--direction", choices=["causal", "bidir"], default="causal",
                    help="causal: the forward scan; bidir: gdn_forward_bidir (forward plus backward "
                         "scan from zero states, the dense checkpoint's form)")
    ap.add_argument("--inputs", choices=["bf16", "fp8"], default="bf16",
                    help="bf16: q, k, v in bf16 (gdn_forward); fp8: q, k, v as e4m3 bytes, v with one "
                         "power-of-two scale (gdn_forward_fp8; layer workloads, forward scan)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------
# distributed plumbing (rank setup, barrier, max over ranks)
# ----------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(backend, world, timeout_s=120):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend,
                                timeout=datetime.timedelta(seconds=timeout_s))


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a float over all ranks (every rank gets the result)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_rank: float, elapsed_s_this_rank: float, world: int, device=None):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    slowest = max_over_ranks(elapsed_s_this_rank, world, device)
    return tokens_per_rank * world / slowest, slowest


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """Samples nvidia-smi every 200 ms while the timed region runs."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="gdn_clocks_", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200", "-f", self.path]
            if self.uuid:
                cmd[1:1] = ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 10:
                        rows.append(parts)
            os.unlink(self.path)
        except OSError:
            return None
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "", 1).isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "", 1).isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# roofline bookkeeping
# ----------------------------------------------------------------------------

def algorithmic_bytes(w, state_in: bool, state_out: bool, in_elem: int = 2) -> int:
    """Bytes one gdn_forward call must move at least: q, k, v (in_elem bytes each:
    2 for bf16, 1 for e4m3), out (bf16), the beta logits, the per-frame gate logits
    and the state (float32)."""
    th = w.B * w.T * w.H
    b = th * ((2 * w.d_k + w.d_v) * in_elem + w.d_v * 2 + 4)
    b += w.B * w.n_frames * w.H * 4
    st = w.B * w.H * w.d_k * w.d_v * 4
    return b + (st if state_in else 0) + (st if state_out else 0)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """dram bytes per launch from the committed ncu summary, if the kernel sources
    are the ones it was captured from; otherwise None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None, None
    if rec.get("kernel_source_sha") != kernel_source_sha():
        return None, rec.get("kernel")
    return rec.get("dram_bytes_per_launch"), rec.get("kernel")


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ----------------------------------------------------------------------------

def slice_tokens(inp, n_tok):
    """The first n_tok tokens of every (batch, head) chain, with their frames' gates."""
    from workloads import Inputs
    F = -(-n_tok // inp.frame_len)
    return Inputs(q=inp.q[:, :n_tok], k=inp.k[:, :n_tok], v=inp.v[:, :n_tok],
                  gate=inp.gate[:, :F], beta=inp.beta[:, :n_tok], state=None,
                  io_dtype=inp.io_dtype, frame_len=inp.frame_len)


def oracle_sample_size(inp, seconds, threads):
    """Tokens per chain the oracle processes in about `seconds` (whole frames)."""
    from oracle import gdn_reference as R
    fl = inp.frame_len
    probe = slice_tokens(inp, fl)
    t0 = time.perf_counter()
    R.c_forward(probe, None, n_threads=threads, want_state=False)
    dt = max(time.perf_counter() - t0, 1e-4)
    frames = max(1, min(inp.q.shape[1] // fl, int(seconds / dt)))
    return frames * fl


def time_oracle(inp, n_tok, threads, repeats=1, bidir=False):
    from oracle import gdn_reference as R
    sub = slice_tokens(inp, n_tok)
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        if bidir:
            R.c_bidirectional(sub, n_threads=threads)
        else:
            R.c_forward(sub, None, n_threads=threads, want_state=True)
        times.append(time.perf_counter() - t0)
    return times


def oracle_threads(w):
    return max(1, min(os.cpu_count() or 1, w.B * w.H))


def cpu_baseline(w, inp, seconds, bidir=False):
    threads = oracle_threads(w)
    n_tok = oracle_sample_size(inp, seconds / (2 if bidir else 1), threads)
    (dt,) = time_oracle(inp, n_tok, threads, bidir=bidir)
    form = "forward plus backward token recurrence" if bidir else "token recurrence"
    return {"value": w.B * n_tok / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"float64 C {form}, first {n_tok} tokens of all {w.B * w.H} "
                      f"(batch, head) chains of one layer, {threads} OpenMP threads "
                      f"(host has {os.cpu_count()} cores), {dt:.2f} s"}


def run_reference(args, w, rank, world):
    """Reference arm: the float64 CPU oracle on bounded samples of the same workload
    (the GDN layer, its bidirectional form, or the softmax layer, as the flags say)."""
    if rank != 0:
        return None
    from workloads import make_inputs
    if args.inputs == "fp8":
        from oracle import gdn_reference as R
        from workloads import make_fp8_inputs
        inp = R.widen_fp8(make_fp8_inputs(w))           # the layer's values of the e4m3 inputs
    else:
        inp = make_inputs(w)
    threads = oracle_threads(w)
    budget = 150.0 / max(1, args.steps + args.warmup)      # whole run within a few minutes
    layers = calls_per_step(args, w)
    if args.layer == "softmax":
        per_call = min(args.cpu_seconds, budget)
        for _ in range(args.warmup):
            attention_cpu_baseline(w, inp, per_call)
        runs = [attention_cpu_baseline(w, inp, per_call) for _ in range(args.steps)]
        value = statistics.mean(r["value"] for r in runs)
        per_step = w.B * w.T / value
        sample = runs[-1]["sample"] + " per step"
        metric, config, cores = ATTN_METRIC, attention_config(w, layers), os.cpu_count()
    else:
        bidir = args.direction == "bidir"
        n_tok = oracle_sample_size(inp, min(args.cpu_seconds, budget) / (2 if bidir else 1), threads)
        time_oracle(inp, n_tok, threads, repeats=args.warmup, bidir=bidir)
        times = time_oracle(inp, n_tok, threads, repeats=args.steps, bidir=bidir)
        per_step = sum(times) / len(times)
        value = w.B * n_tok / per_step
        form = "forward plus backward token recurrence" if bidir else "token recurrence"
        sample = (f"float64 C {form}, first {n_tok} tokens of all {w.B * w.H} chains "
                  f"of one layer per step, {threads} OpenMP threads (host has {os.cpu_count()} cores)")
        metric, config, cores = METRIC, run_config(args, w), threads
    return {"metric": metric, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def workload_config(w, layers):
    what = {"minute": "minute-scale SANA-WM GDN layer", "block": "one SANA-WM streaming block (3 latent frames)",
            "clip241": "241-frame clip GDN layer (31 latent frames)",
            "sessions": "batched streaming sessions"}.get(w.name, w.name)
    if w.name == "sessions":
        per_step = (f"{w.blocks} successive blocks of {w.T} tokens per session per step, state carried "
                    "block to block in place")
        l2 = f"every block its own inputs ({w.blocks} sets, 7.9 GB)"
        state = f"initial state N(0, {w.state_std}) per session (seed {w.session_seed_base} + s), carried"
    elif w.name == "block":
        per_step = f"{layers} calls per step over {BLOCK_SETS} buffer sets in rotation"
        l2 = f"{BLOCK_SETS} rotating input sets, 396 MB in all vs the 126 MB L2"
        state = f"state in N(0, {w.state_std}) and out"
    else:
        per_step = f"{layers} layers back-to-back per step"
        l2 = "inputs larger than L2 ({:.2f} GB per layer vs 126 MB)".format(w.B * w.T * w.H * 900 / 1e9)
        state = "zero initial state, final state written"
    return {"workload": f"{w.name}: {what}, B={w.B} H={w.H} T={w.T} d_k=d_v={w.d_k}, frame {w.frame_len} "
                        f"tokens, chunk {w.chunk_len}, {per_step}",
            "B": w.B, "H": w.H, "T": w.T, "d_k": w.d_k, "d_v": w.d_v, "frame_len": w.frame_len,
            "chunk_len": w.chunk_len, "calls_per_step": layers,
            "gate_logits": f"N({w.gate_mean}, {w.gate_std})", "seed": w.seed, "state": state,
            "l2": l2, "parallelism": "weak: every rank runs the full workload on its own GPU"}


BLOCK_SETS = 8


def workload_of(args):
    from workloads import BLOCK, CLIP241, MINUTE, SESSIONS
    return {"minute": MINUTE, "block": BLOCK, "clip241": CLIP241, "sessions": SESSIONS}[args.workload]


def calls_per_step(args, w):
    if w.name == "sessions":
        return w.blocks
    return args.layers or 20


def run_config(args, w):
    """The config object of the JSON line; the same for both arms of one invocation."""
    layers = calls_per_step(args, w)
    bidir = args.direction == "bidir"
    gate_mode = args.gate_mode == "frame"
    stream_step = w.name == "sessions"
    if bidir:
        api = "gdn_forward_bidir (C ABI, device buffers, caller workspace reused by every layer)"
    elif gate_mode:
        api = "gdn_forward_gated" + (" with a workspace" if args.path == "ws" else "") + " (C ABI, device buffers)"
    elif stream_step:
        api = ("gdn_state_step_ws (C ABI, device buffers, caller workspace)" if args.path == "ws"
               else "gdn_state_step (C ABI, device buffers, state in place)")
    elif args.inputs == "fp8":
        api = "gdn_forward_fp8 (C ABI, device buffers, no workspace)"
    else:
        api = ("gdn_forward_ws (C ABI, device buffers, caller workspace reused by every layer)"
               if args.path == "ws" else "gdn_forward (C ABI, device buffers, no workspace)")
    cfg = dict(workload_config(w, layers),
               direction=("forward plus backward scan (gdn_forward_bidir)" if bidir else "forward scan"),
               gate_placement=("once per frame, at its first token (gate_mode 1)" if gate_mode
                               else "at every token of the frame"),
               api=api,
               inputs=("q, k, v as e4m3 bytes (round to nearest even from the float32 draws), v with "
                       "one power-of-two scale; out bf16" if args.inputs == "fp8" else "q, k, v, out bf16"))
    return cfg


# ----------------------------------------------------------------------------
# softmax attention layer
# ----------------------------------------------------------------------------

ATTN_GEOMETRY = {"frames_per_block": 3, "cached_blocks": 2, "sink_frames": 1}


def attention_flops(w) -> int:
    """2 (d_k + d_v) flops per (query, visible key) pair: the QK^T and PV products.
    A query of block b sees the sink frames and blocks max(0, b - cached) .. b."""
    bl = ATTN_GEOMETRY["frames_per_block"] * w.frame_len
    sink = min(w.T, ATTN_GEOMETRY["sink_frames"] * w.frame_len)
    pairs = 0
    for b in range(-(-w.T // bl)):
        lo, hi = max(0, b - ATTN_GEOMETRY["cached_blocks"]) * bl, min(w.T, (b + 1) * bl)
        keys = hi if lo <= sink else sink + hi - lo
        pairs += (hi - b * bl) * keys
    return 2 * (w.d_k + w.d_v) * pairs * w.B * w.H


ATTN_METRIC = ("softmax attention tokens/s per layer (20 heads x d112, chunk-causal with KV cache) "
               "on 1 B200; % of roofline")


def attention_config(w, layers):
    cfg = workload_config(w, layers)
    cfg["workload"] = (f"{w.name}: minute-scale SANA-WM softmax attention layer, B={w.B} H={w.H} T={w.T} "
                       f"d_k=d_v={w.d_k}, blocks of 3 frames of {w.frame_len} tokens, 2 cached blocks, "
                       f"1 sink frame, {layers} layers back-to-back per step")
    cfg.update(ATTN_GEOMETRY)
    cfg["api"] = "gdn_softmax_attention (C ABI, device buffers)"
    for key in ("chunk_len", "gate_logits"):
        cfg.pop(key, None)
    return cfg


def attention_cpu_baseline(w, inp, seconds):
    """The float64 oracle on one full query block of the layer (a bounded sample)."""
    from oracle import attention_reference as A
    bl = ATTN_GEOMETRY["frames_per_block"] * w.frame_len
    b = min(-(-w.T // bl) - 1, 3)                   # a block with the full window (2 cached + sink)
    t0 = time.perf_counter()
    A.attention_block(inp.q[:, :, :1], inp.k[:, :, :1], inp.v[:, :, :1], b, w.frame_len,
                      ATTN_GEOMETRY["frames_per_block"], ATTN_GEOMETRY["cached_blocks"],
                      ATTN_GEOMETRY["sink_frames"])
    per_head = max(time.perf_counter() - t0, 1e-3)
    heads = max(1, min(w.H, int(seconds / per_head)))
    t0 = time.perf_counter()
    A.attention_block(inp.q[:, :, :heads], inp.k[:, :, :heads], inp.v[:, :, :heads], b, w.frame_len,
                      ATTN_GEOMETRY["frames_per_block"], ATTN_GEOMETRY["cached_blocks"],
                      ATTN_GEOMETRY["sink_frames"])
    dt = time.perf_counter() - t0
    nq = min(w.T, (b + 1) * bl) - b * bl
    return {"value": w.B * nq * heads / w.H / dt, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"float64 numpy/BLAS softmax over the visible keys, query block {b} ({nq} queries) of "
                      f"{heads} of {w.H} heads, scaled to the layer's heads, {dt:.2f} s"}


def run_softmax(args, w, rank, world, local):
    import numpy as np
    import torch
    import hybrid_linear_attention_frame_b200 as G
    from workloads import bf16_bits, make_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init("nccl", world)
    layers = args.layers or w.layers
    lib = G.load()
    inp = make_inputs(w)

    def bf16(x):
        return torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(device)
    q, k, v = bf16(inp.q), bf16(inp.k), bf16(inp.v)
    out = torch.empty_like(v)
    stream = torch.cuda.current_stream(device)
    sptr = stream.cuda_stream
    geo = (w.frame_len, ATTN_GEOMETRY["frames_per_block"], ATTN_GEOMETRY["cached_blocks"],
           ATTN_GEOMETRY["sink_frames"])

    def layer_call():
        st = lib.gdn_softmax_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.B, w.H, w.T,
                                       w.d_k, w.d_v, *geo, sptr)
        if st != 0:
            raise G.GdnError(st, "gdn_softmax_attention")

    for _ in range(args.warmup):
        for _ in range(layers):
            layer_call()
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps * layers)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        uuid = None
    clocks = ClockSampler(uuid).start() if rank == 0 else None
    barrier(world, device)
    torch.cuda.synchronize(device)
    t_start.record(stream)
    i = 0
    for _ in range(args.steps):
        for _ in range(layers):
            ev[i][0].record(stream)
            layer_call()
            ev[i][1].record(stream)
            i += 1
    t_end.record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    clock_rec = clocks.stop() if clocks else None
    dev_status = G.gdn_get_last_device_status()
    if dev_status != G.GDN_OK:
        raise G.GdnError(dev_status, "device status after the timed region")

    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    value, slowest = aggregate_throughput(w.B * w.T * layers * args.steps, elapsed_s, world, device)
    avg_launch_s = statistics.mean(s_.elapsed_time(e_) for (s_, e_) in ev) / 1e3
    peaks, peak_kind = measured_peaks()
    flops = attention_flops(w)
    achieved = flops / avg_launch_s / 1e12
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": None, "kernel": "chunk_attn_kernel",
                "peak_source": f"{peak_kind} bf16_tflops_sustained (cuBLAS bf16 GEMM, seconds-long loop)",
                "algorithmic_flops_per_launch": flops, "avg_launch_us": round(avg_launch_s * 1e6, 2),
                "frac_of_burst_peak": round(achieved / peaks["bf16_tflops"], 4)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = attention_cpu_baseline(w, inp, args.cpu_seconds)
    cfg = attention_config(w, layers)
    line = {"metric": ATTN_METRIC,
            "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(slowest * 1e3 / args.steps, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": None, "gpu_launches": args.steps * layers, "clocks": clock_rec}
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    return line if rank == 0 else None


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def upload_sets(w, device, fp8=False):
    """Host (pinned later for e2e) and device copies of the workload's input sets.

    Returns a list of dicts with host tensors h_q, h_k, h_v, h_g, h_b, h_s (state or
    None) and their device copies q, k, v, g, b, s."""
    import numpy as np
    import torch
    from workloads import bf16_bits, make_inputs, make_session_blocks

    def bf16(x):
        return torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16)

    if fp8:
        from workloads import make_fp8_inputs
        n = BLOCK_SETS if w.name == "block" else 1
        sets = []
        x8s = [make_fp8_inputs(w, seed=w.seed + i) for i in range(n)]
        for x8 in x8s:
            h = {"h_q": torch.from_numpy(x8.q8), "h_k": torch.from_numpy(x8.k8), "h_v": torch.from_numpy(x8.v8),
                 "h_g": torch.from_numpy(np.ascontiguousarray(x8.gate)),
                 "h_b": torch.from_numpy(np.ascontiguousarray(x8.beta)),
                 "h_s": None if x8.state is None else torch.from_numpy(np.ascontiguousarray(x8.state, np.float32)),
                 "v_scale": x8.v_scale}
            for key in ("q", "k", "v", "g", "b", "s"):
                h[key] = None if h["h_" + key] is None else h["h_" + key].to(device)
            sets.append(h)
        return sets, x8s[0]
    if w.name == "sessions":
        state0, blocks = make_session_blocks(w)
        inps = blocks
        states = [state0] + [None] * (len(blocks) - 1)
    else:
        n = BLOCK_SETS if w.name == "block" else 1
        inps = [make_inputs(w, seed=w.seed + i) for i in range(n)]
        states = [x.state for x in inps]
    sets = []
    for inp, st in zip(inps, states):
        h = {"h_q": bf16(inp.q), "h_k": bf16(inp.k), "h_v": bf16(inp.v),
             "h_g": torch.from_numpy(np.ascontiguousarray(inp.gate)),
             "h_b": torch.from_numpy(np.ascontiguousarray(inp.beta)),
             "h_s": None if st is None else torch.from_numpy(np.ascontiguousarray(st, dtype=np.float32))}
        for key in ("q", "k", "v", "g", "b", "s"):
            h[key] = None if h["h_" + key] is None else h["h_" + key].to(device)
        sets.append(h)
    return sets, inps[0]


def run_ours(args, w, rank, world, local):
    import torch
    import hybrid_linear_attention_frame_b200 as G

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init("nccl", world)
    layers = calls_per_step(args, w)
    lib = G.load()
    fp8 = args.inputs == "fp8"
    if fp8 and (w.name == "sessions" or args.direction == "bidir" or args.gate_mode == "frame" or args.path == "ws"):
        raise SystemExit("--inputs fp8: layer workloads (minute, clip241, block), forward scan, plain path")
    sets, inp0 = upload_sets(w, device, fp8)
    stream_step = w.name == "sessions"
    out = torch.empty(sets[0]["v"].shape, dtype=torch.bfloat16, device=device)
    st_out = torch.empty((w.B, w.H, w.d_k, w.d_v), dtype=torch.float32, device=device)
    if stream_step:
        st_out.copy_(sets[0]["s"])             # the sessions' state, carried in place
    stream = torch.cuda.current_stream(device)
    sptr = stream.cuda_stream
    dims = (w.B, w.H, w.T, w.d_k, w.d_v, w.frame_len, w.chunk_len)
    bidir = args.direction == "bidir"
    gate_mode = 1 if args.gate_mode == "frame" else 0
    if bidir and (gate_mode or w.name != "minute"):
        raise SystemExit("--direction bidir: minute workload, gate at every token")
    if gate_mode and stream_step:
        raise SystemExit("--gate-mode frame applies to the layer workloads")
    use_ws = args.path == "ws" and G.gdn_workspace_bytes(*dims[:5], w.chunk_len) > 0
    if bidir:
        ws = G.bidir_workspace(w.B, w.H, w.T, w.d_k, w.d_v, w.chunk_len, device)
    else:
        ws = G.workspace(w.B, w.H, w.T, w.d_k, w.d_v, w.chunk_len, device) if use_ws else None
    ws_args = (ws.data_ptr(), ws.numel()) if ws is not None else (None, 0)
    with_state_in = w.name == "block" or stream_step

    def layer_call(i):
        x = sets[i % len(sets)]
        ptr = (x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["g"].data_ptr(), x["b"].data_ptr())
        if bidir:
            st = lib.gdn_forward_bidir(*ptr, out.data_ptr(), *dims, *ws_args, sptr)
            name = "gdn_forward_bidir"
        elif stream_step:
            if use_ws:
                st = lib.gdn_state_step_ws(*ptr, st_out.data_ptr(), out.data_ptr(), *dims, *ws_args, sptr)
                name = "gdn_state_step_ws"
            else:
                st = lib.gdn_state_step(*ptr, st_out.data_ptr(), out.data_ptr(), *dims, sptr)
                name = "gdn_state_step"
        else:
            s_in = x["s"].data_ptr() if (with_state_in and x["s"] is not None) else None
            args_ = (*ptr, s_in, st_out.data_ptr(), out.data_ptr())
            if fp8:
                st = lib.gdn_forward_fp8(*ptr[:3], x["v_scale"], *ptr[3:], s_in, st_out.data_ptr(),
                                         out.data_ptr(), *dims, sptr)
                name = "gdn_forward_fp8"
            elif gate_mode:
                st = lib.gdn_forward_gated(*args_, *dims, gate_mode, *ws_args, sptr)
                name = "gdn_forward_gated"
            elif use_ws:
                st = lib.gdn_forward_ws(*args_, *dims, *ws_args, sptr)
                name = "gdn_forward_ws"
            else:
                st = lib.gdn_forward(*args_, *dims, sptr)
                name = "gdn_forward"
        if st != 0:
            raise G.GdnError(st, name)

    for _ in range(args.warmup):
        for i in range(layers):
            layer_call(i)
    torch.cuda.synchronize(device)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps * layers)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        uuid = None
    clocks = ClockSampler(uuid).start() if rank == 0 else None
    barrier(world, device)
    torch.cuda.synchronize(device)
    t_start.record(stream)
    n = 0
    for _ in range(args.steps):
        for i in range(layers):
            ev[n][0].record(stream)
            layer_call(i)
            ev[n][1].record(stream)
            n += 1
    t_end.record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    clock_rec = clocks.stop() if clocks else None
    dev_status = G.gdn_get_last_device_status()
    if dev_status != G.GDN_OK:
        raise G.GdnError(dev_status, "device status after the timed region")

    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    tokens_per_rank = w.B * w.T * layers * args.steps
    value, slowest = aggregate_throughput(tokens_per_rank, elapsed_s, world, device)
    ms_per_step = slowest * 1e3 / args.steps
    launch_ms = [a_.elapsed_time(b_) for (a_, b_) in ev]
    avg_launch_s = statistics.mean(launch_ms) / 1e3

    peaks, peak_kind = measured_peaks()
    abytes = algorithmic_bytes(w, state_in=with_state_in, state_out=not bidir, in_elem=1 if fp8 else 2)
    achieved = abytes / avg_launch_s / 1e9
    traffic, traffic_kernel = recorded_traffic()
    if bidir:
        kernel = ("gdn_forward_bidir (one layer call: reverse copy, 2 x "
                  + ("gdn_seq_kernel" if G.gdn_bf16_path(w.d_k, w.d_v, w.chunk_len) == 2 else "gdn_ring_kernel")
                  + ", combine)")
    elif use_ws:
        kernel = "gdn_ring_kernel"
    elif fp8:
        kernel = "gdn_seq_kernel (e4m3 inputs)"
    elif G.gdn_bf16_path(w.d_k, w.d_v, w.chunk_len) == 2:
        kernel = "gdn_seq_kernel"
    else:
        kernel = "gdn_chunk_tc_kernel" if G.gdn_bf16_path(w.d_k, w.d_v, w.chunk_len) == 1 \
            else "chunk_ffma_kernel<bf16,64>"
    flops_scans = 2 if bidir else 1
    flops = flops_scans * CHUNKED_FLOPS_PER_TOKEN_HEAD * w.B * w.T * w.H
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic if (traffic_kernel == kernel and w.name == "minute") else None,
                "kernel": kernel, "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth)",
                "algorithmic_bytes_per_launch": abytes,
                "avg_launch_us": round(avg_launch_s * 1e6, 2),
                "tensor_flops_frac": round(flops / avg_launch_s / 1e12 / peaks["bf16_tflops"], 4),
                "roofline_frac": round(max(abytes / (peaks["hbm_gbs"] * 1e9),
                                           flops / (peaks["bf16_tflops"] * 1e12)) / avg_launch_s, 4)}
    if stream_step:
        roofline["per_block_us"] = round(avg_launch_s * 1e6, 2)

    e2e = None
    if not args.no_e2e and not bidir and not fp8:
        e2e = run_e2e(lib, G, w, device, stream, sets, out, st_out, world,
                      max(2, min(args.steps, 3)) if not stream_step else 1, layers if stream_step else 1, ws)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if fp8:
            from oracle import gdn_reference as R
            inp0 = R.widen_fp8(inp0)
        cpu = cpu_baseline(w, inp0, args.cpu_seconds, bidir=bidir)

    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": run_config(args, w),
            "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps * layers * (4 if bidir else 1),
            "clocks": clock_rec}
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    return line if rank == 0 else None


def run_e2e(lib, G, w, device, stream, sets, out, st_out, world, steps, calls, ws=None):
    """The same metric through gdn_forward_host(_ws): pinned host inputs copied
    in, output and final state copied out, every call (a layer, or a streaming
    block whose state goes in and out through the host)."""
    import torch
    pinned = []
    for x in sets[:max(1, min(len(sets), calls))]:
        pinned.append({key: (None if x["h_" + key] is None else x["h_" + key].pin_memory())
                       for key in ("q", "k", "v", "g", "b", "s")})
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_st = torch.empty(st_out.shape, dtype=torch.float32).pin_memory()
    x0 = sets[0]
    sptr = stream.cuda_stream
    api = "gdn_forward_host_ws" if ws is not None else "gdn_forward_host"
    stream_step = w.name == "sessions"

    def call(i):
        hp = pinned[i % len(pinned)]
        if stream_step:
            h_s = h_st if i > 0 else hp["s"]        # the state goes out to the host and back in
        else:
            h_s = hp["s"]
        a = (hp["q"].data_ptr(), hp["k"].data_ptr(), hp["v"].data_ptr(), hp["g"].data_ptr(), hp["b"].data_ptr(),
             None if h_s is None else h_s.data_ptr(), h_st.data_ptr(), h_out.data_ptr(),
             x0["q"].data_ptr(), x0["k"].data_ptr(), x0["v"].data_ptr(), x0["g"].data_ptr(), x0["b"].data_ptr(),
             st_out.data_ptr(), out.data_ptr(), w.B, w.H, w.T, w.d_k, w.d_v, w.frame_len, w.chunk_len)
        if ws is not None:
            st = lib.gdn_forward_host_ws(*a, ws.data_ptr(), ws.numel(), sptr)
        else:
            st = lib.gdn_forward_host(*a, sptr)
        if st != 0:
            raise G.GdnError(st, api)

    call(0)
    barrier(world, device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        for i in range(calls):
            call(i)
    t1.record(stream)
    torch.cuda.synchronize(device)
    elapsed = t0.elapsed_time(t1) / 1e3
    value, _ = aggregate_throughput(w.B * w.T * steps * calls, elapsed, world, device)
    hp = pinned[0]
    h2d = sum(hp[key].numel() * hp[key].element_size() for key in ("q", "k", "v", "g", "b"))
    if hp["s"] is not None or stream_step:
        h2d += h_st.numel() * 4
    d2h = h_out.numel() * h_out.element_size() + h_st.numel() * 4
    return {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d * calls,
            "d2h_bytes_per_step": d2h * calls, "steps": steps,
            "api": f"{api} (C ABI, pinned host buffers, {calls} call(s) per step)"}


def run_profile_case(w, tokens, path="ws"):
    """Two layer calls (warm-up + the one a profiler captures) on the first
    `tokens` tokens of the layer; small enough for a many-pass ncu capture."""
    import numpy as np
    import torch
    import hybrid_linear_attention_frame_b200 as G
    from workloads import bf16_bits, make_inputs
    inp = make_inputs(w, T=tokens)
    def bf16(x):
        return torch.from_numpy(bf16_bits(x).view(np.int16).copy()).view(torch.bfloat16).cuda()
    q, k, v = bf16(inp.q), bf16(inp.k), bf16(inp.v)
    g = torch.from_numpy(inp.gate).cuda()
    b = torch.from_numpy(inp.beta).cuda()
    out = torch.empty_like(v)
    st = torch.empty((w.B, w.H, w.d_k, w.d_v), dtype=torch.float32, device="cuda")
    ws = G.workspace(w.B, w.H, tokens, w.d_k, w.d_v, w.chunk_len) if path == "ws" else None
    for _ in range(2):
        if ws is not None:
            G.gdn_forward_ws(q, k, v, g, b, None, st, out, w.B, w.H, tokens, w.d_k, w.d_v,
                             w.frame_len, w.chunk_len, ws)
        else:
            G.gdn_forward(q, k, v, g, b, None, st, out, w.B, w.H, tokens, w.d_k, w.d_v,
                          w.frame_len, w.chunk_len)
    torch.cuda.synchronize()
    status = G.gdn_get_last_device_status()
    print(f"profile case: T={tokens}, device status {status}")
    return 0 if status == G.GDN_OK else 1


def run_profile_case_softmax(w, tokens):
    """Two softmax-attention layer calls on the first `tokens` tokens (profiling case)."""
    import numpy as np
    import torch
    import hybrid_linear_attention_frame_b200 as G
    from workloads import bf16_bits, make_inputs
    inp = make_inputs(w, T=tokens)

    def bf16(x):
        return torch.from_numpy(bf16_bits(x).view(np.int16).copy()).view(torch.bfloat16).cuda()
    q, k, v = bf16(inp.q), bf16(inp.k), bf16(inp.v)
    out = torch.empty_like(v)
    for _ in range(2):
        G.gdn_softmax_attention(q, k, v, out, w.B, w.H, tokens, w.d_k, w.d_v, w.frame_len,
                                ATTN_GEOMETRY["frames_per_block"], ATTN_GEOMETRY["cached_blocks"],
                                ATTN_GEOMETRY["sink_frames"])
    torch.cuda.synchronize()
    status = G.gdn_get_last_device_status()
    print(f"softmax profile case: T={tokens}, device status {status}")
    return 0 if status == G.GDN_OK else 1


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    w = workload_of(args)
    if args.layer == "softmax" and w.name != "minute":
        raise SystemExit("--layer softmax runs on the minute workload")
    if args.profile_tokens > 0 and args.layer == "softmax":
        return run_profile_case_softmax(w, args.profile_tokens)
    if args.profile_tokens > 0:
        return run_profile_case(w, args.profile_tokens, args.path)
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
    elif args.layer == "softmax":
        line = run_softmax(args, w, rank, world, local)
    else:
        line = run_ours(args, w, rank, world, local)
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
