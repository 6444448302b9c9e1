#!/usr/bin/env python3
"""Benchmark of the same-step KV chunk-attention hot path on B200.

Workload (one "step"): one denoising step of one 880-token latent-frame chunk
at the profile's steady state (1280x704 -> 40x22 tokens, 24 heads x 128, a
2,640-token sink plus 18 ring slots = 18,480 keys), over 30 layers:
per layer one pv_rope_append (3D RoPE of q, k and the append of k, v into the
per-step ring) and one pv_chunk_attn, then one pv_euler_step on the chunk's
48 x 44 x 80 latent.  Inputs are synthetic (seeded generator), the history of
every layer is pre-filled, and the working set (6.9 GB of K/V) is far larger
than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload step|schedule|dense|multistream|cross_attn|sampler|qkv]

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

W, HH, HEADS, D, R, LAYERS, STEP = 40, 22, 24, 128, 18, 30, 2
T = W * HH
CHUNK = 28                      # steady state: 17 earlier chunks + this one in the ring
N_KEYS = (3 + R) * T            # 18,480
LATENT = 48 * 44 * 80           # values of one latent frame
ATTN_FLOPS = 4 * T * N_KEYS * HEADS * D          # one chunk_attn launch
ROPE_BYTES = 6 * T * HEADS * D * 2               # q,k,v read; q_rot,k_rot,v written
WORKLOAD = "steady chunk 880 q x 18480 k, 24x128, 30 layers + Euler 48x44x80"
METRIC = "chunk-attention TFLOP/s (whole step: 30 x rope_append + chunk_attn, Euler)"


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("pv_attn.cu", "pv_internal.h", "pv_plan.cu"):
        with open(os.path.join(ROOT, "same_step_kv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per chunk_attn launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "chunk_attn_880x18480.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    src = tb = None
    for line in text.splitlines():
        if line.startswith("source_hash:"):
            src = line.split(":", 1)[1].strip()
        if line.startswith("dram_bytes_per_launch:"):
            tb = float(line.split(":", 1)[1].strip())
    return tb if (src == attn_source_hash() and tb) else None


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # nvidia-smi takes a moment to start: let sampling be live before
            # the timed region begins
            t_end = time.time() + 3.0
            while not self.lines and time.time() < t_end:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        mhz, mx, reasons = [], None, set()
        capped = 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                mhz.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, p in zip(names, parts[3:7]):
                if p.lower() == "active":
                    reasons.add(n)
                    capped += n == "sw_power_cap"
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz),
                "power_cap_share": capped / len(mhz) if mhz else None}


def tensor_peak(peaks, src, clocks, seconds):
    """The dense bf16 peak that a tensor-bound kernel timed in this run is held
    against: the burst figure (cuBLAS in a short run) unless the timed region
    lasted a second or more with the power cap active in at least half of its
    clock samples, when the sustained figure (a seconds-long cuBLAS loop under
    the cap) applies.  Returns (peak, label, the other figure)."""
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    share = (clocks or {}).get("power_cap_share")
    if seconds >= 1.0 and share is not None and share >= 0.5:
        return sustained, (f"{src} bf16_tflops_sustained ({seconds:.1f} s timed, power cap in "
                           f"{share:.0%} of samples)"), burst
    return burst, (f"{src} bf16_tflops (burst; {seconds:.2f} s timed, power cap in "
                   f"{share or 0:.0%} of samples)"), sustained


def tensor_roofline(achieved, peaks, src, clocks, seconds, kernel, **extra):
    """Roofline object of a tensor-bound kernel: achieved TFLOP/s against the
    peak tensor_peak() picks for a timed region of `seconds`, with the
    fractions of both measured peaks."""
    peak, label, _ = tensor_peak(peaks, src, clocks, seconds)
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    line = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "peak_source": label,
            "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
            "kernel": kernel, "traffic": None}
    line.update(extra)
    return line


def oracle_inputs(heads=HEADS):
    """Host fp64 inputs of one layer of the workload for the first `heads`
    heads: the chunk's q, k, v and the pre-filled K/V history.  The history
    is drawn for those heads only; it is head-major, so that draw is exactly
    the first `heads` heads of the full one."""
    from same_step_kv_b200 import synth
    q, k, v = synth.chunk_qkv(0, CHUNK, STEP, 0, T, HEADS, D)
    kf, vf = synth.store_fill(0, 0, STEP, heads, N_KEYS, D)
    q, k, v = (t[:, :heads].double().numpy() for t in (q, k, v))
    K = kf.double().numpy().transpose(1, 0, 2).copy()
    V = vf.double().numpy().transpose(1, 0, 2).copy()
    return q, k, v, K, V


def blas_threads() -> int:
    """Threads of the BLAS that numpy (the oracle's matrix products) runs on."""
    import numpy  # noqa: F401  (loads the BLAS, so that it is listed)
    from threadpoolctl import threadpool_info
    n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
    return max(n) if n else 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(inputs):
    """The fp64 oracle on one layer of the workload: RoPE of the chunk's q and
    k, their append into the ring slot, and the attention of all 880 queries
    of the inputs' heads over 18,480 keys.  Returns (flops, seconds, threads).
    The append writes the same rows every time, so samples repeat exactly."""
    import torch
    from oracle import attention, rope
    q, k, v, K, V = inputs
    heads = q.shape[1]
    t0 = time.perf_counter()
    f, hh, ww = rope.token_coords(T, W, HH, 2 + CHUNK)
    qr = rope.rotate(q, f, hh, ww)
    kr = rope.rotate(k, f, hh, ww)
    slot = (CHUNK - 1) % R
    K[3 * T + slot * T: 3 * T + slot * T + T] = kr
    V[3 * T + slot * T: 3 * T + slot * T + T] = v
    attention.attend_heads(qr, K, V)
    dt = time.perf_counter() - t0
    return ATTN_FLOPS * heads // HEADS, dt, blas_threads()


def oracle_one_core(heads=2, runs=2):
    """The oracle on one core (BLAS limited to one thread) on `heads` heads of
    one layer: the per-core baseline beside the all-core one."""
    from threadpoolctl import threadpool_limits
    inputs = oracle_inputs(heads=heads)
    with threadpool_limits(limits=1, user_api="blas"):
        rs = [oracle_sample(inputs) for _ in range(runs)]
    fl, dt = rs[0][0], statistics.median(r[1] for r in rs)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": 1,
            "sample": f"{heads} of the 24 heads of one layer (880 x 18480 each), "
                      f"median of {runs} runs"}


def run_reference(args, rank):
    if rank != 0:
        return
    vals = []
    inputs = oracle_inputs(heads=2)
    for i in range(args.warmup + args.steps):
        fl, dt, thr = oracle_sample(inputs)
        if i >= args.warmup:
            vals.append(fl / dt / 1e12)
    v = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "sample": "per step: RoPE + 880 x 18480 attention of 2 of the 24 heads of one layer"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                         "sample": "per step: 2 heads of one layer (880 queries x 18480 keys each)",
                         "cpu_model": cpu_model()},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "vs_baseline": None,
    }
    print(json.dumps(line), flush=True)


def timed_steps(step, args, local, world, cs):
    """W untimed steps, then K steps between CUDA events on `cs`, with clocks
    sampled meanwhile.  Returns (ms per step, max over ranks; clock summary)."""
    import torch
    import torch.distributed as dist
    from same_step_kv_b200.dist import max_over_ranks
    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(cs)
        for _ in range(args.steps):
            step(True)
        t1.record(cs)
        torch.cuda.synchronize()
    return max_over_ranks(t0.elapsed_time(t1)) / args.steps, clk.summary()


def bound_roofline(flops, nbytes, seconds, peaks, src, kernel, clocks, timed_s):
    """Roofline object for a kernel that may be bound by either pipe: the bound
    is whichever of flops / tensor peak and bytes / HBM peak takes longer."""
    tpeak = tensor_peak(peaks, src, clocks, timed_s)[0]
    hbm_peak = float(peaks["hbm_gbs"])
    if flops / (tpeak * 1e12) >= nbytes / (hbm_peak * 1e9):
        return tensor_roofline(flops / seconds / 1e12, peaks, src, clocks, timed_s, kernel,
                               hbm_achieved_gbs=nbytes / seconds / 1e9)
    a = nbytes / seconds / 1e9
    return {"bound": "hbm", "achieved": a, "peak": hbm_peak, "unit": "GB/s", "frac": a / hbm_peak,
            "peak_source": f"{src} hbm_gbs", "kernel": kernel, "traffic": None,
            "tensor_achieved_tflops": flops / seconds / 1e12}


N_PROMPTS = 8       # cross-attention: prompts served together, one latent frame each
MAX_TEXT = 512      # longest text context (tokens)


def run_cross_attn(args, rank, world, local):
    """Cross-attention of N_PROMPTS prompts, each one latent frame (880 video
    tokens) querying its own text context of 1..512 tokens, 24 x 128, one
    pv_attn_varlen launch per layer, 30 layers per step."""
    import torch
    from same_step_kv_b200 import pv, synth
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()
    NL = args.layers
    n_k = synth.text_lengths(N_PROMPTS, MAX_TEXT, seed=rank)
    n_q = [T] * N_PROMPTS
    tq, tk = sum(n_q), sum(n_k)
    q = [synth.normal_bf16(synth.seed_of(0x5101, rank, l), (HEADS * tq * D,), dev) for l in range(NL)]
    k = [synth.normal_bf16(synth.seed_of(0x5102, rank, l), (HEADS * tk * D,), dev) for l in range(NL)]
    v = [synth.normal_bf16(synth.seed_of(0x5103, rank, l), (HEADS * tk * D,), dev) for l in range(NL)]
    out = torch.empty(tq, HEADS, D, dtype=torch.bfloat16, device=dev)
    wsb = pv.pv_attn_varlen_ws_bytes(n_q, n_k, HEADS, D)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    ev = []

    def step(record):
        for l in range(NL):
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(cs)
            pv.pv_attn_varlen(q[l], k[l], v[l], n_q, n_k, HEADS, D, out, None, ws, wsb, cs)
            if record:
                e1.record(cs)
                ev.append((e0, e1))

    ms_step, clocks = timed_steps(step, args, local, world, cs)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = sum(4 * a * b * HEADS * D for a, b in zip(n_q, n_k))
    nbytes = (2 * tq + 2 * tk) * HEADS * D * 2          # q, out; k, v
    # e2e: each layer's q and text context from pinned host memory, output read back
    hq = [t.cpu().pin_memory() for t in q]
    hk = [t.cpu().pin_memory() for t in k]
    hv = [t.cpu().pin_memory() for t in v]
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q[0]), torch.empty_like(k[0]), torch.empty_like(v[0])

    def e2e_step(record):
        for l in range(NL):
            dq.copy_(hq[l], non_blocking=True)
            dk.copy_(hk[l], non_blocking=True)
            dv.copy_(hv[l], non_blocking=True)
            pv.pv_attn_varlen(dq, dk, dv, n_q, n_k, HEADS, D, out, None, ws, wsb, cs)
        hout.copy_(out, non_blocking=True)

    e2e_ms, _ = timed_steps(e2e_step, args, local, world, cs)
    if rank == 0:
        peaks, src = load_peaks()
        line = {
            "metric": "cross-attention TFLOP/s (30 layers x 8 prompts, one launch per layer)",
            "value": NL * flops * world / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"cross-attention, {N_PROMPTS} prompts x 880 video tokens, "
                                   f"text 1..{MAX_TEXT} tokens, 24x128, {NL} layers",
                       "text_lengths": n_k,
                       "l2": f"inputs larger than L2 ({NL * (tq + 2 * tk) * HEADS * D * 2 / 1e9:.2f} GB "
                             "per step), no flush"},
            "roofline": bound_roofline(flops, nbytes, launch_ms * 1e-3, peaks, src,
                                       "attn_kernel<128> (pv_attn_varlen)", clocks,
                                       ms_step * args.steps * 1e-3),
            "e2e": {"value": NL * flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": NL * (tq + 2 * tk) * HEADS * D * 2,
                    "d2h_bytes_per_step": tq * HEADS * D * 2},
            "gpu_launches": args.steps * NL, "clocks": clocks, "cpu_baseline": None,
        }
        line["roofline"]["ms_per_launch"] = launch_ms
        print(json.dumps(line), flush=True)


def run_qkv(args, rank, world, local):
    """The q, k, v projection with QK-Norm, RoPE and append of the steady chunk
    (880 tokens of dim 3072 = 24 x 128), one pv_qkv_rope_append per layer
    (its own weights), 30 layers per step.  At this size every GEMM tile is
    resident at once, so the call is one cooperative launch with the norm,
    RoPE and append in the GEMM's epilogue.  Metric: the GEMM's algorithmic
    FLOPs (2 x 880 x 3072 x 9216 per layer) over the time of the whole call."""
    import torch
    from same_step_kv_b200 import pv, synth
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()
    NL = args.layers
    dim = HEADS * D
    cfg = pv.make_config(NL, HEADS, D, W, HH, ring_slots=R, max_streams=1, max_frames=64)
    store = pv.KVStore(cfg, device=dev)
    h = store.handle
    st = pv.pv_kv_state()
    st.phase, st.chunk = pv.PV_PHASE_STEADY, CHUNK
    pv.pv_kv_set_state(h, 0, st)
    x = [synth.normal_bf16(synth.seed_of(0x6101, rank, l), (T, dim), dev) for l in range(NL)]
    w = [(synth.normal_f32(synth.seed_of(0x6102, rank, l), (3 * dim, dim), dev) / dim ** 0.5)
         .to(torch.bfloat16) for l in range(NL)]
    bias = [0.1 * synth.normal_f32(synth.seed_of(0x6103, rank, l), (3 * dim,), dev) for l in range(NL)]
    g = 1.0 + 0.1 * synth.normal_f32(synth.seed_of(0x6104, rank), (2, dim), dev)
    q_rot = torch.empty(HEADS * T * D, dtype=torch.bfloat16, device=dev)
    wsb = pv.pv_qkv_ws_bytes(T, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    ev = []

    def call(l, xl):
        pv.pv_qkv_rope_append(h, [0], l, STEP, xl, w[l], bias[l], g[0], g[1], 1e-6, q_rot, ws, wsb,
                              cs)

    def step(record):
        for l in range(NL):
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(cs)
            call(l, x[l])
            if record:
                e1.record(cs)
                ev.append((e0, e1))

    ms_step, clocks = timed_steps(step, args, local, world, cs)
    call_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = 2 * T * dim * 3 * dim
    # e2e: each layer's tokens from pinned host memory, q_rot read back
    hx = [t.cpu().pin_memory() for t in x]
    hq = torch.empty(q_rot.shape, dtype=q_rot.dtype).pin_memory()
    dx = torch.empty_like(x[0])

    def e2e_step(record):
        for l in range(NL):
            dx.copy_(hx[l], non_blocking=True)
            call(l, dx)
        hq.copy_(q_rot, non_blocking=True)

    e2e_ms, _ = timed_steps(e2e_step, args, local, world, cs)
    if rank == 0:
        peaks, src = load_peaks()
        a = flops / (call_ms * 1e-3) / 1e12
        line = {
            "metric": "qkv projection TFLOP/s (QK-Norm, RoPE, append fused around a tcgen05 GEMM)",
            "value": NL * flops * world / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"qkv projection of the steady chunk, 880 tokens x {dim} -> "
                                   f"3 x {dim}, {NL} layers (random weights)",
                       "l2": f"weights larger than L2 ({NL * 3 * dim * dim * 2 / 1e9:.2f} GB "
                             "per step), no flush"},
            "roofline": tensor_roofline(
                a, peaks, src, clocks, ms_step * args.steps * 1e-3,
                "qkv_gemm_kernel<256, fused> (one cooperative launch per call)",
                ms_per_launch=call_ms),
            "e2e": {"value": NL * flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": NL * T * dim * 2,
                    "d2h_bytes_per_step": HEADS * T * D * 2},
            "gpu_launches": NL * args.steps, "clocks": clocks, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    store.close()


SAMPLER_FRAMES = 248   # 8 streams x 31 latent frames


def run_sampler(args, rank, world, local):
    """One sampler step over a batch of SAMPLER_FRAMES latent frames (48 x 44 x 80
    each): the CFG-guided Euler update (x, v_cond, v_uncond in, x out: 16 B per
    value), the plain Euler update of a second latent batch (x, v in, x out:
    12 B per value) and the x0 estimate (x, v in, x0 out: 12 B per value)."""
    import torch
    from same_step_kv_b200 import pv, synth
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()
    n = SAMPLER_FRAMES * LATENT
    x = synth.normal_f32(synth.seed_of(0x5A01, rank), (n,), dev)
    vc = synth.normal_f32(synth.seed_of(0x5A02, rank), (n,), dev)
    vu = synth.normal_f32(synth.seed_of(0x5A03, rank), (n,), dev)
    x0 = torch.empty_like(x)
    xe = synth.normal_f32(synth.seed_of(0x5A04, rank), (n,), dev)
    sig = pv.pv_sigma_schedule(40, 12.0)[0]
    d = float(sig[21] - sig[20])
    w = 5.0
    ev = []

    def step(record):
        if record:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(cs)
        pv.pv_euler_cfg_step(x, vc, vu, n, w, d, cs)
        if record:
            e1.record(cs)
            ev.append((e0, e1))
        pv.pv_euler_step(xe, vu, n, d, cs)
        pv.pv_x0_estimate(x0, x, vc, n, float(sig[21]), cs)

    ms_step, clocks = timed_steps(step, args, local, world, cs)
    cfg_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    step_bytes = 16 * n + 12 * n + 12 * n
    # e2e: velocities in from pinned host memory, x0 read back
    hvc, hvu = vc.cpu().pin_memory(), vu.cpu().pin_memory()
    hx0 = torch.empty(n, dtype=torch.float32).pin_memory()

    def e2e_step(record):
        vc.copy_(hvc, non_blocking=True)
        vu.copy_(hvu, non_blocking=True)
        pv.pv_euler_cfg_step(x, vc, vu, n, w, d, cs)
        pv.pv_euler_step(xe, vu, n, d, cs)
        pv.pv_x0_estimate(x0, x, vc, n, float(sig[21]), cs)
        hx0.copy_(x0, non_blocking=True)

    e2e_ms, _ = timed_steps(e2e_step, args, local, world, cs)
    if rank == 0:
        peaks, src = load_peaks()
        hbm = float(peaks["hbm_gbs"])
        a = 16 * n / (cfg_ms * 1e-3) / 1e9
        line = {
            "metric": "sampler GB/s (CFG-guided Euler step, Euler step, x0 estimate)",
            "value": step_bytes * world / (ms_step * 1e-3) / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": f"sampler, {SAMPLER_FRAMES} latent frames of 48x44x80 "
                                   "(shift 12, step 20 of 40, guide scale 5)",
                       "values": n, "l2": f"inputs larger than L2 ({4 * n * 4 / 1e9:.2f} GB), no flush"},
            "roofline": {"bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm,
                         "peak_source": f"{src} hbm_gbs", "kernel": "euler_cfg_kernel",
                         "ms_per_launch": cfg_ms, "traffic": None},
            "e2e": {"value": step_bytes * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": 8 * n, "d2h_bytes_per_step": 4 * n},
            "gpu_launches": 3 * args.steps, "clocks": clocks, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)


DENSE_FRAMES = 21   # whole-video attention: 21 latent frames = 18,480 tokens
N_STREAMS = 8       # batched serving: streams in one launch


def run_dense(args, rank, world, local):
    """Full bidirectional attention over a whole latent video (21 frames x 880
    tokens attending to all 18,480), 24 x 128, 3D RoPE at frames 0..20: per
    layer one pv_rope_dense and one pv_attn_dense."""
    import torch
    from same_step_kv_b200 import pv, synth
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()
    n = DENSE_FRAMES * T
    cfg = pv.make_config(1, HEADS, D, W, HH, ring_slots=R, max_streams=1, max_frames=64)
    store = pv.KVStore(cfg, device=dev)
    q, k, v = synth.chunk_qkv(rank, 0, 0, 0, n, HEADS, D, dev)
    q_rot = torch.empty(HEADS, n, D, dtype=torch.bfloat16, device=dev)
    k_rot, v_hm = torch.empty_like(q_rot), torch.empty_like(q_rot)
    out = torch.empty(n, HEADS, D, dtype=torch.bfloat16, device=dev)
    wsb = pv.pv_attn_dense_ws_bytes(n, n, HEADS, D)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    ev = []

    def step(record):
        pv.pv_rope_dense(store.handle, n, 0, q, k, v, q_rot, k_rot, v_hm, cs)
        if record:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(cs)
        pv.pv_attn_dense(q_rot, k_rot, v_hm, n, n, HEADS, D, out, None, ws, wsb, cs)
        if record:
            e1.record(cs)
            ev.append((e0, e1))

    ms_step, clocks = timed_steps(step, args, local, world, cs)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = 4 * n * n * HEADS * D
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step(record):
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        step(False)
        hout.copy_(out, non_blocking=True)

    e2e_ms, _ = timed_steps(e2e_step, args, local, world, cs)
    if rank == 0:
        peaks, src = load_peaks()
        achieved = flops / (launch_ms * 1e-3) / 1e12
        line = {
            "metric": "dense video attention TFLOP/s (18,480 x 18,480, 24x128, RoPE + attention)",
            "value": flops * world / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"whole video: {DENSE_FRAMES} latent frames x 880 tokens, "
                                   "all-to-all, 24x128, one layer per step",
                       "l2": "q, k, v of 0.34 GB per step (larger than L2), no flush"},
            "roofline": tensor_roofline(achieved, peaks, src, clocks, ms_step * args.steps * 1e-3,
                                        "attn_kernel<128> (pv_attn_dense)",
                                        ms_per_launch=launch_ms),
            "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": 3 * n * HEADS * D * 2,
                    "d2h_bytes_per_step": n * HEADS * D * 2},
            "gpu_launches": 2 * args.steps, "clocks": clocks, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    store.close()


def run_multistream(args, rank, world, local):
    """Batched serving: N_STREAMS streams, each at its own steady chunk with a
    seeded ragged ring fill (0..18 earlier chunks), one pv_rope_append and one
    pv_chunk_attn over all streams per layer, 30 layers, then the Euler update
    of the streams' latent frames."""
    import torch
    from same_step_kv_b200 import pv, synth
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()
    NL = args.layers
    fills = synth.ragged_fills(N_STREAMS, R, seed=rank)
    # one step buffer per layer and stream (the step timed is one denoising
    # step): 30 layers x 8 streams x 18,480 keys is 54.5 GB of K/V
    cfg = pv.make_config(NL, HEADS, D, W, HH, ring_slots=R, steps=1, max_streams=N_STREAMS,
                         max_frames=64)
    store = pv.KVStore(cfg, device=dev)
    h = store.handle
    Kr, Vr = store.k_region(), store.v_region()
    n_keys = []
    for i, f in enumerate(fills):
        st = pv.pv_kv_state()
        st.phase, st.chunk = pv.PV_PHASE_STEADY, f + 1
        pv.pv_kv_set_state(h, i, st)
        nk = pv.pv_kv_get_state(h, i).n_keys
        n_keys.append(nk)
        kf, vf = synth.store_fill(rank * N_STREAMS + i, 0, 0, HEADS, nk, D, dev)
        for layer in range(NL):
            Kr[layer, 0, i, :, :nk] = kf
            Vr[layer, 0, i, :, :nk] = vf
        del kf, vf
    streams = list(range(N_STREAMS))
    tok = N_STREAMS * T
    qkv = [synth.chunk_qkv(rank, 1000 + layer, 0, layer, tok, HEADS, D, dev) for layer in range(NL)]
    q_rot = torch.empty(HEADS * tok * D, dtype=torch.bfloat16, device=dev)
    out = torch.empty(tok, HEADS, D, dtype=torch.bfloat16, device=dev)
    x = synth.latent(rank, N_STREAMS, 48, 44, 80, dev).reshape(-1)
    vel = synth.velocity(rank, 0, 0, N_STREAMS * LATENT, dev)
    ev = []

    def step(record):
        for layer in range(NL):
            q, k, v = qkv[layer]
            pv.pv_rope_append(h, streams, layer, 0, q, k, v, q_rot, cs)
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(cs)
            pv.pv_chunk_attn(h, streams, layer, 0, q_rot, out, None, cs)
            if record:
                e1.record(cs)
                ev.append((e0, e1))
        pv.pv_euler_step(x, vel, N_STREAMS * LATENT, -0.25, cs)

    ms_step, clocks = timed_steps(step, args, local, world, cs)
    launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = sum(4 * T * nk * HEADS * D for nk in n_keys)
    hq = [[t.cpu().pin_memory() for t in qkv[layer]] for layer in range(NL)]
    dq = [torch.empty_like(t) for t in qkv[0]]
    hx = x.cpu().pin_memory()

    def e2e_step(record):
        x.copy_(hx, non_blocking=True)
        for layer in range(NL):
            for a, b in zip(dq, hq[layer]):
                a.copy_(b, non_blocking=True)
            pv.pv_rope_append(h, streams, layer, 0, dq[0], dq[1], dq[2], q_rot, cs)
            pv.pv_chunk_attn(h, streams, layer, 0, q_rot, out, None, cs)
        pv.pv_euler_step(x, vel, N_STREAMS * LATENT, -0.25, cs)
        hx.copy_(x, non_blocking=True)

    e2e_ms, _ = timed_steps(e2e_step, args, local, world, cs)
    if rank == 0:
        peaks, src = load_peaks()
        achieved = flops / (launch_ms * 1e-3) / 1e12
        line = {
            "metric": "batched chunk-attention TFLOP/s; latent frames/s per denoise step",
            "value": NL * flops * world / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"{N_STREAMS} streams x 880 tokens, ragged ring fills {fills}, "
                                   f"24x128, {NL} layers + Euler",
                       "keys_per_stream": n_keys,
                       "l2": "K/V working set larger than L2, no flush"},
            "latent_frames_per_s": world * N_STREAMS / (ms_step * 1e-3),
            "roofline": tensor_roofline(achieved, peaks, src, clocks, ms_step * args.steps * 1e-3,
                                        "attn_kernel<128> (pv_chunk_attn, 8 streams)",
                                        ms_per_launch=launch_ms),
            "e2e": {"value": NL * flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": NL * 3 * tok * HEADS * D * 2 + x.numel() * 4,
                    "d2h_bytes_per_step": x.numel() * 4},
            "gpu_launches": args.steps * (2 * NL + 1), "clocks": clocks, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    store.close()


N_CHUNKS = 28       # one-frame chunks after the 3-frame first chunk: 31 latent frames
POOL = 4            # distinct synthetic q, k, v sets cycled through the schedule


def run_schedule(args, rank, world, local):
    """The whole generation schedule of one stream: the first chunk (3 frames,
    4 steps), the sigma = 0 sink pass, then N_CHUNKS one-frame chunks of 4
    steps, each step a rope/append + chunk attention per layer and an Euler
    update of the chunk's latent.  One bench step = the whole schedule."""
    import torch
    from same_step_kv_b200 import pv, synth
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()
    NL = args.layers
    cfg = pv.make_config(NL, HEADS, D, W, HH, ring_slots=R, max_streams=1, max_frames=64)
    store = pv.KVStore(cfg, device=dev)
    h = store.handle
    big = [synth.chunk_qkv(rank, 0, i, 0, 3 * T, HEADS, D, dev) for i in range(POOL)]
    small = [synth.chunk_qkv(rank, 1, i, 0, T, HEADS, D, dev) for i in range(POOL)]
    q_rot = torch.empty(HEADS * 3 * T * D, dtype=torch.bfloat16, device=dev)
    out = torch.empty(3 * T, HEADS, D, dtype=torch.bfloat16, device=dev)
    x = synth.latent(rank, 3 + N_CHUNKS, 48, 44, 80, dev).reshape(-1)
    vel = synth.velocity(rank, 0, 0, 3 * LATENT, dev)
    sig = [1.0, 0.75, 0.5, 0.25, 0.0]
    new_state = pv.pv_kv_state()
    new_state.phase, new_state.chunk = pv.PV_PHASE_NEW, -1

    def keys(j):  # key count of chunk j >= 1 at any step
        return 3 * T + min(j, R) * T

    flops = 4 * NL * (4 + 1) * (3 * T) ** 2 * HEADS * D
    flops += sum(4 * NL * 4 * T * keys(j) * HEADS * D for j in range(1, N_CHUNKS + 1))
    attn_ev = []

    def layer_pass(j, s, n, inputs, record):
        step_arg = pv.PV_STEP_SINK if s is None else s
        for layer in range(NL):
            q, k, v = inputs[(j * 7 + (0 if s is None else s) * 3 + layer) % POOL]
            pv.pv_rope_append(h, [0], layer, step_arg, q, k, v, q_rot, cs)
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(cs)
            pv.pv_chunk_attn(h, [0], layer, step_arg, q_rot[: HEADS * n * D], out[:n], None, cs)
            if record:
                e1.record(cs)
                attn_ev.append((e0, e1))

    def step(record):
        pv.pv_kv_set_state(h, 0, new_state)
        pv.pv_kv_begin_chunk(h, 0, 3)
        for s in range(4):
            layer_pass(0, s, 3 * T, big, record)
            pv.pv_euler_step(x[: 3 * LATENT], vel, 3 * LATENT, sig[s + 1] - sig[s], cs)
        pv.pv_kv_begin_sink(h, 0)
        layer_pass(0, None, 3 * T, big, record)
        for j in range(1, N_CHUNKS + 1):
            pv.pv_kv_begin_chunk(h, 0, 1)
            xj = x[(2 + j) * LATENT:(3 + j) * LATENT]
            for s in range(4):
                layer_pass(j, s, T, small, record)
                pv.pv_euler_step(xj, vel[:LATENT], LATENT, sig[s + 1] - sig[s], cs)

    # the schedule timed without per-launch events (3,510 pairs would add to
    # it), then one more pass with them for the attention kernel's own time
    ms_step, clocks = timed_steps(lambda record: step(False), args, local, world, cs)
    step(True)
    torch.cuda.synchronize()
    attn_ms = sum(a.elapsed_time(b) for a, b in attn_ev)
    # e2e: the latent from pinned host memory and back, every input set too
    hx = x.cpu().pin_memory()
    hpool = [[t.cpu().pin_memory() for t in qkv] for qkv in big + small]
    dpool = big + small

    def e2e_step(record):
        x.copy_(hx, non_blocking=True)
        for dst, src in zip(dpool, hpool):
            for a, b in zip(dst, src):
                a.copy_(b, non_blocking=True)
        step(False)
        hx.copy_(x, non_blocking=True)

    e2e_ms, _ = timed_steps(e2e_step, args, local, world, cs)
    h2d = x.numel() * 4 + sum(t.numel() * 2 for qkv in dpool for t in qkv)
    launches = 2 * NL * (4 + 1 + 4 * N_CHUNKS) + 4 * (1 + N_CHUNKS)
    if rank == 0:
        peaks, src = load_peaks()
        achieved = flops / (attn_ms * 1e-3) / 1e12
        line = {
            "metric": "chunk-attention TFLOP/s over the whole generation schedule; latent frames/s",
            "value": flops * world / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"whole schedule: first chunk 3 x 880 tokens (4 steps) + sink "
                                   f"pass + {N_CHUNKS} chunks x 880 tokens x 4 steps, ring {R}, "
                                   f"24x128, {NL} layers, Euler on 48x44x80 per frame",
                       "l2": "K/V store of %.1f GB, no flush" % (store.kv_bytes / 1e9)},
            "latent_frames_per_s": world * (3 + N_CHUNKS) / (ms_step * 1e-3),
            "roofline": tensor_roofline(
                achieved, peaks, src, clocks, ms_step * args.steps * 1e-3,
                "attn_kernel<128> (every pv_chunk_attn of the schedule)",
                ms_attention_per_step=attn_ms),
            "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": x.numel() * 4},
            "gpu_launches": args.steps * launches, "clocks": clocks, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    store.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: step 100, schedule 3, dense 20, multistream 20, "
                         "cross_attn 400, sampler 2000, qkv 50)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layers per step (30 in the profile; fewer only for small ncu captures)")
    ap.add_argument("--workload", default="step",
                    choices=["step", "schedule", "dense", "multistream", "cross_attn", "sampler",
                             "qkv"],
                    help="step: the same-step KV chunk step (default); schedule: the whole "
                         "29-chunk generation of one stream; dense: whole-video attention "
                         "(18,480 tokens); multistream: 8 streams at ragged ring fills in "
                         "one launch; cross_attn, sampler, qkv: the "
                         "cross-attention, sampler-variant and q/k/v projection kernels on "
                         "their own")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = {"step": 100, "schedule": 3, "dense": 20, "multistream": 20,
                      "cross_attn": 400, "sampler": 2000, "qkv": 50}[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3
    NL = args.layers
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.workload != "step":
        {"schedule": run_schedule, "dense": run_dense, "multistream": run_multistream,
         "cross_attn": run_cross_attn, "sampler": run_sampler, "qkv": run_qkv}[args.workload](
            args, rank, world, local)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import torch
    import torch.distributed as dist
    from same_step_kv_b200 import pv, synth
    from same_step_kv_b200.dist import max_over_ranks

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    cs = torch.cuda.current_stream()

    # ---- setup: store with every layer's history at the steady state
    cfg = pv.make_config(NL, HEADS, D, W, HH, ring_slots=R, max_streams=1, max_frames=64)
    store = pv.KVStore(cfg, device=dev)
    h = store.handle
    st = pv.pv_kv_state()
    st.phase, st.chunk = pv.PV_PHASE_STEADY, CHUNK
    pv.pv_kv_set_state(h, 0, st)
    Kr, Vr = store.k_region(), store.v_region()
    for layer in range(NL):
        kf, vf = synth.store_fill(rank, layer, STEP, HEADS, N_KEYS, D, dev)
        Kr[layer, STEP, 0] = kf
        Vr[layer, STEP, 0] = vf
    del kf, vf
    qkv = [synth.chunk_qkv(rank, CHUNK, STEP, layer, T, HEADS, D, dev) for layer in range(NL)]
    q_rot = torch.empty(HEADS * T * D, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, HEADS, D, dtype=torch.bfloat16, device=dev)
    x = synth.latent(rank, 1, 48, 44, 80, dev).reshape(-1)
    vel = synth.velocity(rank, CHUNK, STEP, LATENT, dev)
    dsigma = 0.25 - 0.5

    attn_ev = []

    def step(record=False):
        for layer in range(NL):
            q, k, v = qkv[layer]
            pv.pv_rope_append(h, [0], layer, STEP, q, k, v, q_rot, cs)
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(cs)
            pv.pv_chunk_attn(h, [0], layer, STEP, q_rot, out, None, cs)
            if record:
                e1.record(cs)
                attn_ev.append((e0, e1))
        pv.pv_euler_step(x, vel, LATENT, dsigma, cs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(cs)
        for _ in range(args.steps):
            step(record=True)
        t1.record(cs)
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_ev)
    ms = max_over_ranks(ms)       # the slowest rank sets the job's time
    ms_step = ms / args.steps

    # ---- e2e: the same step through the public API from pinned host buffers
    hq = [tuple(t.cpu().pin_memory() for t in qkv[l]) for l in range(NL)]
    hv = vel.cpu().pin_memory()
    hx = x.cpu().pin_memory()
    hres = torch.empty(LATENT, dtype=torch.float32).pin_memory()
    dq = [tuple(torch.empty_like(t) for t in qkv[0]) for _ in range(2)]
    dv = torch.empty_like(vel)
    copy_s = torch.cuda.Stream(device=dev)
    done = [torch.cuda.Event() for _ in range(2)]
    used = [torch.cuda.Event() for _ in range(2)]

    def e2e_step():
        with torch.cuda.stream(copy_s):
            dv.copy_(hv, non_blocking=True)
        for layer in range(NL):
            b = layer % 2
            with torch.cuda.stream(copy_s):
                if layer >= 2:
                    copy_s.wait_event(used[b])
                for dst, src in zip(dq[b], hq[layer]):
                    dst.copy_(src, non_blocking=True)
                done[b].record(copy_s)
            cs.wait_event(done[b])
            q, k, v = dq[b]
            pv.pv_rope_append(h, [0], layer, STEP, q, k, v, q_rot, cs)
            used[b].record(cs)
            pv.pv_chunk_attn(h, [0], layer, STEP, q_rot, out, None, cs)
        pv.pv_euler_step(x, dv, LATENT, dsigma, cs)
        hres.copy_(x, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    for _ in range(args.steps):
        e2e_step()
    e1.record(cs)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    e2e_ms = max_over_ranks(e2e_ms)
    h2d = NL * 3 * T * HEADS * D * 2 + LATENT * 4
    d2h = LATENT * 4

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inputs = oracle_inputs()
        runs = [oracle_sample(inputs) for _ in range(4)]
        fl, dt = runs[0][0], statistics.median(r[1] for r in runs)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": runs[0][2], "kind": "oracle",
               "sample": "one of the 30 layers of a step (RoPE + 880 x 18480 attention, "
                         "24 heads), median of 4 runs",
               "cpu_model": cpu_model(), "one_core": oracle_one_core()}

    if rank == 0:
        peaks, src = load_peaks()
        step_flops = NL * ATTN_FLOPS * world
        value = step_flops / (ms_step * 1e-3) / 1e12
        achieved = ATTN_FLOPS / (attn_ms * 1e-3) / 1e12
        clocks = clk.summary()
        peak = tensor_peak(peaks, src, clocks, ms_step * args.steps * 1e-3)[0]
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD if NL == LAYERS else WORKLOAD.replace("30 layers", f"{NL} layers"), "heads": HEADS, "head_dim": D, "queries": T,
                       "keys": N_KEYS, "layers": NL,
                       "l2": "inputs larger than L2 (6.9 GB of K/V per step), no flush"},
            "latent_frames_per_s": world / (ms_step * 1e-3),
            "pct_of_bf16_peak": 100.0 * value / peak,
            "roofline": tensor_roofline(achieved, peaks, src, clocks, ms_step * args.steps * 1e-3,
                                        "attn_kernel<128> (pv_chunk_attn)",
                                        ms_per_launch=attn_ms, traffic=profiled_traffic()),
            "e2e": {"value": step_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * (2 * NL + 1),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    store.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
