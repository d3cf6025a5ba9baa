"""Benchmark of the tokenizer hot path on B200: Haar patcher + unpatcher + FSQ encode + decode.

One step = tok_haar_fwd and tok_haar_inv on a 121-frame 704x1280 bf16 clip
([1,3,121,704,1280] -> [1,192,31,176,320] -> back), then tok_fsq_encode and
tok_fsq_decode on the 64-clip latent grid of that geometry ([64,16,16*44*80]
fp32, 16 -> 6 projection, levels (8,8,8,5,5,5)).  Inputs are seeded synthetic
data resident in HBM; every input (654 MB clip, 231 MB latent) is larger than
the 126 MB L2, so nothing is flushed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU, weak scaling)

Rank 0 prints one JSON line.  ``value`` is algorithmic bytes moved per second
(GB/s) summed over all ranks, timed on the device with CUDA events between
barriers, max over ranks.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload on the host cores instead.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Haar fwd/inv + FSQ enc/dec GB/s & Mvoxel/s at 121x704x1280 bf16; % HBM peak"
CLIP = (1, 3, 121, 704, 1280)          # bf16 clip
LATENT = (64, 16, 16 * 44 * 80)        # fp32 latent grid: 64 clips at 8x16x16 compression
FALLBACK_HBM_GBS = 6650.0
# Bounded sample for the CPU oracle: the first 33 frames of the clip, 8 of the 64 latent grids.
CPU_SAMPLE_FRAMES = 33
CPU_SAMPLE_GRIDS = 8


def haar_bytes(shape, elem=2):
    B, C, T, H, W = shape
    tq = 1 if T == 1 else 1 + (T - 1) // 4
    nx = B * C * T * H * W
    ny = B * C * (16 if T == 1 else 64) * tq * (H // 4) * (W // 4)
    return nx * elem, ny * elem


def fsq_bytes(shape):
    B, C, S = shape
    return B * C * S * 4, B * S * 4


def step_bytes(clip=CLIP, latent=LATENT):
    hx, hy = haar_bytes(clip)
    fu, fi = fsq_bytes(latent)
    return {"haar_fwd": hx + hy, "haar_inv": hx + hy, "fsq_encode": fu + fi, "fsq_decode": fu + fi}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# The sources each timed kernel is compiled from (its .cu file and the headers it includes).
KERNEL_SOURCES = {
    "haar_fwd": ("haar_tma.cu", "tma.cuh", "tok_common.cuh", "tok_internal.h"),
    "haar_inv": ("haar_tma.cu", "tma.cuh", "tok_common.cuh", "tok_internal.h"),
    "fsq_encode": ("fsq.cu", "tma.cuh", "tok_common.cuh", "tok_internal.h"),
    "fsq_decode": ("fsq.cu", "tma.cuh", "tok_common.cuh", "tok_internal.h"),
}


def kernel_source_digest(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "haar_wavelet_patching_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    digest = kernel_source_digest(kernel)
    for ln in lines:
        parts = [p.strip() for p in ln.strip().strip("|").split("|")]
        if len(parts) >= 3 and parts[0] == kernel and parts[2] == digest:
            try:
                return float(parts[1])
            except ValueError:
                return None
    return None


def earlier_traffic(kernel):
    """The newest recorded row of a kernel taken on other sources than the current ones, as
    {"bytes", "digest", "current_digest"}, or None: shown beside a null roofline.traffic so
    that the last capture stays visible, labelled as not describing the current build."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    digest = kernel_source_digest(kernel)
    for ln in lines:
        parts = [p.strip() for p in ln.strip().strip("|").split("|")]
        if len(parts) >= 3 and parts[0] == kernel and parts[2] != digest:
            try:
                return {"bytes": float(parts[1]), "digest": parts[2], "current_digest": digest}
            except ValueError:
                continue
    return None


def max_over_ranks(v: float, device) -> float:
    """Max of a per-rank time over the default process group (any backend); v itself on one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return v
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Weak scaling: every rank moves bytes_per_step per step; GB/s of the whole job over the slowest rank."""
    return world * bytes_per_step * steps / (max_ms / 1e3) / 1e9


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=5)
        rows = [ln for ts, ln in self.lines if t0 - 0.15 <= ts <= t1 + 0.15] or [ln for _, ln in self.lines[-3:]]
        mhz, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            f = [v.strip() for v in r.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ---------------------------------------------------------------------------
# The CPU oracle on a bounded sample (cpu_baseline and --impl reference).
# ---------------------------------------------------------------------------
def oracle_sample_inputs(frames=CPU_SAMPLE_FRAMES, grids=CPU_SAMPLE_GRIDS):
    import synth
    clip = synth.smooth_field((1, 3, frames, 704, 1280), seed=3)  # the first frames of the benchmark clip
    lat = synth.fsq_input(4)[:grids]
    return synth.bf16_bits_to_f64(clip), lat, synth.fsq_weight()


def oracle_step(x64, lat, w):
    import oracle
    y = oracle.haar_fwd(x64)
    oracle.haar_inv(y, *x64.shape[2:])
    idx, _, _ = oracle.fsq_encode(lat, w)
    oracle.fsq_decode(idx, w)


def oracle_sample_bytes(frames=CPU_SAMPLE_FRAMES, grids=CPU_SAMPLE_GRIDS):
    b = step_bytes((1, 3, frames, 704, 1280), (grids,) + LATENT[1:])
    return sum(b.values())


def sample_text(frames, grids):
    return (f"clip frames [0,{frames}) of [1,3,121,704,1280] bf16 (Haar fwd+inv) and {grids} of 64 latent "
            f"grids (FSQ enc+dec); single-threaded C oracle in double")


def cpu_baseline(reps=3):
    x64, lat, w = oracle_sample_inputs()
    oracle_step(x64, lat, w)  # load / warm
    t = time.perf_counter()
    for _ in range(reps):
        oracle_step(x64, lat, w)
    dt = (time.perf_counter() - t) / reps
    return {"value": round(oracle_sample_bytes() / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{sample_text(CPU_SAMPLE_FRAMES, CPU_SAMPLE_GRIDS)}; {reps} reps of {dt:.2f} s"}


def oracle_step_parts(x64, lat, w, windows_per_part=1):
    """The oracle step split into independent parts for a thread pool: per clip channel, the
    windows in groups (the first chunk with the frame-0 replica, then chunks of 4k frames, the
    oracle's streaming calls: together exactly the whole clip's transform), and the FSQ calls
    per latent grid.  Each part returns its outputs (for the equivalence test)."""
    import oracle
    B, C, T, H, W = x64.shape
    parts = []
    for c in range(C):
        f0 = 0
        while f0 < T:
            first = f0 == 0
            f1 = min(T, (1 if first else f0) + 4 * windows_per_part)

            def haar_part(c=c, f0=f0, f1=f1, first=first):
                xs = x64[:, c:c + 1, f0:f1]
                y = oracle.haar_fwd_chunk(xs, first)
                return ("haar", c, f0, y, oracle.haar_inv_chunk(y, f1 - f0, H, W, first))
            parts.append(haar_part)
            f0 = f1
    for g in range(lat.shape[0]):
        def fsq_part(g=g):
            idx, _, _ = oracle.fsq_encode(lat[g:g + 1], w)
            return ("fsq", g, idx, oracle.fsq_decode(idx, w)[0])
        parts.append(fsq_part)
    return parts


def cpu_baseline_threads(reps=3):
    """The same sample as cpu_baseline, its independent parts on a pool of the host's cores
    (ctypes releases the interpreter lock during each oracle call)."""
    from concurrent.futures import ThreadPoolExecutor
    x64, lat, w = oracle_sample_inputs()
    parts = oracle_step_parts(x64, lat, w)
    cores = len(os.sched_getaffinity(0))
    with ThreadPoolExecutor(max_workers=cores) as pool:
        list(pool.map(lambda f: f(), parts))  # warm
        t = time.perf_counter()
        for _ in range(reps):
            list(pool.map(lambda f: f(), parts))
        dt = (time.perf_counter() - t) / reps
    return {"value": round(oracle_sample_bytes() / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{sample_text(CPU_SAMPLE_FRAMES, CPU_SAMPLE_GRIDS).replace('single-threaded', 'the same')}, "
                      f"split into {len(parts)} independent parts on {cores} threads; {reps} reps of {dt:.2f} s"}


def reference_sample(steps, warmup, budget_s=150.0):
    """Per-step sample (frames = 1 + 4m, grids) sized so steps + warmup oracle passes take about budget_s."""
    x64, lat, w = oracle_sample_inputs(5, 1)
    t = time.perf_counter()
    oracle_step(x64, lat, w)
    probe = time.perf_counter() - t
    scale = budget_s / max(steps + warmup, 1) / max(probe, 1e-3)
    m = int(max(1, min(30, scale)))          # latent frames beyond the first, up to the whole clip
    grids = int(max(1, min(64, scale)))
    return 1 + 4 * m, grids


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    frames, grids = reference_sample(args.steps, args.warmup)
    x64, lat, w = oracle_sample_inputs(frames, grids)
    for _ in range(args.warmup):
        oracle_step(x64, lat, w)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(x64, lat, w)
    dt = (time.perf_counter() - t) / max(args.steps, 1)
    value = oracle_sample_bytes(frames, grids) / dt / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "per step: " + sample_text(frames, grids)},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def workload_config():
    return {"workload": "clip [1,3,121,704,1280] bf16 Haar fwd+inv; latent [64,16,16x44x80] fp32 FSQ enc+dec",
            "clip": list(CLIP), "coeffs": [1, 192, 31, 176, 320], "latent": list(LATENT), "levels": [8, 8, 8, 5, 5, 5],
            "fsq_codes_output": False, "l2": "no flush: every input is larger than the 126 MB L2",
            "parallelism": "data-parallel replicas, one per GPU"}


# ---------------------------------------------------------------------------
# GPU arm.
# ---------------------------------------------------------------------------
E2E_CHUNKS = 8
_H2D, _D2H = 1, 2


def _memcpy2d():
    """cudaMemcpy2DAsync of the CUDA runtime torch has loaded (strided chunk copies)."""
    import ctypes
    f = ctypes.CDLL("libcudart.so.12").cudaMemcpy2DAsync
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_size_t,
                  ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
    return f


def chunk_bounds(n, k):
    """k contiguous, nearly equal chunks of range(n)."""
    edges = [round(i * n / k) for i in range(k + 1)]
    return [(edges[i], edges[i + 1]) for i in range(k) if edges[i + 1] > edges[i]]


def make_e2e_step(torch, hwp, x_host, u_host, w_dev, x, y, xr, u, idx, ur, y_host, xr_host, idx_host, ur_host, dev):
    memcpy2d = _memcpy2d()
    B, C, T, H, W = x.shape
    Tq, h, w = y.shape[2:]
    G = y.shape[1] // C
    es = x.element_size()
    win = chunk_bounds(Tq, E2E_CHUNKS)
    grids = chunk_bounds(u.shape[0], len(win))
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in win]
    ev_cmp = [torch.cuda.Event() for _ in win]
    ev_out = [torch.cuda.Event() for _ in win]
    state = {"first": True}

    def frames(a, b):  # pixel frames [f0, f1) of latent windows [a, b), b > a
        return (0 if a == 0 else 4 * a - 3), 4 * b - 3

    def copy2d(dst, src, pitch, off, width, rows, kind, st):
        rc = memcpy2d(dst + off, pitch, src + off, pitch, width, rows, kind, st.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"cudaMemcpy2DAsync failed: {rc}")

    def step(start_after=None):
        for j, ((a, b), (g0, g1)) in enumerate(zip(win, grids)):
            f0, f1 = frames(a, b)
            if start_after is not None:
                s_in.wait_event(start_after)
            if not state["first"]:
                s_in.wait_event(ev_cmp[j])   # the previous step's kernels are done with chunk j's inputs
            copy2d(x.data_ptr(), x_host.data_ptr(), T * H * W * es, f0 * H * W * es, (f1 - f0) * H * W * es,
                   B * C, _H2D, s_in)
            with torch.cuda.stream(s_in):
                u[g0:g1].copy_(u_host[g0:g1], non_blocking=True)
            ev_in[j].record(s_in)
            s_cmp.wait_event(ev_in[j])
            if not state["first"]:
                s_cmp.wait_event(ev_out[j])  # the previous step's copies out of chunk j are done
            hwp.tok_haar_fwd_windows(x, y, a, b, stream=s_cmp)
            hwp.tok_haar_inv_windows(y, xr, a, b, stream=s_cmp)
            hwp.tok_fsq_encode(u[g0:g1], w_dev, idx[g0:g1], stream=s_cmp)
            hwp.tok_fsq_decode(idx[g0:g1], w_dev, ur[g0:g1], stream=s_cmp)
            ev_cmp[j].record(s_cmp)
            s_out.wait_event(ev_cmp[j])
            copy2d(y_host.data_ptr(), y.data_ptr(), Tq * h * w * es, a * h * w * es, (b - a) * h * w * es,
                   B * G * C, _D2H, s_out)
            copy2d(xr_host.data_ptr(), xr.data_ptr(), T * H * W * es, f0 * H * W * es, (f1 - f0) * H * W * es,
                   B * C, _D2H, s_out)
            with torch.cuda.stream(s_out):
                idx_host[g0:g1].copy_(idx[g0:g1], non_blocking=True)
                ur_host[g0:g1].copy_(ur[g0:g1], non_blocking=True)
            ev_out[j].record(s_out)
        state["first"] = False

    def join(st):
        st.wait_event(ev_out[-1])
        st.wait_event(ev_cmp[-1])
        st.wait_event(ev_in[-1])

    step.join = join
    return step
GRAD_ITERS = 20


def time_gradients(torch, hwp, stream, x, y, xr, u, idx, ur, w_dev, dev, iters=GRAD_ITERS):
    """The gradient calls on the headline workload, each timed alone (CUDA events on the
    launching stream, mean over `iters` launches after one warm-up), outside the step's timed
    region.  Buffers of the step are reused as inputs and outputs; returns per call the mean ms,
    the algorithmic bytes per call (inputs read once, outputs written once; the FSQ workspace
    rows are not counted) and the kernel launches per call."""
    B, _, S = u.shape
    g6 = torch.randn(B, 6, S, device=dev, generator=torch.Generator(device=dev).manual_seed(7))
    gcodes = torch.empty_like(g6)
    gw = torch.empty_like(w_dev)
    ws = torch.empty(max(hwp.fsq_backward_workspace_size(B, u.shape[1], S), 1), dtype=torch.uint8, device=dev)
    hb = x.numel() * x.element_size() + y.numel() * y.element_size()
    calls = {
        "haar_fwd_adjoint": (lambda: hwp.tok_haar_fwd_adjoint(y, xr), hb, 1),
        "haar_inv_adjoint": (lambda: hwp.tok_haar_inv_adjoint(x, y), hb, 1),
        "fsq_encode_backward": (lambda: hwp.tok_fsq_encode_backward(u, w_dev, g6, ur, gw, ws),
                                (2 * u.numel() + g6.numel()) * 4, 2),
        "fsq_decode_backward": (lambda: hwp.tok_fsq_decode_backward(idx, w_dev, u, gcodes, gw, ws),
                                (u.numel() + idx.numel() + gcodes.numel()) * 4, 2),
    }
    out = {}
    for name, (call, nbytes, launches) in calls.items():
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = {"ms": max_over_ranks(e0.elapsed_time(e1) / iters, dev), "bytes": nbytes, "launches": launches}
    return out


STREAM_CLIP = (1, 3, 120, 720, 1280)  # 120 frames: one mirrored frame makes 121; also 30 continuation windows


def time_single(torch, hwp, stream, x, dev, iters=GRAD_ITERS):
    """The single-level patcher / unpatcher (patch_size=2) on the headline clip, timed alone:
    [1,3,121,704,1280] <-> [1,24,61,352,640] bf16; algorithmic bytes: the clip plus the
    coefficients, each once."""
    y1 = torch.empty(hwp.single_coeff_shape(*x.shape), dtype=x.dtype, device=dev)
    xr = torch.empty_like(x)
    nbytes = (x.numel() + y1.numel()) * x.element_size()
    out = {}
    for name, call in (("haar_fwd_single", lambda: hwp.tok_haar_fwd_single(x, y1)),
                       ("haar_inv_single", lambda: hwp.tok_haar_inv_single(y1, xr))):
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = {"ms": max_over_ranks(e0.elapsed_time(e1) / iters, dev), "bytes": nbytes}
    del y1, xr
    return out


CONV_CH = (256, 256)  # C_mid, C_out of the factorized convolution after the patcher (k = 3)


def time_patch_embed(torch, hwp, stream, x, dev, iters=10):
    """The patcher's channels-last output feeding the first causal factorized convolution
    (1x3x3 then 3x1x1 causal) on the headline clip, each call timed alone: flops of the two
    implicit GEMMs, 2 * positions * (C_mid * 9 * C_in + C_out * 3 * C_mid).  patch_embed_fused
    is the patcher fused into the 1x3x3 convolution (one kernel, pixels in, the spatial layer's
    output out): the same flops as conv_spatial, the work of haar_fwd_channels_last + conv_spatial."""
    B, C, T, H, W = x.shape
    Cmid, Cout = CONV_CH
    y_cl = torch.empty(hwp.channels_last_shape(B, C, T, H, W), dtype=torch.bfloat16, device=dev)
    Bq, Tq, h, w, Cin = y_cl.shape
    g = torch.Generator(device=dev).manual_seed(13)
    ws = (torch.randn((Cmid, 3, 3, Cin), generator=g, device=dev) * (9 * Cin) ** -0.5).to(torch.bfloat16)
    wt = (torch.randn((Cout, 3, Cmid), generator=g, device=dev) * (3 * Cmid) ** -0.5).to(torch.bfloat16)
    mid = torch.empty((Bq, Tq, h, w, Cmid), dtype=torch.bfloat16, device=dev)
    mid2 = torch.empty_like(mid)
    out = torch.empty((Bq, Tq, h, w, Cout), dtype=torch.bfloat16, device=dev)
    wp = hwp.patch_embed_pack_weights(ws)  # once per filter, outside the timed calls
    pos = Bq * Tq * h * w
    calls = {
        "patch_embed_fused": (lambda: hwp.tok_patch_embed_spatial(x, wp, mid2), 2 * pos * Cmid * 9 * Cin,
                              (x.numel() + mid2.numel()) * 2, 1),
        "haar_fwd_channels_last": (lambda: hwp.tok_haar_fwd_channels_last(x, y_cl), 0,
                                   (x.numel() + y_cl.numel()) * 2, 1),
        "conv_spatial": (lambda: hwp.tok_conv_spatial(y_cl, ws, mid), 2 * pos * Cmid * 9 * Cin,
                         (y_cl.numel() + mid.numel()) * 2, 1),
        "conv_temporal_causal": (lambda: hwp.tok_conv_temporal_causal(mid, wt, out), 2 * pos * Cout * 3 * Cmid,
                                 (mid.numel() + out.numel()) * 2, 1),
    }
    res = {}
    for name, (call, flops, nbytes, launches) in calls.items():
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        res[name] = {"ms": max_over_ranks(e0.elapsed_time(e1) / iters, dev), "flops": flops, "bytes": nbytes}
    del y_cl, mid, mid2, out
    return res


def time_streaming(torch, hwp, stream, dev, iters=GRAD_ITERS):
    """The arbitrary-extent and streaming calls on a 120-frame 720p clip (bf16), each timed alone
    like the gradients: the padded patcher / cropped unpatcher (spatial multiple 16, temporal 8:
    one frame mirrored in, 121 frames' worth of windows) and the same 120 frames as one
    continuation chunk (30 windows, no replica).  Algorithmic bytes: the clip read or written once
    plus the coefficients written or read once."""
    B, C, T, H, W = STREAM_CLIP
    g = torch.Generator(device=dev).manual_seed(11)
    x = (torch.rand(STREAM_CLIP, generator=g, device=dev) * 2 - 1).to(torch.bfloat16)
    xr = torch.empty_like(x)
    yp = torch.empty(hwp.padded_coeff_shape(B, C, T, H, W, 16, 8), dtype=torch.bfloat16, device=dev)
    yc = torch.empty(hwp.chunk_coeff_shape(B, C, T, H, W, False), dtype=torch.bfloat16, device=dev)
    xb = x.numel() * 2
    calls = {
        "haar_fwd_padded": (lambda: hwp.tok_haar_fwd_padded(x, yp, 16, 8), xb + yp.numel() * 2),
        "haar_inv_cropped": (lambda: hwp.tok_haar_inv_cropped(yp, xr, 16, 8), xb + yp.numel() * 2),
        "haar_fwd_chunk": (lambda: hwp.tok_haar_fwd_chunk(x, yc, False), xb + yc.numel() * 2),
        "haar_inv_chunk": (lambda: hwp.tok_haar_inv_chunk(yc, xr, False), xb + yc.numel() * 2),
    }
    out = {}
    for name, (call, nbytes) in calls.items():
        call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = {"ms": max_over_ranks(e0.elapsed_time(e1) / iters, dev), "bytes": nbytes, "launches": 1}
    return out


STRESS_ITERS = 10


def _flush_l2(torch, bufs):
    """Evict L2 between timed kernels: write one buffer larger than L2, then read another, so
    the next kernel starts with neither its inputs nor dirty lines of the flush in L2."""
    bufs[0].zero_()
    bufs[1].sum()


def time_sequence(torch, stream, calls, iters, flush=None):
    """Run the calls back to back on one stream `iters` times after one warm-up pass, an event
    pair around each call (a flush, if given, runs between calls outside the events); returns
    the mean ms per call."""
    for _, call in calls:
        call()
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
           for _ in range(iters)]
    for k in range(iters):
        for (_, call), (e0, e1) in zip(calls, evs[k]):
            if flush is not None:
                flush()
            e0.record(stream)
            call()
            e1.record(stream)
    torch.cuda.synchronize()
    return {name: float(np.mean([evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(iters)]))
            for i, (name, _) in enumerate(calls)}


def stress_inputs(torch, cfg, dev):
    """Seeded host inputs of a Haar config (pinned, then copied once to the device) and the
    latent of the matching FSQ config."""
    import synth
    shape = synth.HAAR_CONFIGS[cfg]["shape"]
    x_host = torch.empty(shape, dtype=torch.int16).pin_memory()
    synth.haar_input(cfg, out=x_host.numpy().view(np.uint16))
    x = x_host.view(torch.bfloat16).to(dev)
    del x_host
    u = torch.from_numpy(synth.fsq_input(cfg)).to(dev)
    return x, u


def time_stress(torch, hwp, stream, w_dev, dev, iters=STRESS_ITERS):
    """The throughput-stress clip and the image batch, outside the headline step.  Stress: four
    121-frame 1088x1920 clips [4,3,121,1088,1920] bf16 through the patcher and unpatcher, then
    FSQ encode + decode of the [4,16,16*68*120] latent, back to back on one stream (its Haar
    tensors are 6 GB each, so nothing survives in L2 from one call to the next; its 35 MB latent
    is L2-sized).  Image batch: the image path on [16,3,1024,1024] bf16 (2D Haar) and FSQ on
    [16,16,64*64]; none of its tensors exceeds L2, so L2 is flushed before each call (outside
    its events).  Per call: mean ms, algorithmic bytes (inputs read once, outputs written once)."""
    out = {}
    for cfg in (5, 2):
        x, u = stress_inputs(torch, cfg, dev)
        B, C, T, H, W = x.shape
        y = torch.empty(hwp.haar_coeff_shape(B, C, T, H, W), dtype=x.dtype, device=dev)
        xr = torch.empty_like(x)
        idx = torch.empty(u.shape[0], u.shape[2], dtype=torch.int32, device=dev)
        ur = torch.empty_like(u)
        hx, hy = haar_bytes(x.shape)
        fu, fi = fsq_bytes(u.shape)
        calls = [("haar_fwd", lambda: hwp.tok_haar_fwd(x, y)), ("haar_inv", lambda: hwp.tok_haar_inv(y, xr)),
                 ("fsq_encode", lambda: hwp.tok_fsq_encode(u, w_dev, idx)),
                 ("fsq_decode", lambda: hwp.tok_fsq_decode(idx, w_dev, ur))]
        nbytes = {"haar_fwd": hx + hy, "haar_inv": hx + hy, "fsq_encode": fu + fi, "fsq_decode": fu + fi}
        flush = None
        if cfg == 2:
            fb = [torch.empty(256 << 20, dtype=torch.uint8, device=dev) for _ in range(2)]
            flush = lambda: _flush_l2(torch, fb)  # noqa: E731
        ms = time_sequence(torch, stream, calls, iters, flush)
        out[cfg] = {"clip": list(x.shape), "latent": list(u.shape),
                    "calls": {n: {"ms": max_over_ranks(ms[n], dev), "bytes": nbytes[n]} for n in ms},
                    "voxels": B * T * H * W, "tokens": u.shape[0] * u.shape[2]}
        del x, u, y, xr, idx, ur
        torch.cuda.empty_cache()
    return out


def stress_report(stress, peak):
    rep = {}
    for cfg, d in stress.items():
        e = {"clip": d["clip"], "latent": d["latent"],
             "l2": "flushed before each call" if cfg == 2 else "no flush: each Haar tensor is 6 GB, back to back"}
        for n, g in d["calls"].items():
            gbs = g["bytes"] / (g["ms"] / 1e3) / 1e9
            r = {"ms": round(g["ms"], 4), "GB/s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                 "bytes": g["bytes"]}
            if n.startswith("haar"):
                r["mvoxel_per_s"] = round(d["voxels"] / g["ms"] / 1e3, 1)
            else:
                r["mtoken_per_s"] = round(d["tokens"] / g["ms"] / 1e3, 1)
            e[n] = r
        rep["stress_clip" if cfg == 5 else "image_batch"] = e
    return rep


def tensor_peak():
    """(burst, sustained) bf16 TFLOP/s from MEASURED_PEAKS.json, else the recipe's fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, "fallback"


def patch_embed_report(embed, hbm_peak):
    burst, sustained, kind = tensor_peak()
    out = {"channels": {"C_in": 192, "C_mid": CONV_CH[0], "C_out": CONV_CH[1], "k": 3},
           "tensor_peak_tflops": burst, "tensor_peak_sustained_tflops": sustained, "peak_source": kind}
    for n, g in embed.items():
        e = {"ms": round(g["ms"], 4), "GB/s": round(g["bytes"] / (g["ms"] / 1e3) / 1e9, 1)}
        if g["flops"]:
            tf = g["flops"] / (g["ms"] / 1e3) / 1e12
            e.update({"TFLOP/s": round(tf, 1), "frac_of_tensor_peak": round(tf / burst, 4),
                      "frac_of_sustained": round(tf / sustained, 4), "flops": g["flops"]})
        else:
            e["frac_of_hbm_peak"] = round(g["bytes"] / (g["ms"] / 1e3) / 1e9 / hbm_peak, 4)
        out[n] = e
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import haar_wavelet_patching_b200 as hwp
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)

    # Inputs: seeded, generated on the host, pinned, copied once to HBM.
    x_host = torch.from_numpy(synth.haar_input(3).view(np.int16)).view(torch.bfloat16).pin_memory()
    u_host = torch.from_numpy(synth.fsq_input(4)).pin_memory()
    w_dev = torch.from_numpy(synth.fsq_weight()).to(dev)
    x = x_host.to(dev)
    u = u_host.to(dev)
    y = torch.empty(hwp.haar_coeff_shape(*CLIP), dtype=torch.bfloat16, device=dev)
    xr = torch.empty_like(x)
    idx = torch.empty(LATENT[0], LATENT[2], dtype=torch.int32, device=dev)
    ur = torch.empty_like(u)
    T, H, W = CLIP[2:]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        hwp.tok_haar_fwd(x, y)
        if ev is not None:
            ev[1].record(stream)
        hwp.tok_haar_inv(y, xr)
        if ev is not None:
            ev[2].record(stream)
        hwp.tok_fsq_encode(u, w_dev, idx)
        if ev is not None:
            ev[3].record(stream)
        hwp.tok_fsq_decode(idx, w_dev, ur)
        if ev is not None:
            ev[4].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    try:
        gpu_id = f"GPU-{torch.cuda.get_device_properties(dev).uuid}"
    except (AttributeError, RuntimeError):
        gpu_id = str(local_rank)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for k in range(K):
        step(evs[k])
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    clocks = sampler.stop(t0, t1)

    total_ms = max_over_ranks(evs[0][0].elapsed_time(evs[K - 1][4]), dev)
    names = ("haar_fwd", "haar_inv", "fsq_encode", "fsq_decode")
    per = {n: float(np.mean([evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(K)])) for i, n in enumerate(names)}
    ms_per_step = total_ms / K
    sb = step_bytes()
    bytes_step = sum(sb.values())
    value = job_throughput(bytes_step, K, world, total_ms)

    # End to end through the C ABI with host buffers (pinned): every step copies the clip and the
    # latent in, runs the four calls and copies out the coefficients, the reconstruction, the indices
    # and the decoded latent.  The step is cut into E2E_CHUNKS chunks of latent frames (the windowed
    # Haar calls) and of latent grids (FSQ), so copies in, compute and copies out overlap on three
    # streams; events keep a chunk's buffers from being reused before the previous step is done.
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    xr_host = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    idx_host = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    ur_host = torch.empty(u.shape, dtype=u.dtype).pin_memory()
    h2d = x_host.numel() * 2 + u_host.numel() * 4
    d2h = y.numel() * 2 + xr.numel() * 2 + idx.numel() * 4 + ur.numel() * 4
    Ke = max(3, min(K, 10))
    e2e_step = make_e2e_step(torch, hwp, x_host, u_host, w_dev, x, y, xr, u, idx, ur, y_host, xr_host, idx_host,
                             ur_host, dev)
    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        e2e_step(start_after=e0)
    e2e_step.join(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    barrier()

    grads = time_gradients(torch, hwp, stream, x, y, xr, u, idx, ur, w_dev, dev)
    streaming = time_streaming(torch, hwp, stream, dev)
    single = time_single(torch, hwp, stream, x, dev)
    embed = time_patch_embed(torch, hwp, stream, x, dev)
    stress = time_stress(torch, hwp, stream, w_dev, dev) if not args.no_stress else None
    barrier()

    if rank != 0:
        return 0
    peak, peak_kind = measured_peak()
    dom = max(("haar_fwd", "haar_inv"), key=lambda n: per[n])
    achieved = sb[dom] / (per[dom] / 1e3) / 1e9
    voxels = CLIP[0] * CLIP[2] * CLIP[3] * CLIP[4]
    tokens = LATENT[0] * LATENT[2]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s", "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(dom), "algorithmic_bytes_per_launch": sb[dom]},
        "per_kernel": {n: {"ms": round(per[n], 4), "GB/s": round(sb[n] / (per[n] / 1e3) / 1e9, 1),
                           "frac_of_peak": round(sb[n] / (per[n] / 1e3) / 1e9 / peak, 4),
                           "bytes": sb[n]} for n in names},
        "mvoxel_per_s": {"haar_fwd": round(voxels / per["haar_fwd"] / 1e3, 1),
                         "haar_inv": round(voxels / per["haar_inv"] / 1e3, 1)},
        "mtoken_per_s": {"fsq_encode": round(tokens / per["fsq_encode"] / 1e3, 1),
                         "fsq_decode": round(tokens / per["fsq_decode"] / 1e3, 1)},
        "e2e": {"value": round(job_throughput(bytes_step, Ke, world, e2e_ms), 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke,
                "ms_per_step": round(e2e_ms / Ke, 3),
                "mode": f"pinned host buffers, {E2E_CHUNKS} chunks overlapped on 3 streams "
                        "(H2D / kernels / D2H), tok_haar_*_windows per chunk"},
        "gpu_launches": 4 * K,
        "clocks": clocks,
        "gradients": {n: {"ms": round(g["ms"], 4), "GB/s": round(g["bytes"] / (g["ms"] / 1e3) / 1e9, 1),
                          "frac_of_peak": round(g["bytes"] / (g["ms"] / 1e3) / 1e9 / peak, 4),
                          "bytes": g["bytes"], "launches": g["launches"]} for n, g in grads.items()},
        "streaming": {"clip": list(STREAM_CLIP), "dtype": "bf16",
                      **{n: {"ms": round(g["ms"], 4), "GB/s": round(g["bytes"] / (g["ms"] / 1e3) / 1e9, 1),
                             "frac_of_peak": round(g["bytes"] / (g["ms"] / 1e3) / 1e9 / peak, 4),
                             "bytes": g["bytes"]} for n, g in streaming.items()}},
        "single_level": {n: {"ms": round(g["ms"], 4), "GB/s": round(g["bytes"] / (g["ms"] / 1e3) / 1e9, 1),
                             "frac_of_peak": round(g["bytes"] / (g["ms"] / 1e3) / 1e9 / peak, 4),
                             "bytes": g["bytes"]} for n, g in single.items()},
        "patch_embed": patch_embed_report(embed, peak),
    }
    if stress is not None:
        line["stress"] = stress_report(stress, peak)
    if line["roofline"]["traffic"] is None:
        earlier = earlier_traffic(dom)
        if earlier is not None:
            line["roofline"]["traffic_earlier_sources"] = earlier
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
        line["cpu_baseline_threads"] = cpu_baseline_threads()
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stress", action="store_true", help="skip the throughput-stress clip / image batch block")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
