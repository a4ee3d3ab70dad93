#!/usr/bin/env python3
"""Benchmark of the W4A16 quantized-expert MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one call of the whole layer (router GEMV, top-k, grouping, gate/up, SiLU*up,
down, combine with the shared expert) on one batch of T synthetic tokens.  The default
workload is single-user decode: T=1, H=6144, I=2048, E=256, top-8, one shared expert,
int4 weights with per-row fp32 scales (about 19 MB per expert).  The layers rotate
through R copies at distinct HBM addresses and the tokens through R distinct batches, so
every step streams its ~177 MB of weights from HBM (more than the 126 MB L2).

The timed region replays one CUDA graph of exactly K consecutive layer calls (layer
i mod R at step i; the layers' launch chain runs unbroken through the region),
bracketed by a barrier and device synchronisation, timed with CUDA events on the launch
stream; under torchrun every rank runs its own replica (weak scaling) and rank 0 reports
the maximum time over ranks.  One JSON line is printed.

``--impl reference`` times the plain FP64 CPU oracle on the same workload instead (the
reference arm), on rank 0 only.
"""
from __future__ import annotations

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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s and achieved HBM GB/s vs peak (W4A16 decode, T=1 and T=8)"
UNIT = "tokens/s"

# workload -> (default steps, default warmup, rotating layers)
DEFAULTS = {
    "decode1": (40000, 400, 8),
    "decode8": (4000, 200, 8),
    "nvfp4_1": (20000, 400, 32),
    "nvfp4_16": (8000, 400, 16),
    "prefill512": (400, 20, 2),
    "prefill2048": (100, 5, 1),
    "batch128": (800, 20, 2),
    "decode1_topp": (20000, 400, 8),
    "tiny": (20000, 200, 8),
    "int8_1": (10000, 400, 4),
    "int8_8": (4000, 200, 4),
    "int2_1": (20000, 400, 8),
    "int2_8": (4000, 200, 8),
}

FMT_NAMES = {synth.FMT_INT4: "int4", synth.FMT_NVFP4: "nvfp4", synth.FMT_INT8: "int8",
             synth.FMT_INT2: "int2"}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}

# DRAM traffic per launch (bytes) of the dominant kernel from an ncu capture, keyed by
# workload; valid only while the kernel source hashes to the recorded value.
NCU_TRAFFIC = {
    # ncu capture of the decode gate/up kernel: dram read 113,488,896 + write 3,410,176
    # bytes per launch (a T=1 step reads the same 9 experts at E=32 as at E=256).  Taken
    # on sources 12b50175da0b6a30; the one change since (three CTAs per SM for the down
    # kernels: launch bounds and ring budget of the !GU int8-path variants) leaves the
    # gate/up kernel's code and launch configuration as they were.
    "decode1": {"kernel": "gate_up", "bytes": 116899072, "kernel_hash": "2ad01ac547573c66"},
}


def describe(w) -> str:
    fmt = "NVFP4 (E2M1 + E4M3/16 + fp32)" if w.fmt == synth.FMT_NVFP4 else f"{FMT_NAMES[w.fmt]} row-scale"
    bias = "Zipf(1.1) bias in [-0.5,0.5]" if w.bias == "zipf" else "bias U(-0.1,0.1)"
    topp = f", adaptive expert top-p {w.top_p}" if getattr(w, "top_p", 0.0) else ""
    return (f"{w.name}: T={w.T}, H={w.H}, I={w.I}, E={w.E}, top-{w.k}, {w.n_shared} shared "
            f"(I={w.I_sh}), {fmt}, {bias}, scaling {w.scaling}{topp}")


# ------------------------------------------------------------------ byte accounting
def expert_bytes(w, shared=False) -> dict:
    """Bytes of one expert's quantised weights, per matrix group."""
    H, I = w.H, (w.I_sh if shared else w.I)
    if w.fmt != synth.FMT_NVFP4:   # codes at b bits + one fp32 scale per row
        b = synth.ROWSCALED_BITS[w.fmt]
        gu = 2 * (I * H * b // 8) + 2 * I * 4
        dn = H * I * b // 8 + H * 4
    else:
        gu = 2 * (I * H // 2) + 2 * (I * H // 16) + 2 * 4
        dn = H * I // 2 + H * I // 16 + 4
    return {"gate_up": gu, "down": dn}


def algorithmic_bytes(w, U: float) -> dict:
    """Bytes the layer must move per call: the weights of the U unique routed experts and
    the shared expert, the router, x in and y out (workspace traffic excluded)."""
    r, s = expert_bytes(w), expert_bytes(w, shared=True)
    ns = w.n_shared
    router = w.E * w.H * 4 + w.E * 4 + w.T * w.H * 2
    gate_up = U * r["gate_up"] + ns * s["gate_up"] + w.T * w.H * 2
    down = U * r["down"] + ns * s["down"] + w.T * w.H * 2
    total = U * (r["gate_up"] + r["down"]) + ns * (s["gate_up"] + s["down"]) + router + w.T * w.H * 2
    weights = U * (r["gate_up"] + r["down"]) + ns * (s["gate_up"] + s["down"])
    return {"router": router, "gate_up": gate_up, "down": down, "total": total, "weights": weights}


def flops(w, assignments=None) -> float:
    """Expert and router FLOPs of one layer call; ``assignments`` = (token, expert) pairs
    that reach an expert (T*k, fewer with adaptive top-p)."""
    a = w.T * w.k if assignments is None else assignments
    return 6.0 * w.I * w.H * a + 6.0 * w.I_sh * w.H * w.T * w.n_shared + 2.0 * w.T * w.E * w.H


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def kernel_hash() -> str:
    """Hash of the sources the decode expert kernels are built from: the shared device
    helpers and parameter blocks, and moe_ffn.cu without its tensor-memory section (a
    separate kernel for larger batches), so that an ncu capture of the decode kernels
    stays attached to exactly the code it measured."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w4a16_quantized_expert_b200", "csrc")
    for f in ("moe_device.cuh", "moe_internal.h", "moe_expert.cuh", "moe_ffn.cu"):
        txt = open(os.path.join(csrc, f), "rb").read()
        if f == "moe_ffn.cu":
            a = txt.find(b"// ============================================================================ tcgen05 path")
            b = txt.find(b"// ---------------------------------------------------------------------------- test hook")
            if a >= 0 and b > a:
                txt = txt[:a] + txt[b:]
        h.update(txt)
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples every 200 ms while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark(self):
        return time.time()

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float) -> dict:
        sm, mx, reasons = [], None, set()
        for ts, line in self.rows:
            if not (t0 - 0.25 <= ts <= t1 + 0.25):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed
def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    """The largest of the ranks' values (device timings are reported as the max)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, steps: int, T: int, ms_max: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of T tokens (weak scaling);
    the job takes the slowest rank's time."""
    return world * steps * T / (ms_max / 1000.0)


# ------------------------------------------------------------------ CPU baseline (oracle)
def oracle_tokens_per_s(w, host, xs, seconds: float = 10.0) -> dict:
    """The FP64 oracle as it stands, on full tokens of the same workload, for about
    ``seconds`` of CPU time (at least one token)."""
    import oracle
    o = oracle.default()
    desc = oracle.desc_of(w)
    n, t0 = 0, time.perf_counter()
    while True:
        x = xs[n % len(xs)]
        o.forward_token(desc, host, x[n // len(xs) % x.shape[0]])
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": n / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} full tokens of {w.name} through the FP64 oracle ({el:.1f} s)"}


# ------------------------------------------------------------------ reference arm
def run_reference(args, w):
    """Reference arm: the FP64 CPU oracle times K steps of the same workload.  Each step
    is a bounded sample: the full router + top-k of one batch, and every routed and shared
    expert on a slice of rows (gate/up: the first R of I rows; down: all H rows over the
    first R of I inputs), extrapolated by I/R.  R is chosen so that K steps take about
    two minutes."""
    import oracle
    o = oracle.default()
    desc = oracle.desc_of(w)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    host = synth.make_layer(w)
    xs = [synth.make_tokens(w, batch=b) for b in range(4)]
    # one full token, to size the sample
    t0 = time.perf_counter()
    o.forward_token(desc, host, xs[0][0])
    t_tok = time.perf_counter() - t0
    budget = 120.0
    per_step = budget / max(1, args.steps + args.warmup)
    tok_per_step = w.T
    frac = min(1.0, per_step / (t_tok * tok_per_step))
    R = max(16, int(round(w.I * frac / 16)) * 16)
    R = min(R, w.I)
    frac = R / w.I
    Rs = max(16, min(w.I_sh, int(round(w.I_sh * frac / 16)) * 16))

    def sliced(e):
        if e is None:
            g, u, d = host["sh_g"], host["sh_u"], host["sh_d"]
            key = "sh_"
            I_ = w.I_sh
            RR = Rs
        else:
            g, u, d = host["g"][e], host["u"][e], host["d"][e]
            key = ""
            I_ = w.I
            RR = R
        out = []
        if w.fmt != synth.FMT_NVFP4:
            f, nb = w.fmt, RR * synth.ROWSCALED_BITS[w.fmt] // 8   # code bytes of RR inputs
            sc = (host[key + "sg"], host[key + "su"], host[key + "sd"]) if e is None else \
                 (host["sg"][e], host["su"][e], host["sd"][e])
            out.append({"format": f, "codes": np.ascontiguousarray(g[:RR]), "row_scale": sc[0][:RR]})
            out.append({"format": f, "codes": np.ascontiguousarray(u[:RR]), "row_scale": sc[1][:RR]})
            out.append({"format": f, "codes": np.ascontiguousarray(d[:, :nb]), "row_scale": sc[2]})
        else:
            if e is None:
                bs = (host["sh_bg"], host["sh_bu"], host["sh_bd"])
                ts = (host["sh_tg"], host["sh_tu"], host["sh_td"])
            else:
                bs = (host["bg"][e], host["bu"][e], host["bd"][e])
                ts = (host["tg"][e], host["tu"][e], host["td"][e])
            out.append({"format": 1, "codes": np.ascontiguousarray(g[:RR]), "block_scale": bs[0][:RR], "tensor_scale": ts[0]})
            out.append({"format": 1, "codes": np.ascontiguousarray(u[:RR]), "block_scale": bs[1][:RR], "tensor_scale": ts[1]})
            out.append({"format": 1, "codes": np.ascontiguousarray(d[:, : RR // 2]),
                        "block_scale": np.ascontiguousarray(bs[2][:, : RR // 16]), "tensor_scale": ts[2]})
        return out

    cache = {}

    def step(i):
        x = xs[i % len(xs)]
        a = time.perf_counter()
        logits = o.router_logits(x, host["Wr"])
        idx, wts, _, _ = o.route(logits, host["bias"], w.k, desc["scaling"])
        b = time.perf_counter()
        xd = x.view(np.float16).astype(np.float64)
        t_ffn = 0.0
        for t in range(x.shape[0]):
            for e in list(idx[t]) + ([None] * w.n_shared):
                key = -1 if e is None else int(e)
                if key not in cache:
                    cache[key] = sliced(None if e is None else int(e))
                m = cache[key]
                c = time.perf_counter()
                o.expert_ffn(m[0], m[1], m[2], xd[t])
                t_ffn += time.perf_counter() - c
        return (b - a) + t_ffn / frac

    for i in range(args.warmup):
        step(i)
    total = 0.0
    wall0 = time.perf_counter()
    for i in range(args.steps):
        total += step(i)
    wall = time.perf_counter() - wall0
    value = args.steps * w.T / total
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = (f"per step: router+top-k of {w.T} token(s) in full; each routed/shared expert on "
              f"{R}/{w.I} intermediate rows, extrapolated x{1 / frac:.1f}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w), "T": w.T},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
# workloads measured beside the headline one in the default run (the rest of the
# metric's configurations: T=8 decode, NVFP4 at T=1 and T=16, the T=512 batch; adaptive
# top-p on decode1; and the int8 and int2 widths at the decode1 shape, T=1 and T=8)
EXTRA_CONFIGS = ("decode8", "nvfp4_1", "nvfp4_16", "prefill512", "batch128", "decode1_topp", "int8_1",
                 "int8_8", "int2_1", "int2_8")
MIN_REGION_S = 0.5     # timed regions are repeated until they add up to at least this


def region_count(first_ms: float, min_s: float) -> int:
    """Timed regions to run so that they add up to ``min_s`` seconds, given the slowest
    rank's first region (at least three)."""
    return max(3, int(np.ceil(min_s * 1000.0 / max(first_ms, 1e-3))))


def timed_regions(run_steps, world, dev, stream, min_s):
    """Times regions of exactly K steps -- barrier and device synchronisation on both
    sides, CUDA events on the launch stream -- until they add up to ``min_s`` (at least
    three regions; every rank runs the same number, decided from the slowest rank's first
    region).  Returns this rank's per-region milliseconds."""
    import torch

    def one():
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e0.record(stream)
            run_steps()
            e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize(dev)
        barrier(world)
        return e0.elapsed_time(e1)

    ms = [one()]
    n = region_count(max_over_ranks(world, ms[0]), min_s)
    for _ in range(n - 1):
        ms.append(one())
    return ms


def bench_config(args, w, world, dev, stream, host=None, want_e2e=True):
    """One workload: R rotating layer copies resident in HBM, K steps per timed region."""
    import torch

    import w4a16_quantized_expert_b200 as moe
    from w4a16_quantized_expert_b200.device import DeviceLayer

    R = args.layers or DEFAULTS.get(w.name, (0, 0, 8))[2]
    K, Wm = args.steps, args.warmup
    desc = {"H": w.H, "I": w.I, "I_sh": w.I_sh, "E": w.E, "k": w.k, "n_shared": w.n_shared,
            "scaling": w.scaling, "fmt": w.fmt, "top_p": w.top_p}
    if host is None:
        host = synth.make_layer(w)
    base = DeviceLayer(desc, host, max_tokens=w.T, device=dev)
    layers = [base] + [base.clone_weights() for _ in range(R - 1)]
    xs_host = [synth.make_tokens(w, batch=b) for b in range(R)]
    xs = [torch.from_numpy(x.copy()).to(dev) for x in xs_host]
    ys = [torch.empty_like(x) for x in xs]
    ws = layers[0].workspace(w.T)

    # unique experts per batch (for the byte accounting), from the library's own grouping
    U, A = [], []
    with torch.cuda.stream(stream):
        for x in xs:
            idx, _, _ = base.route(x, w.T, ws, stream=stream)
            _, _, _, _, nu = base.group(idx, w.T, ws, stream=stream)
            U.append(int(nu.item()))
            A.append(int((idx >= 0).sum().item()))   # fewer than T*k with adaptive top-p
    U_mean, A_mean = float(np.mean(U)), float(np.mean(A))
    ab = algorithmic_bytes(w, U_mean)

    # ---- one CUDA graph of exactly K consecutive layer calls (layer i % R at step i), so
    # that a timed region is one replay and the layers' launch chain runs unbroken
    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                fn(i % R)
        return g

    warm_reps = max(1, (Wm + K - 1) // K)   # warm-up replays: at least Wm steps

    def fwd(i):
        layers[i].forward(xs[i], ws, y=ys[i], stream=stream)

    with torch.cuda.stream(stream):
        for i in range(R):      # eager warm-up of every layer
            fwd(i)
    torch.cuda.synchronize(dev)
    g_full = capture(fwd, K)

    def steps(g):
        def run():
            g.replay()
        return run

    with torch.cuda.stream(stream):      # warm-up steps (graphs replay on the current stream)
        for _ in range(warm_reps):
            g_full.replay()
    torch.cuda.synchronize(dev)
    st = moe.moe_get_device_status(base.handle)
    assert st == moe.MOE_OK, moe.status_string(st)

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.4)
    t_wall0 = time.time()
    region_ms = timed_regions(steps(g_full), world, dev, stream, args.min_region_s)
    t_wall1 = time.time()
    time.sleep(0.3)
    clocks.stop()
    ms_region = max_over_ranks(world, float(np.median(region_ms)))
    ms_step = ms_region / K
    st = moe.moe_get_device_status(base.handle)
    assert st == moe.MOE_OK, moe.status_string(st)

    # ---- per-kernel durations: the same kernels on the same work launched without PDL,
    # event-record nodes between them, captured in a graph (no host gap inside an interval)
    nk = R * max(1, min(K, 512) // R)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(R)]
    with torch.cuda.stream(stream):
        for e4 in evs:
            for e in e4:
                e.record(stream)
    torch.cuda.synchronize(dev)
    info = [0, 0]

    def fwd_timed(i):
        info[:] = moe.moe_forward_timed(layers[i].handle, xs[i].data_ptr(), w.T, ys[i].data_ptr(),
                                        ws.data_ptr(), ws.numel(), stream.cuda_stream,
                                        [e.cuda_event for e in evs[i]])

    gk = capture(fwd_timed, R)
    dur = []
    with torch.cuda.stream(stream):
        for _ in range(nk // R):
            gk.replay()
            torch.cuda.synchronize(dev)
            dur += [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(R)]
    parts, launches = info
    k_ms = np.array(dur).mean(axis=0)
    if parts == 1:      # one kernel does the whole layer
        names, k_ms, kbytes = ["layer"], k_ms[:1], [ab["total"]]
    else:
        names, kbytes = ["router", "gate_up", "down"], [ab["router"], ab["gate_up"], ab["down"]]
    dom = int(np.argmax(k_ms))
    peaks = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    achieved = kbytes[dom] / (k_ms[dom] * 1e-3) / 1e9
    tr = NCU_TRAFFIC.get(w.name)
    traffic = (tr["bytes"] if tr and tr.get("kernel") == names[dom] and tr.get("kernel_hash") == kernel_hash()
               else None)

    # ---- end to end through the public API with host buffers
    e2e = None
    if want_e2e:
        xh = [torch.from_numpy(x.copy()).pin_memory() for x in xs_host]
        yh = [torch.empty_like(x).pin_memory() for x in xh]

        def fwd_host(i):
            layers[i].forward_host(xh[i], yh[i], ws, stream=stream)

        ge = capture(fwd_host, K)
        with torch.cuda.stream(stream):
            for _ in range(warm_reps):
                ge.replay()
        torch.cuda.synchronize(dev)
        e_ms = timed_regions(steps(ge), world, dev, stream, args.min_region_s / 2)
        e2e_ms = max_over_ranks(world, float(np.median(e_ms)))
        e2e = {"value": job_tokens_per_s(world, K, w.T, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 2,
               "timed_regions": len(e_ms),
               "how": "moe_forward_host (pinned host x in, y out), one CUDA graph of K calls per region"}
        st = moe.moe_get_device_status(base.handle)
        assert st == moe.MOE_OK, moe.status_string(st)
        del ge

    # ---- the one-launch decode path on the same layers and tokens (T <= 16)
    fused = None
    if w.T <= 16 and w.fmt in (synth.FMT_INT4, synth.FMT_NVFP4) and not args.no_fused:
        def fwd_fused(i):
            layers[i].forward(xs[i], ws, y=ys[i], stream=stream, fused=True)

        with torch.cuda.stream(stream):
            for i in range(R):
                fwd_fused(i)
        torch.cuda.synchronize(dev)
        gf = capture(fwd_fused, K)
        with torch.cuda.stream(stream):
            for _ in range(warm_reps):
                gf.replay()
        torch.cuda.synchronize(dev)
        f_ms = timed_regions(steps(gf), world, dev, stream, args.min_region_s / 2)
        f_step = max_over_ranks(world, float(np.median(f_ms))) / K
        st = moe.moe_get_device_status(base.handle)
        assert st == moe.MOE_OK, moe.status_string(st)
        fq = ab["weights"] / (f_step * 1e-3) / 1e9
        fused = {"ms_per_layer": f_step, "tokens_per_s": job_tokens_per_s(world, K, w.T, f_step * K),
                 "quantized_weight_gbs": fq, "frac_quantized_of_8tbs": fq / 8000.0,
                 "timed_regions": len(f_ms), "launches_per_step": 1,
                 "how": "moe_forward_fused (router, experts and combine in one persistent launch)"}
        del gf

    tflops = flops(w, A_mean) / (ms_step * 1e-3) / 1e12
    out = {
        "w": w, "host": host, "ms_step": ms_step, "region_ms": region_ms, "R": R, "U": U_mean,
        "ab": ab, "tflops": tflops, "kernels_ms": {n: float(v) for n, v in zip(names, k_ms)},
        "launches_per_step": launches,
        "roofline": {
            "kernel": names[dom], "bound": "hbm", "achieved": achieved, "peak": hbm_peak,
            "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
            "algorithmic_bytes_per_launch": kbytes[dom],
            "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)" if peaks["source"] == "measured" else "fallback",
        },
        "e2e": e2e, "clocks": clocks.summary(t_wall0, t_wall1), "peaks": peaks, "fused": fused,
        "timed_region_s": float(np.sum(region_ms)) / 1000.0,
    }
    del g_full, gk
    for L in layers:
        L.close()
    del layers, xs, ys, ws
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return out


def config_entry(world, r, K) -> dict:
    """A workload's figures for the ``configs`` object of the JSON line."""
    w, ab, ms = r["w"], r["ab"], r["ms_step"]
    hbm_peak = r["roofline"]["peak"]
    qgbs = ab["weights"] / (ms * 1e-3) / 1e9
    e = {
        "workload": describe(w), "T": w.T,
        "ms_per_layer": ms, "tokens_per_s": job_tokens_per_s(world, K, w.T, ms * K),
        "unique_experts_per_step": r["U"],
        "quantized_weight_gbs": qgbs, "frac_quantized_of_8tbs": qgbs / 8000.0,
        "frac_quantized_of_measured": qgbs / hbm_peak,
        "layer_gbs": ab["total"] / (ms * 1e-3) / 1e9,
        "kernels_ms": r["kernels_ms"], "roofline": r["roofline"],
        "tflops": r["tflops"], "timed_regions": len(r["region_ms"]), "steps": K,
        "clocks": r["clocks"],
    }
    if w.T >= 256:     # the batch configuration: tensor throughput against the dense peak
        pk = float(r["peaks"].get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        e["tflops_frac_of_dense_fp16_peak"] = r["tflops"] / pk
        e["dense_peak_tflops"] = pk
    if r["e2e"]:
        e["e2e_tokens_per_s"] = r["e2e"]["value"]
    if r.get("fused"):
        e["fused_path"] = r["fused"]
    return e


def config_steps(name: str, K: int, Wm: int):
    """Steps and warm-up steps of a workload of the ``configs`` object: the headline's K
    and W, capped by the workload's own defaults, so that a line with several workloads
    ends within minutes (the headline workload itself runs exactly K steps)."""
    d = DEFAULTS.get(name)
    if d is None:
        return K, Wm
    return min(K, d[0]), max(3, min(Wm, d[1]))


def run_ours(args, w):
    import copy

    import torch

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.Stream(device=dev)
    K, Wm = args.steps, args.warmup

    head = bench_config(args, w, world, dev, stream)
    extras = {}
    if w.name == "decode1" and not args.no_configs:
        shared_experts = {}
        for name in EXTRA_CONFIGS:
            wx = synth.WORKLOADS[name]
            # workloads that differ only in T, bias or top-p share their experts' weights
            key = (wx.seed, wx.fmt, wx.H, wx.I, wx.I_sh, wx.E, wx.n_shared)
            if key not in shared_experts:
                shared_experts.clear()
                shared_experts[key] = synth.make_experts(wx)
            Wr, b = synth.make_router(wx)
            host = {"Wr": Wr, "bias": b, **shared_experts[key]}
            ax = copy.copy(args)
            ax.steps, ax.warmup = config_steps(name, K, Wm)
            extras[name] = bench_config(ax, wx, world, dev, stream, host=host)
            extras[name]["K"] = ax.steps
    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        xs_host = [synth.make_tokens(w, batch=b) for b in range(4)]
        cpu = oracle_tokens_per_s(w, head["host"], xs_host, seconds=args.cpu_seconds)

    ab, ms_step = head["ab"], head["ms_step"]
    hbm_peak = head["roofline"]["peak"]
    layer_gbs = ab["total"] / (ms_step * 1e-3) / 1e9
    weights_gbs = ab["weights"] / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": job_tokens_per_s(world, K, w.T, ms_step * K),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {
            "workload": describe(w),
            "T": w.T, "H": w.H, "I": w.I, "E": w.E, "top_k": w.k, "top_p": w.top_p, "n_shared": w.n_shared,
            "weights": FMT_NAMES[w.fmt],
            "rotating_layers": head["R"],
            "unique_experts_per_step": head["U"],
            "l2": f"no flush: {head['R']} layer copies at distinct addresses, "
                  f"{ab['total'] / 1e6:.0f} MB of weights per step > 126 MB L2",
            "timing": f"one CUDA graph of {K} consecutive layer calls per timed region, CUDA events "
                      f"on the launch stream; {len(head['region_ms'])} timed regions, median",
            "parallelism": f"replicas x{world}",
        },
        "timed_regions": len(head["region_ms"]),
        "timed_region_s": head["timed_region_s"],
        "hbm": {
            "bytes_per_step": ab["total"],
            "layer_gbs": layer_gbs,
            "quantized_weight_gbs": weights_gbs,
            "peak_gbs": hbm_peak,
            "frac_layer": layer_gbs / hbm_peak,
            "frac_quantized_of_8tbs": weights_gbs / 8000.0,
            "peak_source": head["peaks"]["source"],
        },
        "tflops": head["tflops"],
        "kernels_ms": head["kernels_ms"],
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["launches_per_step"] * K * len(head["region_ms"]),
        "clocks": head["clocks"],
        "cpu_baseline": cpu,
        "fused_path": head["fused"],
        "configs": {name: config_entry(world, r, r["K"]) for name, r in extras.items()},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--layers", type=int, default=None, help="rotating layer copies")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (smaller profiling-size layers; not a bench line)")
    ap.add_argument("--hidden", type=int, default=None, help="override H (profiling only)")
    ap.add_argument("--inter", type=int, default=None, help="override I and I_sh (profiling only)")
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="measure the chosen workload only (no other configurations in the line)")
    ap.add_argument("--no-fused", action="store_true",
                    help="do not also time the one-launch decode path (moe_forward_fused)")
    ap.add_argument("--min-region-s", type=float, default=MIN_REGION_S,
                    help="repeat each timed region of K steps until they add up to this")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    d = DEFAULTS.get(w.name, (1000, 50, 8))
    if args.experts:
        w = w.with_(E=args.experts, k=min(w.k, args.experts), name=f"{w.name}_e{args.experts}")
    if args.hidden or args.inter:
        w = w.with_(H=args.hidden or w.H, I=args.inter or w.I, I_sh=args.inter or w.I_sh,
                    name=f"{w.name}_h{args.hidden or w.H}_i{args.inter or w.I}")
    if args.tokens:
        w = w.with_(T=args.tokens, name=f"{w.name}_t{args.tokens}")
    if args.steps is None:
        args.steps = d[0]
    if args.warmup is None:
        args.warmup = d[1]
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
