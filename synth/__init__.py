"""Seeded synthetic workloads for the W4A16 quantized-expert MoE layer.

This package draws every input the layer consumes (activations, router weights and
bias, quantised expert weights and their scales) from a counter-based generator
written in C (``synth.c``).  It holds no part of the layer's arithmetic and is the
only code that the CPU oracle's tests and the CUDA path's tests share.

Workloads (sizes and distributions as the layer is described for GLM-class decode):

* ``tiny``   -- T=4, H=256, I=128, E=16, k=2, one shared expert, int4.
* ``decode1`` -- T=1, H=6144, I=2048, E=256, k=8, one shared expert, int4
  (about 19 MB of int4 per expert).
* ``decode8`` -- as ``decode1`` with T=8 and a Zipf(1.1) selection bias in [-0.5, 0.5].
* ``nvfp4_1`` / ``nvfp4_16`` -- H=2048, I=512, E=256, k=8, one shared expert, NVFP4,
  T=1 and T=16.
* ``prefill512`` -- T=512, otherwise as ``decode1``.
* ``int8_1`` / ``int8_8`` / ``int2_1`` / ``int2_8`` -- the decode1 shape with int8 or int2
  codes (one fp32 scale per row), T=1 and T=8.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "synth.c")

FMT_INT4 = 0
FMT_NVFP4 = 1
FMT_INT8 = 2
FMT_INT2 = 3
# bits per code of the row-scaled formats, and the factor on their U(0.01, 0.03) row scales
# that gives every format about the same weight spread (uniform codes: std 73.9, 4.6 and
# 1.1 for int8, int4, int2; powers of two keep the scales' fp32 values exact)
ROWSCALED_BITS = {FMT_INT4: 4, FMT_INT8: 8, FMT_INT2: 2}
_SCALE_FACTOR = {FMT_INT4: 1.0, FMT_INT8: 1.0 / 16.0, FMT_INT2: 4.0}


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-o", _SO, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, sz, dbl = ctypes.c_uint64, ctypes.c_size_t, ctypes.c_double
        vp = ctypes.c_void_p
        L.synth_normal_f16.argtypes = [u64, u64, dbl, vp, sz]
        L.synth_normal_f32.argtypes = [u64, u64, dbl, vp, sz]
        L.synth_uniform_f32.argtypes = [u64, u64, dbl, dbl, vp, sz]
        L.synth_bytes.argtypes = [u64, u64, vp, sz]
        L.synth_zipf_bias.argtypes = [u64, u64, ctypes.c_int, dbl, dbl, dbl, vp]
        L.synth_nvfp4.argtypes = [u64, u64, ctypes.c_int, ctypes.c_int, vp, vp]
        L.synth_half_from_double.argtypes = [dbl]
        L.synth_half_from_double.restype = ctypes.c_uint16
        L.synth_e4m3_from_double.argtypes = [dbl, ctypes.POINTER(ctypes.c_double)]
        L.synth_e4m3_from_double.restype = ctypes.c_uint8
        L.synth_e2m1_from_double.argtypes = [dbl]
        L.synth_e2m1_from_double.restype = ctypes.c_uint8
        for f in ("synth_normal_f16", "synth_normal_f32", "synth_uniform_f32",
                  "synth_bytes", "synth_zipf_bias", "synth_nvfp4"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ----------------------------------------------------------------- stream ids
# stream = tensor id << 20 | expert index (shared expert uses its own tensor ids)
T_X, T_WR, T_BIAS = 1, 2, 3
T_G, T_U, T_D, T_SG, T_SU, T_SD = 4, 5, 6, 7, 8, 9
T_SHG, T_SHU, T_SHD, T_SHSG, T_SHSU, T_SHSD = 10, 11, 12, 13, 14, 15
T_XS = 16   # choices of the edge-case activation rows


def _sid(tensor: int, expert: int = 0) -> int:
    return (tensor << 20) | expert


# ----------------------------------------------------------------- primitives
def normal_f16(seed, stream, n, std=1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    lib().synth_normal_f16(seed, stream, std, _p(out), n)
    return out


def normal_f32(seed, stream, n, std=1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal_f32(seed, stream, std, _p(out), n)
    return out


def uniform_f32(seed, stream, n, lo, hi) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_uniform_f32(seed, stream, lo, hi, _p(out), n)
    return out


def random_bytes(seed, stream, n) -> np.ndarray:
    out = np.empty(n, dtype=np.uint8)
    lib().synth_bytes(seed, stream, _p(out), n)
    return out


def zipf_bias(seed, stream, E, s, lo, hi) -> np.ndarray:
    out = np.empty(E, dtype=np.float32)
    lib().synth_zipf_bias(seed, stream, E, s, lo, hi, _p(out))
    return out


def nvfp4_block(seed, stream, rows, K):
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    bs = np.empty((rows, K // 16), dtype=np.uint8)
    lib().synth_nvfp4(seed, stream, rows, K, _p(codes), _p(bs))
    return codes, bs


# ----------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    I_sh: int
    E: int
    k: int
    n_shared: int
    scaling: float
    fmt: int
    bias: str            # "uniform" (U(-0.1, 0.1)) or "zipf" (Zipf(1.1) ranking into [-0.5, 0.5])
    seed: int
    top_p: float = 0.0   # adaptive expert top-p (0: plain top-k)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


BASE_SEED = 20260925

WORKLOADS = {
    "tiny": Workload("tiny", 4, 256, 128, 128, 16, 2, 1, 2.5, FMT_INT4, "uniform", BASE_SEED + 0),
    "decode1": Workload("decode1", 1, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT4, "uniform",
                        BASE_SEED + 1),
    "decode8": Workload("decode8", 8, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT4, "zipf",
                        BASE_SEED + 2),
    "nvfp4_1": Workload("nvfp4_1", 1, 2048, 512, 512, 256, 8, 1, 2.5, FMT_NVFP4, "uniform",
                        BASE_SEED + 3),
    "nvfp4_16": Workload("nvfp4_16", 16, 2048, 512, 512, 256, 8, 1, 2.5, FMT_NVFP4, "uniform",
                         BASE_SEED + 3),
    "prefill512": Workload("prefill512", 512, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT4,
                           "uniform", BASE_SEED + 4),
    # decode1 with adaptive expert top-p 0.7 (the value of the --topp example on the hakusoku
    # page, section "実行・チューニングパラメータ"); same weights and tokens as decode1
    "decode1_topp": Workload("decode1_topp", 1, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT4,
                             "uniform", BASE_SEED + 1, top_p=0.7),
    # larger batch (about 64 tokens per expert): the tensor-memory kernel's compute-heavier regime
    "prefill2048": Workload("prefill2048", 2048, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT4,
                            "uniform", BASE_SEED + 5),
    # a mid-size batch of about 4 tokens per routed expert (128 x 8 / 256): the regime
    # between the decode batches and prefill512, on the prefill512 layer shape
    "batch128": Workload("batch128", 128, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT4, "uniform",
                         BASE_SEED + 8),
    # the other row-scaled widths (int8 and int2 kernels with per-row scales: hakusoku page,
    # section "実装済み機能") at the decode1 shape, one token and eight
    "int8_1": Workload("int8_1", 1, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT8, "uniform",
                       BASE_SEED + 6),
    "int8_8": Workload("int8_8", 8, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT8, "zipf",
                       BASE_SEED + 6),
    "int2_1": Workload("int2_1", 1, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT2, "uniform",
                       BASE_SEED + 7),
    "int2_8": Workload("int2_8", 8, 6144, 2048, 2048, 256, 8, 1, 2.5, FMT_INT2, "zipf",
                       BASE_SEED + 7),
}


def make_tokens(w: Workload, T: int | None = None, batch: int = 0) -> np.ndarray:
    """fp16 activations x ~ N(0,1), returned as uint16 bit patterns [T, H].
    ``batch`` selects an independent set of tokens from the same seed."""
    T = w.T if T is None else T
    x = normal_f16(w.seed, _sid(T_X, batch), T * w.H)
    return x.reshape(T, w.H)


def make_router(w: Workload):
    Wr = normal_f32(w.seed, _sid(T_WR), w.E * w.H, std=1.0 / np.sqrt(w.H)).reshape(w.E, w.H)
    if w.bias == "zipf":
        b = zipf_bias(w.seed, _sid(T_BIAS), w.E, 1.1, -0.5, 0.5)
    else:
        b = uniform_f32(w.seed, _sid(T_BIAS), w.E, -0.1, 0.1)
    return Wr, b


def _rowscaled_matrix(seed, tid, sid_scale, e, rows, K, fmt, out_q, out_s):
    """Uniform random code bytes (every code value equally likely) and row scales."""
    nb = K * ROWSCALED_BITS[fmt] // 8
    out_q[...] = random_bytes(seed, _sid(tid, e), rows * nb).reshape(rows, nb)
    s = uniform_f32(seed, _sid(sid_scale, e), rows, 0.01, 0.03)
    out_s[...] = (s * np.float32(_SCALE_FACTOR[fmt])).astype(np.float32)


def _nvfp4_matrix(seed, tid, e, rows, K, out_q, out_b):
    q, b = nvfp4_block(seed, _sid(tid, e), rows, K)
    out_q[...] = q
    out_b[...] = b


def make_experts(w: Workload, experts=None) -> dict:
    """Quantised weights of the routed experts (all E, laid out [E][rows][K*bits/8];
    only the listed ``experts`` are filled, the rest stay zero) and of the shared
    expert.  int8 / int4 / int2: codes + fp32 row scales.  NVFP4: codes + E4M3 block scales
    (one per 16 K-elements) + one fp32 tensor scale per (expert, matrix) equal to
    1/sqrt(fan-in)."""
    E, H, I, Ish = w.E, w.H, w.I, w.I_sh
    ex = range(E) if experts is None else sorted(set(int(e) for e in experts))
    zeros = np.zeros if experts is not None else np.empty
    bits = ROWSCALED_BITS.get(w.fmt, 4)
    out = {
        "g": zeros((E, I, H * bits // 8), np.uint8),
        "u": zeros((E, I, H * bits // 8), np.uint8),
        "d": zeros((E, H, I * bits // 8), np.uint8),
    }
    shared = w.n_shared > 0
    if shared:
        out["sh_g"] = np.empty((Ish, H * bits // 8), np.uint8)
        out["sh_u"] = np.empty((Ish, H * bits // 8), np.uint8)
        out["sh_d"] = np.empty((H, Ish * bits // 8), np.uint8)
    if w.fmt in ROWSCALED_BITS:
        f = w.fmt
        out["sg"] = zeros((E, I), np.float32)
        out["su"] = zeros((E, I), np.float32)
        out["sd"] = zeros((E, H), np.float32)
        for e in ex:
            _rowscaled_matrix(w.seed, T_G, T_SG, e, I, H, f, out["g"][e], out["sg"][e])
            _rowscaled_matrix(w.seed, T_U, T_SU, e, I, H, f, out["u"][e], out["su"][e])
            _rowscaled_matrix(w.seed, T_D, T_SD, e, H, I, f, out["d"][e], out["sd"][e])
        if shared:
            out["sh_sg"] = np.empty(Ish, np.float32)
            out["sh_su"] = np.empty(Ish, np.float32)
            out["sh_sd"] = np.empty(H, np.float32)
            _rowscaled_matrix(w.seed, T_SHG, T_SHSG, 0, Ish, H, f, out["sh_g"], out["sh_sg"])
            _rowscaled_matrix(w.seed, T_SHU, T_SHSU, 0, Ish, H, f, out["sh_u"], out["sh_su"])
            _rowscaled_matrix(w.seed, T_SHD, T_SHSD, 0, H, Ish, f, out["sh_d"], out["sh_sd"])
    else:
        out["bg"] = zeros((E, I, H // 16), np.uint8)
        out["bu"] = zeros((E, I, H // 16), np.uint8)
        out["bd"] = zeros((E, H, I // 16), np.uint8)
        out["tg"] = np.full(E, 1.0 / np.sqrt(H), np.float32)
        out["tu"] = np.full(E, 1.0 / np.sqrt(H), np.float32)
        out["td"] = np.full(E, 1.0 / np.sqrt(I), np.float32)
        for e in ex:
            _nvfp4_matrix(w.seed, T_G, e, I, H, out["g"][e], out["bg"][e])
            _nvfp4_matrix(w.seed, T_U, e, I, H, out["u"][e], out["bu"][e])
            _nvfp4_matrix(w.seed, T_D, e, H, I, out["d"][e], out["bd"][e])
        if shared:
            out["sh_bg"] = np.empty((Ish, H // 16), np.uint8)
            out["sh_bu"] = np.empty((Ish, H // 16), np.uint8)
            out["sh_bd"] = np.empty((H, Ish // 16), np.uint8)
            out["sh_tg"] = np.float32(1.0 / np.sqrt(H))
            out["sh_tu"] = np.float32(1.0 / np.sqrt(H))
            out["sh_td"] = np.float32(1.0 / np.sqrt(Ish))
            _nvfp4_matrix(w.seed, T_SHG, 0, Ish, H, out["sh_g"], out["sh_bg"])
            _nvfp4_matrix(w.seed, T_SHU, 0, Ish, H, out["sh_u"], out["sh_bu"])
            _nvfp4_matrix(w.seed, T_SHD, 0, H, Ish, out["sh_d"], out["sh_bd"])
    return out


def make_layer(w: Workload, experts=None) -> dict:
    Wr, b = make_router(w)
    layer = {"Wr": Wr, "bias": b}
    layer.update(make_experts(w, experts))
    return layer


# ----------------------------------------------------------------- edge-case activations
STRESS_KINDS = ("outlier", "near_max", "subnormal", "mixed")


def make_stress_tokens(w: Workload, T: int, kind: str, batch: int = 0) -> np.ndarray:
    """fp16 activation rows [T, H] (uint16 bit patterns) at the edges of the fp16 range,
    for checking that an implementation's activation representation keeps them:

    * ``outlier``: N(0,1) rows in which one or two channels hold +-2^12 .. 2^15 (times
      a mantissa in [1, 2)), so the rest of the row lies 12 to 16 binary orders below its
      largest value;
    * ``near_max``: N(0,1) rows with two channels at +-65504 (the largest finite fp16)
      and one at +-65472 (the next one down);
    * ``subnormal``: every value an fp16 subnormal (|x| = m * 2^-24, m in 1..1023);
    * ``mixed``: N(0,1) rows in which about a quarter of the channels are subnormals.

    Choices (channels, signs, exponents, mantissas) come from the counter-based stream
    keyed by (seed, T_XS, batch); the N(0,1) parts are ``make_tokens``'s rows."""
    if kind not in STRESS_KINDS:
        raise ValueError(kind)
    x = make_tokens(w, T, batch=batch).copy()
    H = w.H
    r = random_bytes(w.seed, _sid(T_XS, batch * 8 + STRESS_KINDS.index(kind)), T * H * 4)
    r = r.view(np.uint32).reshape(T, H)
    sign = (r & 1).astype(np.uint16) << 15
    if kind == "subnormal":
        m = (((r >> 1) % 1023) + 1).astype(np.uint16)
        return (sign | m).reshape(T, H)
    if kind == "mixed":
        m = (((r >> 1) % 1023) + 1).astype(np.uint16)
        pick = ((r >> 11) & 3) == 0
        x[pick] = (sign | m)[pick]
        return x
    for t in range(T):
        c = [int(v % H) for v in r[t, :3] >> 12]
        if kind == "outlier":
            n = 1 + int(r[t, 3] & 1)
            for j in range(n):
                ex = 12 + int((r[t, 4 + j] >> 4) % 4)                 # 12 .. 15
                mant = 1.0 + ((int(r[t, 6 + j]) >> 8) % 1024) / 1024.0   # exact in fp16
                v = np.float16(mant * 2.0 ** ex)
                x[t, c[j]] = np.array([v], np.float16).view(np.uint16)[0] | int(sign[t, j])
        else:   # near_max
            for j, v in enumerate((65504.0, 65504.0, 65472.0)):
                x[t, c[j]] = np.array([np.float16(v)], np.float16).view(np.uint16)[0] | int(sign[t, j])
    return x


def scale_layer(layer: dict, fmt: int, gate_up: float, down: float, router: float = 1.0) -> dict:
    """The same layer with every gate/up weight multiplied by ``gate_up``, every down
    weight by ``down`` and the router weights by ``router`` (powers of two keep the fp32
    values exact), by scaling the int4 row scales or the NVFP4 per-matrix scales.  Used to
    keep h and y of edge-case activation rows inside the fp16 range, and the router
    logits of subnormal rows away from a tie decided by the bias alone."""
    out = dict(layer)
    if "Wr" in out:
        out["Wr"] = (np.asarray(out["Wr"], np.float32) * np.float32(router)).astype(np.float32)
    if fmt != FMT_NVFP4:
        keys_gu, keys_d = ("sg", "su", "sh_sg", "sh_su"), ("sd", "sh_sd")
    else:
        keys_gu, keys_d = ("tg", "tu", "sh_tg", "sh_tu"), ("td", "sh_td")
    for k in keys_gu:
        if k in out:
            out[k] = (np.asarray(out[k], np.float32) * np.float32(gate_up)).astype(np.float32)
    for k in keys_d:
        if k in out:
            out[k] = (np.asarray(out[k], np.float32) * np.float32(down)).astype(np.float32)
    return out
