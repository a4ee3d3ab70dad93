"""Python binding of the plain FP64 C oracle (``oracle.c``).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product path never does.

``Oracle`` wraps one compiled copy of the library; the tests also build deliberately
broken copies of ``oracle.c`` (planted mistakes) and check that the pins catch them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "oracle.c")
HDR = os.path.join(_HERE, "oracle.h")
SO = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-std=c11"]

INT4, NVFP4, INT8, INT2 = 0, 1, 2, 3
_CODES_PER_BYTE = {INT4: 2, NVFP4: 2, INT8: 1, INT2: 4}


def compile_oracle(src: str = SRC, out: str = SO, include_dir: str = _HERE) -> str:
    subprocess.check_call(["gcc", *CFLAGS, "-I", include_dir, "-o", out, src, "-lm"])
    return out


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < newest:
        compile_oracle()
    return SO


vp = ctypes.c_void_p


class OrcMatrix(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
                ("codes", vp), ("row_scale", vp), ("block_scale", vp),
                ("tensor_scale", ctypes.c_float)]


class OrcLayer(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("I", ctypes.c_int), ("I_sh", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("format", ctypes.c_int), ("scaling", ctypes.c_double),
                ("Wr", vp), ("bias", vp),
                ("g", vp), ("u", vp), ("d", vp),
                ("sg", vp), ("su", vp), ("sd", vp),
                ("bg", vp), ("bu", vp), ("bd", vp),
                ("tg", vp), ("tu", vp), ("td", vp),
                ("sh_g", vp), ("sh_u", vp), ("sh_d", vp),
                ("sh_sg", vp), ("sh_su", vp), ("sh_sd", vp),
                ("sh_bg", vp), ("sh_bu", vp), ("sh_bd", vp),
                ("sh_tg", ctypes.c_float), ("sh_tu", ctypes.c_float), ("sh_td", ctypes.c_float),
                ("top_p", ctypes.c_double)]


class OrcResult(ctypes.Structure):
    _fields_ = [("logits", vp), ("sel", vp), ("gap", vp), ("topk_idx", vp), ("topk_w", vp),
                ("counts", vp), ("offsets", vp), ("perm", vp), ("unique", vp),
                ("n_unique", ctypes.c_int32),
                ("h_assign", vp), ("h_shared", vp), ("y_assign", vp), ("y_shared", vp),
                ("y", vp)]


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need C-contiguous arrays"
    return a.ctypes.data


class Oracle:
    """One loaded copy of the oracle library."""

    def __init__(self, so_path: str | None = None):
        path = so_path or build()
        L = ctypes.CDLL(path)
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_half_to_double.restype = ctypes.c_double
        for f in ("orc_int4_at", "orc_int8_at", "orc_int2_at"):
            getattr(L, f).argtypes = [vp, ctypes.c_long]
            getattr(L, f).restype = ctypes.c_int
        L.orc_quantize_rows.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
        L.orc_quantize_rows.restype = None
        L.orc_e2m1_to_double.argtypes = [ctypes.c_uint]
        L.orc_e2m1_to_double.restype = ctypes.c_double
        L.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_double.restype = ctypes.c_double
        L.orc_sigmoid_f32.argtypes = [ctypes.c_float]
        L.orc_sigmoid_f32.restype = ctypes.c_float
        L.orc_dequant_matrix.argtypes = [ctypes.POINTER(OrcMatrix), vp]
        L.orc_dequant_matrix.restype = None
        L.orc_router_logits.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, vp]
        L.orc_route.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                vp, vp, vp, vp]
        L.orc_route_p.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                  ctypes.c_double, vp, vp, vp, vp]
        L.orc_group.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp]
        L.orc_expert_ffn.argtypes = [ctypes.POINTER(OrcMatrix)] * 3 + [vp, vp, vp]
        L.orc_routed_expert.argtypes = [ctypes.POINTER(OrcLayer), ctypes.c_int, vp, vp, vp]
        L.orc_shared_expert.argtypes = [ctypes.POINTER(OrcLayer), vp, vp, vp]
        for f in ("orc_forward", "orc_forward_per_token"):
            getattr(L, f).argtypes = [ctypes.POINTER(OrcLayer), vp, ctypes.c_int, vp,
                                      ctypes.POINTER(OrcResult)]
        L.orc_forward_token.argtypes = [ctypes.POINTER(OrcLayer), vp, vp, vp, vp, vp, vp]
        for f in ("orc_router_logits", "orc_route", "orc_route_p", "orc_group", "orc_expert_ffn",
                  "orc_routed_expert", "orc_shared_expert", "orc_forward",
                  "orc_forward_per_token", "orc_forward_token"):
            getattr(L, f).restype = None
        self.lib = L

    # ------------------------------------------------------------ scalar decodes
    def half_to_double(self, bits: int) -> float:
        return self.lib.orc_half_to_double(bits)

    def int4_row(self, row_bytes: np.ndarray, K: int) -> np.ndarray:
        row = np.ascontiguousarray(row_bytes, dtype=np.uint8)
        return np.array([self.lib.orc_int4_at(_p(row), k) for k in range(K)], dtype=np.int64)

    def int8_row(self, row_bytes: np.ndarray, K: int) -> np.ndarray:
        row = np.ascontiguousarray(row_bytes, dtype=np.uint8)
        return np.array([self.lib.orc_int8_at(_p(row), k) for k in range(K)], dtype=np.int64)

    def int2_row(self, row_bytes: np.ndarray, K: int) -> np.ndarray:
        row = np.ascontiguousarray(row_bytes, dtype=np.uint8)
        return np.array([self.lib.orc_int2_at(_p(row), k) for k in range(K)], dtype=np.int64)

    def quantize(self, w: np.ndarray, bits: int):
        """Per-row symmetric quantisation of fp32 rows [N][K] to bits = 8, 4 or 2.
        Returns (codes [N][K * bits / 8] uint8, row scales [N] fp32)."""
        w = np.ascontiguousarray(w, np.float32)
        N, K = w.shape
        codes = np.empty((N, K * bits // 8), np.uint8)
        scale = np.empty(N, np.float32)
        self.lib.orc_quantize_rows(_p(w), N, K, bits, _p(codes), _p(scale))
        return codes, scale

    def e2m1(self, code: int) -> float:
        return self.lib.orc_e2m1_to_double(code)

    def e4m3(self, byte: int) -> float:
        return self.lib.orc_e4m3_to_double(byte)

    def dequant(self, M: dict) -> np.ndarray:
        m, keep = self._matrix(M)
        out = np.empty((m.N, m.K), np.float64)
        self.lib.orc_dequant_matrix(ctypes.byref(m), _p(out))
        return out

    def sigmoid_f32(self, logit: float) -> np.float32:
        return np.float32(self.lib.orc_sigmoid_f32(logit))

    # ------------------------------------------------------------------ stages
    def router_logits(self, x: np.ndarray, Wr: np.ndarray) -> np.ndarray:
        T, H = x.shape
        E = Wr.shape[0]
        x = np.ascontiguousarray(x, np.uint16)
        Wr = np.ascontiguousarray(Wr, np.float32)
        out = np.empty((T, E), np.float32)
        self.lib.orc_router_logits(_p(x), T, H, _p(Wr), E, _p(out))
        return out

    def route(self, logits: np.ndarray, bias: np.ndarray, k: int, scaling: float, top_p: float = 0.0):
        """Top-k routing (and adaptive top-p when 0 < top_p < 1: dropped entries are
        index -1, weight 0).  Returns idx, w, sel, gap."""
        T, E = logits.shape
        logits = np.ascontiguousarray(logits, np.float32)
        bias = np.ascontiguousarray(bias, np.float32)
        idx = np.empty((T, k), np.int32)
        w = np.empty((T, k), np.float32)
        sel = np.empty((T, E), np.float32)
        gap = np.empty(T, np.float32)
        if top_p:
            self.lib.orc_route_p(_p(logits), _p(bias), T, E, k, scaling, float(top_p), _p(idx), _p(w),
                                 _p(sel), _p(gap))
        else:
            self.lib.orc_route(_p(logits), _p(bias), T, E, k, scaling, _p(idx), _p(w), _p(sel), _p(gap))
        return idx, w, sel, gap

    def group(self, topk_idx: np.ndarray, E: int):
        T, k = topk_idx.shape
        idx = np.ascontiguousarray(topk_idx, np.int32)
        counts = np.empty(E, np.int32)
        offsets = np.empty(E + 1, np.int32)
        perm = np.empty(T * k, np.int32)
        unique = np.empty(E, np.int32)
        nu = ctypes.c_int32(0)
        self.lib.orc_group(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(unique),
                           ctypes.byref(nu))
        # perm holds the offsets[E] grouped assignments (entries dropped by top-p are not)
        return counts, offsets, perm[: offsets[E]].copy(), unique[: nu.value].copy()

    def expert_ffn(self, Wg: dict, Wu: dict, Wd: dict, x: np.ndarray):
        """One expert on one fp64 activation vector.  Each matrix is a dict with
        'format', 'codes' [N][K/2] and 'row_scale' or 'block_scale'/'tensor_scale'."""
        mats = [self._matrix(M) for M in (Wg, Wu, Wd)]
        x = np.ascontiguousarray(x, np.float64)
        I = mats[0][0].N
        h = np.empty(I, np.float64)
        y = np.empty(mats[2][0].N, np.float64)
        self.lib.orc_expert_ffn(ctypes.byref(mats[0][0]), ctypes.byref(mats[1][0]),
                                ctypes.byref(mats[2][0]), _p(x), _p(h), _p(y))
        return h, y

    @staticmethod
    def _matrix(M: dict):
        keep = []
        codes = np.ascontiguousarray(M["codes"], np.uint8)
        keep.append(codes)
        N, Kb = codes.shape
        m = OrcMatrix(format=M["format"], N=N, K=_CODES_PER_BYTE[M["format"]] * Kb, codes=_p(codes))
        if M["format"] != NVFP4:
            rs = np.ascontiguousarray(M["row_scale"], np.float32)
            keep.append(rs)
            m.row_scale = _p(rs)
        else:
            bs = np.ascontiguousarray(M["block_scale"], np.uint8)
            keep.append(bs)
            m.block_scale = _p(bs)
            m.tensor_scale = float(M["tensor_scale"])
        return m, keep

    # ------------------------------------------------------------ whole layer
    def make_layer(self, desc: dict, layer: dict):
        """Build the C layer struct from numpy arrays.  ``desc`` holds H, I, I_sh, E,
        k, n_shared, scaling, fmt.  Returns (struct, keep-alive list)."""
        keep = []

        def P(name):
            a = layer.get(name)
            if a is None:
                return None
            a = np.ascontiguousarray(a)
            keep.append(a)
            return _p(a)

        L = OrcLayer(H=desc["H"], I=desc["I"], I_sh=desc["I_sh"], E=desc["E"], k=desc["k"],
                     n_shared=desc["n_shared"], format=desc["fmt"], scaling=desc["scaling"],
                     top_p=float(desc.get("top_p", 0.0)))
        for f in ("Wr", "bias", "g", "u", "d", "sg", "su", "sd", "bg", "bu", "bd", "tg", "tu",
                  "td", "sh_g", "sh_u", "sh_d", "sh_sg", "sh_su", "sh_sd", "sh_bg", "sh_bu",
                  "sh_bd"):
            setattr(L, f, P(f))
        for f in ("sh_tg", "sh_tu", "sh_td"):
            if f in layer:
                setattr(L, f, float(layer[f]))
        return L, keep

    def forward(self, desc: dict, layer: dict, x: np.ndarray, logits_in=None,
                per_token: bool = False, want_h: bool = False) -> dict:
        L, keep = self.make_layer(desc, layer)
        T = x.shape[0]
        H, E, k, I, Ish = desc["H"], desc["E"], desc["k"], desc["I"], desc["I_sh"]
        x = np.ascontiguousarray(x, np.uint16)
        out = {
            "logits": np.empty((T, E), np.float32), "sel": np.empty((T, E), np.float32),
            "gap": np.empty(T, np.float32), "topk_idx": np.empty((T, k), np.int32),
            "topk_w": np.empty((T, k), np.float32), "counts": np.empty(E, np.int32),
            "offsets": np.empty(E + 1, np.int32), "perm": np.empty(T * k, np.int32),
            "unique": np.empty(E, np.int32),
            "y_assign": np.zeros((T * k, H), np.float64),
            "y_shared": np.zeros((T, H), np.float64), "y": np.empty((T, H), np.float64),
        }
        if want_h:
            out["h_assign"] = np.zeros((T * k, I), np.float64)
            out["h_shared"] = np.zeros((T, Ish), np.float64)
        R = OrcResult()
        for key, arr in out.items():
            setattr(R, key, _p(arr))
        li = None
        if logits_in is not None:
            li = np.ascontiguousarray(logits_in, np.float32)
        fn = self.lib.orc_forward_per_token if per_token else self.lib.orc_forward
        fn(ctypes.byref(L), _p(x), T, _p(li), ctypes.byref(R))
        out["unique"] = out["unique"][: R.n_unique].copy()
        return out

    def forward_token(self, desc: dict, layer: dict, x_t: np.ndarray, logits_t=None):
        L, keep = self.make_layer(desc, layer)
        k, H = desc["k"], desc["H"]
        x_t = np.ascontiguousarray(x_t.reshape(-1), np.uint16)
        idx = np.empty(k, np.int32)
        w = np.empty(k, np.float32)
        gap = np.empty(1, np.float32)
        y = np.empty(H, np.float64)
        li = None if logits_t is None else np.ascontiguousarray(logits_t, np.float32)
        self.lib.orc_forward_token(ctypes.byref(L), _p(x_t), _p(li), _p(idx), _p(w), _p(gap),
                                   _p(y))
        return {"topk_idx": idx, "topk_w": w, "gap": float(gap[0]), "y": y}


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def desc_of(w) -> dict:
    """Layer description dict from a ``synth.Workload``."""
    return {"H": w.H, "I": w.I, "I_sh": w.I_sh, "E": w.E, "k": w.k, "n_shared": w.n_shared,
            "scaling": w.scaling, "fmt": w.fmt, "top_p": float(getattr(w, "top_p", 0.0))}
