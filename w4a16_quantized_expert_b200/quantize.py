"""Offline weight conversion to the library's row-scaled integer layouts.

The source pages describe an offline tool that converts a model's FP8 weights to int4
with one scale per output row ("Show HN: 低速のコンピュータでGLM 5.2を動かす方法", section
"実装済み機能"), and int8/int4/int2 kernels with per-row scales.  This module is that
preparation step for this library (host side, run once per checkpoint, never on the
layer's hot path):

* symmetric per-row quantisation: scale = max|w| / (2^(bits-1) - 1), rounded to fp32;
  code = round-half-to-even(w / scale) with that fp32 scale, clamped to the code range;
  an all-zero row gets scale 0 and zero codes;
* packing along K as the kernels read it: int8 one byte per weight, int4 two codes per
  byte (element 2b in the low nibble), int2 four codes per byte (element 4b+i in bits
  2i..2i+1), all two's complement;
* FP8 (E4M3, OCP "FN") input, decoded exactly, optionally with one fp32 scale per block.
"""
from __future__ import annotations

import numpy as np

BITS = (8, 4, 2)


def quantize_rows(w: np.ndarray, bits: int = 4) -> tuple[np.ndarray, np.ndarray]:
    """Quantise rows of ``w`` [N][K] (any float dtype) to ``bits``-bit codes.

    Returns (codes uint8 [N][K * bits / 8], scales float32 [N])."""
    if bits not in BITS:
        raise ValueError(f"bits must be one of {BITS}")
    w = np.asarray(w)
    if w.ndim != 2 or (w.shape[1] * bits) % 8:
        raise ValueError("w must be [N][K] with K * bits a multiple of 8")
    wf = np.asarray(w, dtype=np.float32).astype(np.float64)
    qmax = (1 << (bits - 1)) - 1
    qmin = -(1 << (bits - 1))
    amax = np.abs(wf).max(axis=1)
    scale = (amax / qmax).astype(np.float32)
    s64 = scale.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s64 > 0, np.rint(wf / np.where(s64 > 0, s64, 1.0)), 0.0)
    q = np.clip(q, qmin, qmax).astype(np.int64)
    return pack(q, bits), scale


def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """Two's-complement codes [N][K] -> packed bytes [N][K * bits / 8]."""
    u = (np.asarray(q, dtype=np.int64) & ((1 << bits) - 1)).astype(np.uint8)
    per = 8 // bits
    N, K = u.shape
    u = u.reshape(N, K // per, per)
    out = np.zeros((N, K // per), np.uint8)
    for i in range(per):
        out |= (u[:, :, i] << (bits * i)).astype(np.uint8)
    return out


def unpack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Packed bytes [N][B] -> two's-complement codes [N][B * 8 / bits]."""
    c = np.asarray(codes, dtype=np.uint8)
    per = 8 // bits
    mask = (1 << bits) - 1
    q = np.stack([(c >> (bits * i)) & mask for i in range(per)], axis=-1).astype(np.int64)
    q = q.reshape(c.shape[0], -1)
    return np.where(q >= (1 << (bits - 1)), q - (1 << bits), q)


def e4m3_to_float32(b: np.ndarray) -> np.ndarray:
    """Exact decode of FP8 E4M3 ("FN": bias 7, subnormals, 0x7F / 0xFF = NaN) bytes."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 15
    m = b & 7
    v = np.where(e == 0, np.ldexp(m.astype(np.float64), -9), np.ldexp(1.0 + m / 8.0, e - 7))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return np.where(s == 1, -v, v).astype(np.float32)


def quantize_fp8_rows(fp8: np.ndarray, bits: int = 4, block_scale: np.ndarray | None = None,
                      block: int = 128) -> tuple[np.ndarray, np.ndarray]:
    """Re-quantise FP8 E4M3 weights [N][K] (bytes) to ``bits``-bit row-scaled codes.

    ``block_scale`` (optional, fp32 [N / block][K / block]) multiplies each block x block
    tile of the decoded values, the usual layout of FP8 checkpoints' scales."""
    w = e4m3_to_float32(fp8).astype(np.float64)
    if np.isnan(w).any():
        raise ValueError("FP8 input holds NaN codes")
    if block_scale is not None:
        bs = np.asarray(block_scale, dtype=np.float32).astype(np.float64)
        rep = np.repeat(np.repeat(bs, block, axis=0), block, axis=1)[: w.shape[0], : w.shape[1]]
        w = w * rep
    return quantize_rows(w.astype(np.float32), bits)
