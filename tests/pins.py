"""Pins of the CPU oracle to facts outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises ``AssertionError`` when the
oracle disagrees with something the pages, a published format definition, the
mathematics or an independent library fixes:

* hand-derived decodes (``tests/golden``), exhaustive comparison with numpy's fp16 and
  torch's FP8 E4M3 conversions;
* closed forms of the sigmoid and of router logits on one-hot activations;
* brute force over all expert subsets for top-k, and over all assignments for grouping;
* invariants: combine weights sum to the routed scaling factor, the bias only selects,
  batch-union results equal per-token results bit for bit, relabelling experts changes
  nothing;
* special cases that reduce to a textbook routine: with one expert, top-1 and no shared
  expert, the layer is a dense SwiGLU FFN (numpy matmuls on the dequantised weights).

``tests/test_oracle_pins.py`` runs them on the real oracle; ``tests/test_oracle_mutants.py``
runs them on copies of ``oracle.c`` with planted mistakes and checks that each mistake
fails at least one pin.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers
def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


def f16_bits(values) -> np.ndarray:
    return np.asarray(values, dtype=np.float16).view(np.uint16)


def np_dequant_int4(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """numpy unpacking of the packed int4 format (low nibble first, two's complement)."""
    lo = (codes & 0x0F).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    q = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    q = np.where(q >= 8, q - 16, q)
    return q.astype(np.float64) * scale.astype(np.float64)[:, None]


def np_dequant_int8(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """numpy reading of int8 codes (one two's-complement byte per weight)."""
    return codes.view(np.int8).astype(np.float64) * scale.astype(np.float64)[:, None]


def np_dequant_int2(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """numpy unpacking of int2 codes (four per byte, element 4b+i in bits 2i..2i+1)."""
    q = np.stack([(codes >> (2 * i)) & 3 for i in range(4)], axis=-1).astype(np.int64)
    q = q.reshape(codes.shape[0], -1)
    q = np.where(q >= 2, q - 4, q)
    return q.astype(np.float64) * scale.astype(np.float64)[:, None]


NP_DEQUANT_ROWSCALED = {0: np_dequant_int4, 2: np_dequant_int8, 3: np_dequant_int2}
BYTES_PER_CODE = {0: 0.5, 1: 0.5, 2: 1.0, 3: 0.25}


def _e2m1_table():
    return np.array([float(r.split()[1]) for r in _rows("e2m1_ocp.txt")], np.float64)


def np_dequant_nvfp4(codes, bscale, tscale):
    import torch
    lo = (codes & 0x0F).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    c = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)
    vals = _e2m1_table()[c]
    sb = torch.from_numpy(np.ascontiguousarray(bscale)).view(torch.float8_e4m3fn).double().numpy()
    return vals * np.repeat(sb, 16, axis=1) * float(tscale)


def silu(v):
    return v / (1.0 + np.exp(-v))


def small_layer(E=1, k=1, n_shared=0, H=64, I=32, I_sh=32, fmt=0, scaling=1.0, seed=1):
    """A small random layer built with numpy (independent of the synth package)."""
    rng = np.random.default_rng(seed)
    L = {"Wr": (rng.standard_normal((E, H)) / math.sqrt(H)).astype(np.float32),
         "bias": rng.uniform(-0.1, 0.1, E).astype(np.float32)}
    def mat(rows, K):
        codes = rng.integers(0, 256, (rows, int(K * BYTES_PER_CODE[fmt])), dtype=np.uint8)
        if fmt != 1:   # row-scaled integer codes
            return codes, rng.uniform(0.01, 0.03, rows).astype(np.float32) * (0.0625 if fmt == 2 else 1.0)
        # E4M3 block scales from a small range of normal values (exponent 5..8, any mantissa)
        bs = (rng.integers(5, 9, (rows, K // 16)) << 3 | rng.integers(0, 8, (rows, K // 16)))
        return codes, bs.astype(np.uint8)
    g = [mat(I, H) for _ in range(E)]
    u = [mat(I, H) for _ in range(E)]
    d = [mat(H, I) for _ in range(E)]
    L["g"] = np.stack([m[0] for m in g]); L["u"] = np.stack([m[0] for m in u])
    L["d"] = np.stack([m[0] for m in d])
    if fmt != 1:
        L["sg"] = np.stack([m[1] for m in g]); L["su"] = np.stack([m[1] for m in u])
        L["sd"] = np.stack([m[1] for m in d])
    else:
        L["bg"] = np.stack([m[1] for m in g]); L["bu"] = np.stack([m[1] for m in u])
        L["bd"] = np.stack([m[1] for m in d])
        L["tg"] = rng.uniform(0.5, 2.0, E).astype(np.float32) / math.sqrt(H)
        L["tu"] = rng.uniform(0.5, 2.0, E).astype(np.float32) / math.sqrt(H)
        L["td"] = rng.uniform(0.5, 2.0, E).astype(np.float32) / math.sqrt(I)
    if n_shared:
        gs, us, ds = mat(I_sh, H), mat(I_sh, H), mat(H, I_sh)
        L["sh_g"], L["sh_u"], L["sh_d"] = gs[0], us[0], ds[0]
        if fmt != 1:
            L["sh_sg"], L["sh_su"], L["sh_sd"] = gs[1], us[1], ds[1]
        else:
            L["sh_bg"], L["sh_bu"], L["sh_bd"] = gs[1], us[1], ds[1]
            L["sh_tg"] = np.float32(0.7 / math.sqrt(H))
            L["sh_tu"] = np.float32(1.3 / math.sqrt(H))
            L["sh_td"] = np.float32(0.9 / math.sqrt(I_sh))
    desc = {"H": H, "I": I, "I_sh": I_sh, "E": E, "k": k, "n_shared": n_shared,
            "scaling": scaling, "fmt": fmt}
    x = f16_bits(rng.standard_normal((5, H)))
    return desc, L, x


def np_expert(desc, L, e, xd):
    """Dense SwiGLU of routed expert e (or the shared expert if e is None), numpy."""
    fmt = desc["fmt"]
    dq = NP_DEQUANT_ROWSCALED.get(fmt)
    if e is None:
        if fmt != 1:
            Wg = dq(L["sh_g"], L["sh_sg"]); Wu = dq(L["sh_u"], L["sh_su"])
            Wd = dq(L["sh_d"], L["sh_sd"])
        else:
            Wg = np_dequant_nvfp4(L["sh_g"], L["sh_bg"], L["sh_tg"])
            Wu = np_dequant_nvfp4(L["sh_u"], L["sh_bu"], L["sh_tu"])
            Wd = np_dequant_nvfp4(L["sh_d"], L["sh_bd"], L["sh_td"])
    else:
        if fmt != 1:
            Wg = dq(L["g"][e], L["sg"][e]); Wu = dq(L["u"][e], L["su"][e])
            Wd = dq(L["d"][e], L["sd"][e])
        else:
            Wg = np_dequant_nvfp4(L["g"][e], L["bg"][e], L["tg"][e])
            Wu = np_dequant_nvfp4(L["u"][e], L["bu"][e], L["tu"][e])
            Wd = np_dequant_nvfp4(L["d"][e], L["bd"][e], L["td"][e])
    h = silu(Wg @ xd) * (Wu @ xd)
    return h, Wd @ h


def _close(a, b, rel, what):
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    err = np.abs(a - b).max() / scale
    assert err <= rel, f"{what}: relative error {err:.3g} > {rel:.3g}"


# ---------------------------------------------------------------- decodes
def pin_half_exhaustive(o):
    """fp16 -> double for all 65536 bit patterns equals numpy's conversion."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "fp16 NaN patterns differ"
    assert np.array_equal(got[~nan], ref[~nan]), "fp16 decode differs from numpy"
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan])), "fp16 sign of zero"


def pin_int4_hand(o):
    """Hand-decoded 5x8 int4 rows (tests/golden/int4_rowscale_4x8.txt)."""
    rows = [r.split("|") for r in _rows("int4_rowscale_4x8.txt")]
    codes = np.array([[int(b, 16) for b in r[0].split()] for r in rows], np.uint8)
    scale = np.array([float(r[1]) for r in rows], np.float32)
    q_ref = np.array([[int(v) for v in r[2].split()] for r in rows])
    v_ref = np.array([[float(v) for v in r[3].split()] for r in rows])
    for n in range(len(rows)):
        assert np.array_equal(o.int4_row(codes[n], 8), q_ref[n]), f"int4 codes, row {n}"
    got = o.dequant({"format": 0, "codes": codes, "row_scale": scale})
    assert np.array_equal(got, v_ref), "int4 dequantised values differ from the hand decode"


def pin_e2m1_table(o):
    """All 16 E2M1 codes against the OCP MX table (tests/golden/e2m1_ocp.txt)."""
    for r in _rows("e2m1_ocp.txt"):
        c, v = r.split()
        got = o.e2m1(int(c))
        assert got == float(v) and math.copysign(1, got) == math.copysign(1, float(v)), \
            f"E2M1 code {c}: {got} != {v}"


def pin_e4m3_exhaustive(o):
    """All 256 E4M3 bytes against torch's float8_e4m3fn conversion and the OFP8 examples."""
    import torch
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = b.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([o.e4m3(i) for i in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "E4M3 NaN set differs"
    assert np.array_equal(got[~nan], ref[~nan]), "E4M3 decode differs from torch"
    for r in _rows("e4m3_ocp.txt"):
        byte, v = r.split()
        g = o.e4m3(int(byte, 16))
        if v == "nan":
            assert math.isnan(g), f"E4M3 {byte} should be NaN"
        else:
            assert g == float(v), f"E4M3 {byte}: {g} != {v}"


def pin_nvfp4_hand(o):
    """Hand-decoded 2x32 NVFP4 matrix (tests/golden/nvfp4_2x32.txt)."""
    kv = {r.split()[0]: r.split()[1:] for r in _rows("nvfp4_2x32.txt")}
    codes = np.array([[int(x, 16) for x in kv[f"row{n}_bytes"]] for n in range(2)], np.uint8)
    bs = np.array([[int(x, 16) for x in kv[f"row{n}_scales"]] for n in range(2)], np.uint8)
    ref = np.array([[float(x) for x in kv[f"row{n}_values"]] for n in range(2)])
    ts = float(kv["tensor_scale"][0])
    got = o.dequant({"format": 1, "codes": codes, "block_scale": bs, "tensor_scale": ts})
    assert np.array_equal(got, ref), f"NVFP4 decode differs:\n{got}\n{ref}"


# ---------------------------------------------------------------- router
def pin_sigmoid_closed_forms(o):
    """sigma(0) = 1/2, sigma(ln 3) = 3/4, sigma(-ln 3) = 1/4, sigma(ln 9) = 9/10,
    sigma(x) + sigma(-x) = 1, monotone, saturation."""
    assert o.sigmoid_f32(0.0) == np.float32(0.5)
    assert o.sigmoid_f32(np.float32(math.log(3))) == np.float32(0.75)
    assert o.sigmoid_f32(np.float32(-math.log(3))) == np.float32(0.25)
    assert abs(float(o.sigmoid_f32(np.float32(math.log(9)))) - 0.9) < 1e-7
    xs = np.float32(np.linspace(-12, 12, 97))
    s = np.array([o.sigmoid_f32(v) for v in xs], np.float64)
    sm = np.array([o.sigmoid_f32(-v) for v in xs], np.float64)
    assert np.all(np.abs(s + sm - 1.0) <= 2 ** -23), "sigmoid symmetry"
    assert np.all(np.diff(s) > 0), "sigmoid not increasing"
    assert o.sigmoid_f32(np.float32(40.0)) == np.float32(1.0)
    assert 0 < o.sigmoid_f32(np.float32(-40.0)) < 1e-17


def pin_router_onehot(o):
    """One-hot activations select one column of W_r: logits = x_h * W_r[:, h] exactly
    (E != H, so a transposed W_r cannot pass)."""
    rng = np.random.default_rng(3)
    E, H = 5, 7
    Wr = rng.standard_normal((E, H)).astype(np.float32)
    vals = [1.0, 2.0, -0.5, 0.25, -4.0, 1.5, 3.0]
    x = np.zeros((H, H), np.float16)
    for h in range(H):
        x[h, h] = vals[h]
    logits = o.router_logits(x.view(np.uint16), Wr)
    ref = (np.array(vals, np.float32)[:, None] * Wr.T).astype(np.float32)
    assert np.array_equal(logits, ref), "router logits on one-hot inputs"


def pin_router_matmul(o):
    """Random case: logits = fp32(x @ W_r^T) with numpy's float64 matmul (library)."""
    rng = np.random.default_rng(4)
    T, E, H = 6, 9, 40
    x = f16_bits(rng.standard_normal((T, H)))
    Wr = (rng.standard_normal((E, H)) / math.sqrt(H)).astype(np.float32)
    ref = (x.view(np.float16).astype(np.float64) @ Wr.astype(np.float64).T).astype(np.float32)
    got = o.router_logits(x, Wr)
    ulp = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1, "router logits differ from numpy by more than 1 ulp"


def _sel_ref(o, logits, bias):
    s = np.array([[o.sigmoid_f32(v) for v in row] for row in logits], np.float32)
    return s, (s + bias[None, :]).astype(np.float32)


def pin_topk_bruteforce(o):
    """Over all C(E,k) subsets, the chosen set maximises the summed selection score and
    the emitted order is descending score, equal scores by lower expert index."""
    rng = np.random.default_rng(5)
    for E, k, trials in ((6, 2, 30), (8, 3, 30), (5, 5, 5), (7, 1, 20)):
        for tr in range(trials):
            T = 3
            if tr % 2:   # coarse values so that ties happen
                logits = rng.integers(-3, 4, (T, E)).astype(np.float32) * 0.5
                bias = rng.integers(-1, 2, E).astype(np.float32) * 0.125
            else:
                logits = rng.standard_normal((T, E)).astype(np.float32)
                bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
            idx, w, sel, gap = o.route(logits, bias, k, 2.5)
            _, sel_ref = _sel_ref(o, logits, bias)
            assert np.array_equal(sel, sel_ref), "selection score = fp32(sigmoid) + bias"
            for t in range(T):
                best = max(sum(float(sel_ref[t, e]) for e in c)
                           for c in itertools.combinations(range(E), k))
                got = sum(float(sel_ref[t, e]) for e in idx[t])
                assert got == best, f"top-{k} of {E}: subset not maximal"
                assert len(set(idx[t].tolist())) == k
                for j in range(k - 1):
                    a, b = idx[t, j], idx[t, j + 1]
                    assert sel_ref[t, a] > sel_ref[t, b] or (sel_ref[t, a] == sel_ref[t, b] and a < b), \
                        "order: descending score, ties by lower index"
                # tie rule at the boundary: an unchosen expert with the same score as the
                # last chosen one must have a higher index
                last = sel_ref[t, idx[t, -1]]
                for e in set(range(E)) - set(idx[t].tolist()):
                    assert sel_ref[t, e] < last or (sel_ref[t, e] == last and e > idx[t, -1])


def pin_route_weights(o):
    """Combine weights: sum to the scaling factor, proportional to the unbiased
    sigmoid score, and equal scaling/k when all scores are equal whatever the bias."""
    rng = np.random.default_rng(6)
    E, k, T = 16, 4, 8
    logits = rng.standard_normal((T, E)).astype(np.float32) * 2
    bias = rng.uniform(-0.5, 0.5, E).astype(np.float32)
    idx, w, sel, gap = o.route(logits, bias, k, 2.5)
    s, _ = _sel_ref(o, logits, bias)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 2.5) <= k * 2 ** -22), "sum w != 2.5"
    for t in range(T):
        ss = s[t, idx[t]].astype(np.float64)
        _close(w[t], 2.5 * ss / ss.sum(), 1e-7, "w proportional to s")
    # all logits equal: the bias alone picks the experts, the weights stay equal
    logits = np.zeros((1, 6), np.float32)
    bias = np.array([0.0, 0.3, 0.0, 0.2, -0.1, 0.0], np.float32)
    idx, w, sel, gap = o.route(logits, bias, 2, 2.5)
    assert idx[0].tolist() == [1, 3], idx
    assert np.array_equal(w[0], np.float32([1.25, 1.25])), w
    assert abs(float(gap[0]) - float(np.float32(0.7) - np.float32(0.5))) < 1e-7, gap


# ---------------------------------------------------------------- int8 / int2 and quantisation
def pin_int8_int2_hand(o):
    """Hand decodes: int8 bytes 0x00 0x01 0x7F 0x80 0xFF 0xFE 0x40 0xC0 are 0 1 127 -128 -1
    -2 64 -64; int2 byte 0xE4 (11 10 01 00) holds 0 1 -2 -1 from element 0 up, 0x1B
    (00 01 10 11) holds -1 -2 1 0; the row scale multiplies."""
    b8 = np.array([0x00, 0x01, 0x7F, 0x80, 0xFF, 0xFE, 0x40, 0xC0], np.uint8)
    assert o.int8_row(b8, 8).tolist() == [0, 1, 127, -128, -1, -2, 64, -64]
    b2 = np.array([0xE4, 0x1B], np.uint8)
    assert o.int2_row(b2, 8).tolist() == [0, 1, -2, -1, -1, -2, 1, 0]
    M8 = {"format": 2, "codes": b8.reshape(1, 8), "row_scale": np.float32([0.5])}
    assert o.dequant(M8)[0].tolist() == [0.0, 0.5, 63.5, -64.0, -0.5, -1.0, 32.0, -32.0]
    M2 = {"format": 3, "codes": np.array([[0xE4, 0x1B], [0xFF, 0x55]], np.uint8),
          "row_scale": np.float32([0.25, 2.0])}
    assert o.dequant(M2).tolist() == [[0.0, 0.25, -0.5, -0.25, -0.25, -0.5, 0.25, 0.0],
                                      [-2.0, -2.0, -2.0, -2.0, 2.0, 2.0, 2.0, 2.0]]


def pin_quantize_hand(o):
    """Exact rows: scale = max|w| / (2^(bits-1) - 1); codes round half to even."""
    codes, sc = o.quantize(np.array([[3.0, -7.0, 1.0, 0.5], [1.5, -3.5, 2.5, 0.25],
                                     [0.0, 0.0, 0.0, 0.0], [0.75, -0.25, 0.0, 1.75]], np.float32), 4)
    assert sc.tolist() == [1.0, 0.5, 0.0, 0.25]
    assert [o.int4_row(codes[r], 4).tolist() for r in range(4)] == [[3, -7, 1, 0], [3, -7, 5, 0],
                                                                     [0, 0, 0, 0], [3, -1, 0, 7]]
    codes, sc = o.quantize(np.array([[127.0, -0.5, 0.5, 1.5, -2.5, 2.5, -127.0, 3.0]], np.float32), 8)
    assert sc.tolist() == [1.0]
    assert o.int8_row(codes[0], 8).tolist() == [127, 0, 0, 2, -2, 2, -127, 3]
    codes, sc = o.quantize(np.array([[2.0, -1.0, 0.5, 1.5, -2.0, 0.0, 1.0, -3.0]], np.float32), 2)
    assert sc.tolist() == [3.0]
    assert o.int2_row(codes[0], 8).tolist() == [1, 0, 0, 0, -1, 0, 0, -1]


def pin_quantize_roundtrip(o):
    """Random rows, every width: codes within range, the largest |w| of a row maps to the
    largest code magnitude, and dequantised values are within half a step of w."""
    rng = np.random.default_rng(12)
    for bits, fmt in ((8, 2), (4, 0), (2, 3)):
        qmax = 2 ** (bits - 1) - 1
        w = (rng.standard_normal((6, 32)) * rng.uniform(0.01, 3.0, (6, 1))).astype(np.float32)
        codes, sc = o.quantize(w, bits)
        deq = o.dequant({"format": fmt, "codes": codes, "row_scale": sc})
        for r in range(6):
            amax = float(np.abs(w[r].astype(np.float64)).max())
            assert sc[r] == np.float32(amax / qmax)
            q = np.rint(deq[r] / float(sc[r])).astype(np.int64)
            assert np.all(np.abs(q) <= qmax) and np.abs(q).max() == qmax
            assert np.all(np.abs(deq[r] - w[r].astype(np.float64)) <= 0.5 * float(sc[r]) * (1 + 1e-6))


# ---------------------------------------------------------------- adaptive top-p
def _logit_of(p):
    """A float32 logit whose fp32 sigmoid is close to p."""
    return np.float32(np.log(p / (1.0 - p)))


def pin_topp_hand(o):
    """Hand example (scores about 0.9, 0.8, 0.3, 0.2 among k = 4 of E = 6, shares of
    the k's mass after 1, 2, 3 experts about 0.41, 0.77, 0.91): p = 0.3 keeps one
    expert, 0.5 two, 0.8 three, 0.95 all four.  A bias that puts the 0.8 expert first
    in top-k order must not change which experts top-p keeps (scores decide), while
    the kept ones stay in top-k order; dropped entries are -1 with weight 0."""
    sv = [0.9, 0.8, 0.3, 0.2, 0.05, 0.04]
    logits = np.array([[_logit_of(v) for v in sv]], np.float32)
    bias = np.zeros(6, np.float32)
    for p, n in ((0.3, 1), (0.5, 2), (0.8, 3), (0.95, 4)):
        idx, w, sel, gap = o.route(logits, bias, 4, 2.5, top_p=p)
        assert idx[0].tolist() == [0, 1, 2, 3][:n] + [-1] * (4 - n), (p, idx)
        assert np.all(w[0, n:] == 0)
        s = np.array([o.sigmoid_f32(float(v)) for v in logits[0, :n]], np.float64)
        _close(w[0, :n], 2.5 * s / s.sum(), 1e-7, "renormalised weights")
    bias = np.array([0.0, 0.2, 0.0, 0.0, 0.0, 0.0], np.float32)   # expert 1 first by selection
    idx, w, sel, gap = o.route(logits, bias, 4, 2.5, top_p=0.3)
    assert idx[0].tolist() == [0, -1, -1, -1], idx                 # the highest score is kept
    idx, w, sel, gap = o.route(logits, bias, 4, 2.5, top_p=0.5)
    assert idx[0].tolist() == [1, 0, -1, -1], idx                  # top-k order kept


def pin_topp_boundary(o):
    """Equal scores (logit 0: s = 1/2 exactly, S = 2 for k = 4).  Expert r is kept only
    while the mass before it is below p * S, so when that mass equals p * S exactly the
    expert is dropped: p = 1/4 keeps one expert, p just above 1/4 keeps two; equal
    scores go in index order.  The gap reports the decision margin."""
    logits = np.zeros((1, 6), np.float32)
    bias = np.array([0.0, 0.0, 0.0, 0.0, -0.5, -0.5], np.float32)
    idx, w, sel, gap = o.route(logits, bias, 4, 2.5, top_p=0.25)
    assert idx[0].tolist() == [0, -1, -1, -1], idx
    assert w[0, 0] == np.float32(2.5)
    assert float(gap[0]) == 0.0, gap
    idx, w, sel, gap = o.route(logits, bias, 4, 2.5, top_p=0.2500001)
    assert idx[0].tolist() == [0, 1, -1, -1], idx
    assert np.array_equal(w[0, :2], np.float32([1.25, 1.25]))
    idx, w, sel, gap = o.route(logits, bias, 4, 2.5, top_p=0.6)
    assert idx[0].tolist() == [0, 1, 2, -1], idx
    assert abs(float(gap[0]) - 0.1) < 1e-6, gap                    # |0.5 - 0.6|


def pin_topp_bruteforce(o):
    """Over all subsets of the k chosen experts: top-p keeps the fewest experts whose
    score mass reaches p times the k's mass, and among those the largest mass; the
    weights sum to the scaling factor; p outside (0, 1) is plain top-k."""
    rng = np.random.default_rng(9)
    for E, k in ((6, 3), (8, 4), (7, 5), (9, 6)):
        for tr in range(25):
            T = 4
            logits = (rng.standard_normal((T, E)) * 1.5).astype(np.float32)
            bias = rng.uniform(-0.2, 0.2, E).astype(np.float32)
            p = float(rng.uniform(0.05, 0.98))
            idx0, w0, _, _ = o.route(logits, bias, k, 2.5)
            idx, w, sel, gap = o.route(logits, bias, k, 2.5, top_p=p)
            for off in (0.0, 1.0, 1.5):
                i2, w2, _, _ = o.route(logits, bias, k, 2.5, top_p=off)
                assert np.array_equal(i2, idx0) and np.array_equal(w2, w0), "top_p off != top-k"
            s, _ = _sel_ref(o, logits, bias)
            for t in range(T):
                chosen = idx0[t].tolist()
                S = sum(float(s[t, e]) for e in chosen)
                kept = [e for e in idx[t].tolist() if e >= 0]
                assert 1 <= len(kept) <= k
                assert kept == [e for e in chosen if e in kept], "kept in top-k order"
                assert all(e == -1 for e in idx[t, len(kept):]) and np.all(w[t, len(kept):] == 0)
                assert abs(float(w[t, :len(kept)].astype(np.float64).sum()) - 2.5) <= len(kept) * 2 ** -22
                if float(gap[t]) < 1e-6:
                    continue   # the decision is within rounding of the threshold
                best = {m: max(itertools.combinations(chosen, m), key=lambda c: sum(float(s[t, e]) for e in c))
                        for m in range(1, k + 1)}
                m_star = min(m for m in range(1, k + 1)
                             if sum(float(s[t, e]) for e in best[m]) >= p * S)
                assert sorted(kept) == sorted(best[m_star]), (p, kept, best[m_star])


# ---------------------------------------------------------------- grouping
def _group_brute(idx, E):
    flat = idx.reshape(-1)   # -1 entries (dropped by top-p) belong to no expert
    counts = np.array([(flat == e).sum() for e in range(E)], np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = np.array([a for e in range(E) for a in range(len(flat)) if flat[a] == e], np.int32)
    unique = np.array([e for e in range(E) if counts[e] > 0], np.int32)
    return counts, offsets, perm, unique


def pin_group_bruteforce(o):
    rng = np.random.default_rng(7)
    cases = [np.zeros((5, 3), np.int32) + 2,                 # all on one expert
             np.arange(12, dtype=np.int32).reshape(4, 3),     # all distinct
             np.array([[4, 0], [0, 4], [3, 1]], np.int32)]
    for _ in range(20):
        T, k, E = int(rng.integers(1, 9)), int(rng.integers(1, 4)), 12
        cases.append(np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32))
    for _ in range(10):   # with top-p drops: a tail of -1 per token
        T, k, E = int(rng.integers(1, 9)), int(rng.integers(2, 5)), 12
        rows = []
        for _ in range(T):
            r = rng.choice(E, k, replace=False).astype(np.int32)
            r[int(rng.integers(1, k + 1)):] = -1
            rows.append(r)
        cases.append(np.stack(rows))
    for idx in cases:
        E = 12
        got = o.group(idx, E)
        ref = _group_brute(idx, E)
        for g, r, name in zip(got, ref, ("counts", "offsets", "perm", "unique")):
            assert np.array_equal(g, r), f"grouping {name} differs from brute force"


# ---------------------------------------------------------------- FFN and layer
def pin_dense_equivalence(o):
    """E=1, k=1, no shared expert, scaling 1: w = s/s = 1, so the layer is a dense
    SwiGLU FFN; with a shared expert and scaling 2.5 it is 2.5*FFN + shared FFN.
    Every weight format: int4, NVFP4, int8, int2."""
    for fmt in (0, 1, 2, 3):
        desc, L, x = small_layer(E=1, k=1, n_shared=0, fmt=fmt, scaling=1.0, seed=11 + fmt)
        r = o.forward(desc, L, x, want_h=True)
        xd = x.view(np.float16).astype(np.float64)
        for t in range(x.shape[0]):
            h, y = np_expert(desc, L, 0, xd[t])
            _close(r["h_assign"][t], h, 1e-12, f"fmt {fmt} dense h")
            _close(r["y"][t], y, 1e-12, f"fmt {fmt} dense y")
        desc, L, x = small_layer(E=1, k=1, n_shared=1, fmt=fmt, scaling=2.5, seed=21 + fmt)
        r = o.forward(desc, L, x)
        xd = x.view(np.float16).astype(np.float64)
        for t in range(x.shape[0]):
            _, y = np_expert(desc, L, 0, xd[t])
            _, ysh = np_expert(desc, L, None, xd[t])
            _close(r["y"][t], 2.5 * y + ysh, 1e-12, f"fmt {fmt} 2.5*FFN + shared")


def pin_layer_composition(o):
    """Several experts: y_t = shared(x_t) + sum_j w_tj * FFN_{e_tj}(x_t) with each
    FFN evaluated densely by numpy and the weights from the (pinned) router."""
    for fmt in (0, 1, 2, 3):
        desc, L, x = small_layer(E=6, k=3, n_shared=1, fmt=fmt, scaling=2.5, seed=31 + fmt)
        r = o.forward(desc, L, x)
        xd = x.view(np.float16).astype(np.float64)
        for t in range(x.shape[0]):
            ref = np_expert(desc, L, None, xd[t])[1].copy()
            for j in range(desc["k"]):
                ref += float(r["topk_w"][t, j]) * np_expert(desc, L, int(r["topk_idx"][t, j]), xd[t])[1]
            _close(r["y"][t], ref, 1e-12, f"fmt {fmt} composed layer")


def pin_union_identity(o):
    """Batch-union driver (each unique expert once over its tokens) == per-token driver,
    bit for bit."""
    for fmt in (0, 1):
        desc, L, x = small_layer(E=4, k=2, n_shared=1, fmt=fmt, scaling=2.5, seed=41 + fmt)
        a = o.forward(desc, L, x)
        b = o.forward(desc, L, x, per_token=True)
        assert a["counts"].max() >= 2, "case should share experts"
        assert np.array_equal(a["y"], b["y"]), "batched != per-token"
        assert np.array_equal(a["y_assign"], b["y_assign"])


def pin_expert_relabel(o):
    """Relabelling experts (permuting W_r rows, bias and expert weights together) maps
    topk_idx through the permutation and leaves y unchanged."""
    desc, L, x = small_layer(E=6, k=2, n_shared=1, fmt=0, scaling=2.5, seed=51)
    pi = np.array([3, 5, 0, 1, 4, 2])          # new index of old expert e is pi[e]
    inv = np.argsort(pi)
    L2 = dict(L)
    for key in ("Wr", "bias", "g", "u", "d", "sg", "su", "sd"):
        L2[key] = np.ascontiguousarray(L[key][inv])
    a = o.forward(desc, L, x)
    b = o.forward(desc, L2, x)
    assert np.array_equal(pi[a["topk_idx"]], b["topk_idx"]), "relabelled routing"
    assert np.array_equal(a["y"], b["y"]), "relabelled output"


def pin_forward_token(o):
    """The single-token driver used for sampled checks equals the batched driver."""
    desc, L, x = small_layer(E=6, k=3, n_shared=1, fmt=0, scaling=2.5, seed=61)
    a = o.forward(desc, L, x)
    for t in range(x.shape[0]):
        b = o.forward_token(desc, L, x[t])
        assert np.array_equal(a["topk_idx"][t], b["topk_idx"])
        assert np.array_equal(a["y"][t], b["y"]), "forward_token != forward"
        assert a["gap"][t] == b["gap"]


def pin_topp_layer(o):
    """With adaptive top-p the batched driver (union of experts) still equals the
    per-token driver bit for bit, the single-token driver equals both, and a layer
    whose p keeps every expert equals the plain top-k layer."""
    desc, L, x = small_layer(E=8, k=4, n_shared=1, fmt=0, scaling=2.5, seed=71)
    desc = dict(desc, top_p=0.55)
    a = o.forward(desc, L, x)
    b = o.forward(desc, L, x, per_token=True)
    assert np.array_equal(a["y"], b["y"]), "top-p: batched != per-token"
    assert (a["topk_idx"] == -1).any(), "p = 0.55 drops some expert"
    for t in range(x.shape[0]):
        c = o.forward_token(desc, L, x[t])
        assert np.array_equal(a["y"][t], c["y"]) and np.array_equal(a["topk_idx"][t], c["topk_idx"])
    assert a["offsets"][-1] == (a["topk_idx"] >= 0).sum(), "only kept assignments are grouped"
    full = o.forward(dict(desc, top_p=0.0), L, x)
    keep_all = o.forward(dict(desc, top_p=0.999999), L, x)
    same = (keep_all["topk_idx"] >= 0).all(axis=1)
    assert np.array_equal(full["y"][same], keep_all["y"][same])


PINS = [pin_half_exhaustive, pin_int4_hand, pin_e2m1_table, pin_e4m3_exhaustive,
        pin_nvfp4_hand, pin_int8_int2_hand, pin_quantize_hand, pin_quantize_roundtrip,
        pin_sigmoid_closed_forms, pin_router_onehot, pin_router_matmul,
        pin_topk_bruteforce, pin_route_weights, pin_topp_hand, pin_topp_boundary,
        pin_topp_bruteforce, pin_group_bruteforce, pin_dense_equivalence,
        pin_layer_composition, pin_union_identity, pin_expert_relabel, pin_forward_token,
        pin_topp_layer]


def run_all(o) -> list[str]:
    """Names of the pins that fail on oracle ``o`` (used by the mutation test)."""
    failed = []
    for p in PINS:
        try:
            p(o)
        except AssertionError:
            failed.append(p.__name__)
    return failed


if __name__ == "__main__":       # python tests/pins.py <liboracle.so>: print failing pins
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    print(",".join(run_all(oracle.Oracle(sys.argv[1]))))
