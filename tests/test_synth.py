"""The seeded input generator: determinism, distributions and its format encoders."""
import math

import numpy as np
import torch

import synth


def test_counter_based_determinism():
    a = synth.random_bytes(7, 123, 1 << 20)
    b = synth.random_bytes(7, 123, 1 << 20)
    c = synth.random_bytes(7, 124, 1 << 20)
    assert np.array_equal(a, b)
    assert (a != c).mean() > 0.99
    # prefix property: a shorter draw is a prefix of a longer one
    assert np.array_equal(synth.random_bytes(7, 123, 1000), a[:1000])


def test_int4_codes_uniform():
    b = synth.random_bytes(1, 1, 1 << 20)
    nib = np.concatenate([b & 15, b >> 4])
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.97 * counts.mean() and counts.max() < 1.03 * counts.mean()


def test_normal_and_uniform_moments():
    z = synth.normal_f32(3, 9, 1 << 20, std=2.0)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 2.0) < 0.01
    u = synth.uniform_f32(3, 10, 1 << 20, 0.01, 0.03)
    assert u.min() >= 0.01 and u.max() <= 0.03 and abs(u.mean() - 0.02) < 1e-4


def test_half_encoder_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(20000) * 10 ** rng.uniform(-8, 4.8, 20000),
                           [0.0, -0.0, 65504.0, 65519.0, 65520.0, 2 ** -24, 2 ** -25, 3 * 2 ** -26]])
    got = np.array([synth.lib().synth_half_from_double(float(v)) for v in vals], np.uint16)
    with np.errstate(over="ignore"):   # 65520 and above round to infinity on purpose
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_e4m3_encoder_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.abs(rng.standard_normal(20000)) * 10 ** rng.uniform(-3.5, 2.6, 20000)
    vals = vals[vals < 440]
    r = torch.from_numpy(vals).to(torch.float8_e4m3fn)
    ref = r.view(torch.uint8).numpy()
    import ctypes
    out = ctypes.c_double()
    got = np.array([synth.lib().synth_e4m3_from_double(float(v), ctypes.byref(out)) for v in vals],
                   np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_encoder_ties_to_even():
    enc = synth.lib().synth_e2m1_from_double
    grid = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    for v, c in grid.items():
        assert enc(v) == c and enc(-v) == (c | 8 if c else 0)
    # midpoints go to the even code
    assert enc(0.25) == 0 and enc(0.75) == 2 and enc(1.25) == 2 and enc(1.75) == 4
    assert enc(2.5) == 4 and enc(3.5) == 6 and enc(5.0) == 6 and enc(9.0) == 7


def test_nvfp4_blocks_use_full_range():
    codes, bs = synth.nvfp4_block(5, 77, 64, 256)
    assert codes.shape == (64, 128) and bs.shape == (64, 16)
    # the block maximum maps near code 6.0 (magnitude code 7) in most blocks
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(64, 256)
    blk = (nib & 7).reshape(64, 16, 16).max(-1)
    assert (blk >= 6).mean() > 0.95
    assert not np.any((bs & 0x7F) == 0x7F)      # never NaN


def test_zipf_bias_range_and_shape():
    b = synth.zipf_bias(9, 1, 256, 1.1, -0.5, 0.5)
    assert math.isclose(b.max(), 0.5) and math.isclose(b.min(), -0.5, abs_tol=1e-7)
    srt = np.sort(b)[::-1]
    z = np.arange(1, 257) ** -1.1
    ref = -0.5 + (z - z.min()) / (z.max() - z.min())
    assert np.allclose(srt, ref, atol=1e-7)


def test_workload_tiny_layer_shapes():
    w = synth.WORKLOADS["tiny"]
    L = synth.make_layer(w)
    assert L["g"].shape == (16, 128, 128) and L["d"].shape == (16, 256, 64)
    assert L["sh_g"].shape == (128, 128) and L["sh_sd"].shape == (256,)
    x = synth.make_tokens(w)
    assert x.shape == (4, 256) and x.dtype == np.uint16
    part = synth.make_experts(w, experts=[3])
    assert np.array_equal(part["g"][3], L["g"][3]) and not part["g"][2].any()


def test_stress_tokens_hold_the_promised_values():
    w = synth.WORKLOADS["decode8"]
    f = {k: synth.make_stress_tokens(w, 8, k).view(np.float16).astype(np.float64) for k in synth.STRESS_KINDS}
    for k, v in f.items():
        assert v.shape == (8, w.H) and np.isfinite(v).all(), k
    a = np.abs(f["outlier"])
    top = np.sort(a, axis=1)[:, -1]
    assert np.all((top >= 2.0 ** 12) & (top < 2.0 ** 16))
    assert np.all(np.sort(a, axis=1)[:, -3] < 8)              # at most two outliers per row
    a = np.abs(f["near_max"])
    assert np.all(a.max(axis=1) == 65504.0) and np.all((a == 65472.0).sum(axis=1) >= 1)
    a = np.abs(f["subnormal"])
    assert np.all((a > 0) & (a < 2.0 ** -14)) and np.all(a * 2.0 ** 24 == np.round(a * 2.0 ** 24))
    a = np.abs(f["mixed"])
    sub = (a > 0) & (a < 2.0 ** -14)
    assert 0.15 < sub.mean() < 0.35
    base = synth.make_tokens(w, 8).view(np.float16).astype(np.float64)
    assert np.array_equal(f["mixed"][~sub], base[~sub])


def test_scale_layer_scales_by_exact_powers_of_two():
    w = synth.WORKLOADS["tiny"]
    L = synth.make_layer(w)
    S = synth.scale_layer(L, w.fmt, 2.0 ** -8, 2.0 ** 3, 2.0 ** 5)
    assert np.array_equal(S["sg"], L["sg"] * np.float32(2.0 ** -8)) and np.array_equal(S["sh_su"], L["sh_su"] / 256)
    assert np.array_equal(S["sd"], L["sd"] * 8) and np.array_equal(S["Wr"], L["Wr"] * 32)
    assert S["g"] is L["g"] and np.array_equal(L["sg"], synth.make_layer(w)["sg"])   # input untouched
