"""The offline converter (package, host side) against the oracle's quantiser: identical
codes and scales for every width, exact FP8 decoding, and the packed layout the int4
expert kernels read."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_quantized_expert_b200 import quantize as qz


def _rows(seed, N=9, K=64):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * rng.uniform(1e-3, 10.0, (N, 1))).astype(np.float32)
    w[3] = 0.0                                                    # an all-zero row
    w[5] = np.float32(np.arange(K) - K / 2) * np.float32(0.5)      # exact halves: ties
    return w


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_converter_matches_oracle_quantiser(bits):
    o = oracle.default()
    for seed in range(4):
        w = _rows(seed)
        codes, scale = qz.quantize_rows(w, bits)
        rc, rs = o.quantize(w, bits)
        assert np.array_equal(scale.view(np.uint32), rs.view(np.uint32)), "row scales"
        assert np.array_equal(codes, rc), "packed codes"


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_pack_unpack_round_trip(bits):
    rng = np.random.default_rng(bits)
    q = rng.integers(-(1 << (bits - 1)), 1 << (bits - 1), (5, 32))
    assert np.array_equal(qz.unpack(qz.pack(q, bits), bits), q)


def test_int4_layout_is_the_kernels_layout():
    """Element 2b in the low nibble of byte b, two's complement: the oracle's decoder
    (pinned by hand decodes, the one the GPU parity tests compare against) reads back
    the converter's codes."""
    o = oracle.default()
    w = _rows(11)
    codes, scale = qz.quantize_rows(w, 4)
    q = qz.unpack(codes, 4)
    for r in range(w.shape[0]):
        assert np.array_equal(o.int4_row(codes[r], w.shape[1]), q[r])


def test_e4m3_decode_exhaustive():
    b = np.arange(256, dtype=np.uint8)
    got = qz.e4m3_to_float32(b)
    ref = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    o = oracle.default()
    assert all(float(got[i]) == o.e4m3(i) for i in range(256) if not nan[i])


def test_fp8_conversion_with_block_scales():
    rng = np.random.default_rng(3)
    N, K, blk = 256, 256, 128
    fp8 = rng.integers(0, 256, (N, K), dtype=np.uint8)
    fp8[(fp8 & 0x7F) == 0x7F] = 0x38          # no NaN codes
    bs = rng.uniform(0.5, 2.0, (N // blk, K // blk)).astype(np.float32)
    codes, scale = qz.quantize_fp8_rows(fp8, 4, block_scale=bs, block=blk)
    w = (qz.e4m3_to_float32(fp8).astype(np.float64) *
         np.repeat(np.repeat(bs.astype(np.float64), blk, 0), blk, 1)).astype(np.float32)
    rc, rs = oracle.default().quantize(w, 4)
    assert np.array_equal(codes, rc) and np.array_equal(scale, rs)
    with pytest.raises(ValueError):
        qz.quantize_fp8_rows(np.full((2, 8), 0x7F, np.uint8))


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        qz.quantize_rows(np.zeros((2, 3), np.float32), 4)    # K * bits not a byte multiple
    with pytest.raises(ValueError):
        qz.quantize_rows(np.zeros((2, 8), np.float32), 3)
