"""GPU parity of the other row-scaled widths: int8 and int2 expert weights, one fp32 scale
per output row (hakusoku page "Show HN: 低速のコンピュータでGLM 5.2を動かす方法", section
"実装済み機能": int8/int4/int2 kernels with per-row scales).

Both widths run the int8 tensor path of the int4 kernels (exact int8 activation limbs,
weights as s8 bytes, exact integer sums, fp64 epilogue), with their own codecs: int8 codes
are the s8 operand as they are, int2 codes are moved to the top two bits of a byte.  The
checks are those of the int4 path (``gpu_cases.py``): per-expert outputs within 4e-3 of
the FP64 oracle's, layer outputs within 4e-3 over tokens whose top-k decision is not a
near tie, at the decode shapes, at ragged K (stages with fewer 64-value groups, int2 limb
rows that end inside a stage), at batches of several 8-token items, and on activation
rows at the edges of the fp16 range."""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a16_quantized_expert_b200 as moe
from gpu_cases import Case, check_y, desc_of, y_to_f64
from w4a16_quantized_expert_b200.device import DeviceLayer

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
FMTS = {"int8": synth.FMT_INT8, "int2": synth.FMT_INT2}


def _forward(dev, x_dev, T):
    ws = dev.workspace(T)
    y = dev.forward(x_dev[:T], ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    return y, ws


@pytest.mark.parametrize("name", ["int8_1", "int8_8", "int2_1", "int2_8"])
def test_forward_full_size(name):
    """The decode1 shape (H 6144, I 2048, E 256, k 8, shared expert) at T = 1 and 8."""
    case = Case(W[name], experts="routed")
    y, _ = _forward(case.dev, case.x_dev, case.T)
    ref = case.oracle_forward()
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"{name}: excluded {excluded}/{case.T}, rel err {err:.3g}")
    case.dev.close()


@pytest.mark.parametrize("name", ["int8_8", "int2_8"])
def test_expert_ffn_full_size(name):
    """Per-assignment expert outputs (the grouping fed from the oracle) and the shared
    expert's, against the oracle's y_assign and y_shared."""
    case = Case(W[name], experts="routed")
    T = case.T
    ref = case.oracle_forward()
    ws = case.dev.workspace(T)
    ya, ys = case.dev.expert_ffn(case.x_dev, T, torch.from_numpy(ref["offsets"]).cuda(),
                                 torch.from_numpy(ref["perm"]).cuda(), ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(case.dev.handle) == moe.MOE_OK
    ya = ya.cpu().numpy().astype(np.float64)
    ys = ys.cpu().numpy().astype(np.float64)
    valid = ref["topk_idx"].reshape(-1) >= 0
    err_a = np.abs(ya[valid] - ref["y_assign"][valid]).max() / np.abs(ref["y_assign"][valid]).max()
    err_s = np.abs(ys - ref["y_shared"]).max() / np.abs(ref["y_shared"]).max()
    print(f"{name}: y_assign rel err {err_a:.3g}, y_shared {err_s:.3g}")
    assert err_a <= 4e-3 and err_s <= 4e-3
    case.dev.close()


def _small(fmt, T, E, k, H, I, seed):
    w = synth.Workload("width_small", T, H, I, I, E, k, 1, 2.5, fmt, "uniform", seed)
    host = synth.make_layer(w)
    desc = desc_of(w)
    x = synth.make_tokens(w, T)
    dev = DeviceLayer(desc, host, max_tokens=T)
    return w, host, desc, x, dev


# (T, E, k, H, I): K = 320 / 192 leave the last int8 stage with one or three 64-value groups
# and end the int2 limb rows inside a stage (two 256-value blocks of a 512-value stage);
# T = 17 and 40 make several 8-token items per expert and more than one router token tile
SMALL = [(1, 16, 2, 256, 128), (6, 16, 4, 320, 192), (17, 8, 8, 576, 320), (40, 32, 4, 512, 256),
         (5, 5, 2, 1088, 64)]


@pytest.mark.parametrize("fmt", sorted(FMTS))
@pytest.mark.parametrize("T,E,k,H,I", SMALL)
def test_forward_small_and_ragged(fmt, T, E, k, H, I):
    w, host, desc, x, dev = _small(FMTS[fmt], T, E, k, H, I, 7000 + T + H)
    y, ws = _forward(dev, torch.from_numpy(x.copy()).cuda(), T)
    ref = oracle.default().forward(desc, host, x)
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"{fmt} T={T} E={E} k={k} H={H} I={I}: excluded {excluded}/{T}, rel err {err:.3g}")
    # deterministic: a second call on the same workspace gives the same bits
    y2 = dev.forward(torch.from_numpy(x.copy()).cuda(), ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    dev.close()


@pytest.mark.parametrize("fmt", sorted(FMTS))
def test_expert_ffn_bits_and_codes(fmt):
    """Every code value of the width in one layer: a tiny layer whose code bytes run through
    all 256 byte values, against the oracle's per-expert outputs."""
    w = synth.Workload("width_codes", 4, 256, 128, 128, 4, 2, 1, 2.5, FMTS[fmt], "uniform", 4242)
    host = synth.make_layer(w)
    for key in ("g", "u", "d", "sh_g", "sh_u", "sh_d"):
        a = host[key]
        host[key] = (np.arange(a.size, dtype=np.int64) * 37 % 256).astype(np.uint8).reshape(a.shape)
    desc = desc_of(w)
    x = synth.make_tokens(w, 4)
    dev = DeviceLayer(desc, host, max_tokens=4)
    ref = oracle.default().forward(desc, host, x)
    ws = dev.workspace(4)
    ya, ys = dev.expert_ffn(torch.from_numpy(x.copy()).cuda(), 4, torch.from_numpy(ref["offsets"]).cuda(),
                            torch.from_numpy(ref["perm"]).cuda(), ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    err_a = np.abs(ya.cpu().numpy() - ref["y_assign"]).max() / np.abs(ref["y_assign"]).max()
    err_s = np.abs(ys.cpu().numpy() - ref["y_shared"]).max() / np.abs(ref["y_shared"]).max()
    assert err_a <= 4e-3 and err_s <= 4e-3, (err_a, err_s)
    dev.close()


FACTORS = {"outlier": (2.0 ** -8, 1.0, 1.0), "near_max": (2.0 ** -9, 2.0 ** -2, 1.0),
           "subnormal": (2.0 ** 12, 1.0, 2.0 ** 14), "mixed": (1.0, 1.0, 1.0)}


@pytest.mark.parametrize("name,T,kind", [("int8_1", 1, "outlier"), ("int8_8", 8, "near_max"),
                                         ("int8_8", 8, "subnormal"), ("int2_1", 1, "outlier"),
                                         ("int2_8", 8, "near_max"), ("int2_8", 8, "mixed")])
def test_forward_activation_edge_cases(name, T, kind):
    """Activation rows at the edges of the fp16 range (outliers 2^12..2^15, values near
    65504, subnormals) through the limb representation, with the weights scaled by powers
    of two so that h and y stay inside the fp16 range."""
    w = W[name]
    fgu, fd, fr = FACTORS[kind]
    x = synth.make_stress_tokens(w, T, kind)
    Wr, bias = synth.make_router(w)
    o = oracle.default()
    logits = o.router_logits(x, synth.scale_layer({"Wr": Wr}, w.fmt, 1.0, 1.0, fr)["Wr"])
    _, _, sel, _ = o.route(logits, bias, w.k, w.scaling)
    host = {"Wr": Wr, "bias": bias}
    host.update(synth.make_experts(w, np.unique(np.argsort(-sel, axis=1, kind="stable")[:, : w.k + 2])))
    host = synth.scale_layer(host, w.fmt, fgu, fd, fr)
    desc = desc_of(w)
    ref = o.forward(desc, host, x)
    dev = DeviceLayer(desc, host, max_tokens=T)
    y, _ = _forward(dev, torch.from_numpy(x.copy()).cuda(), T)
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    assert excluded < T
    print(f"{name} {kind}: excluded {excluded}/{T}, rel err {err:.3g}")
    dev.close()


def test_one_launch_layer_rejects_other_widths():
    """moe_forward_fused takes int4 and NVFP4 weights only."""
    w, host, desc, x, dev = _small(synth.FMT_INT8, 2, 16, 2, 256, 128, 1)
    ws = dev.workspace(2)
    xd = torch.from_numpy(x.copy()).cuda()
    y = torch.empty_like(xd)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward_fused(dev.handle, xd.data_ptr(), 2, y.data_ptr(), ws.data_ptr(), ws.numel(), 0)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
    dev.close()
