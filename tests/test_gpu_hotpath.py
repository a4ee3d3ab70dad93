"""Parity of what the fused layer call (moe_forward) itself computes on the way to y, and of
activations at the edges of the fp16 range.

1. Grouping on the hot path.  moe_forward routes and groups inside its own kernels, not
   through moe_group; a wrong permutation order would still give the right y, so y alone
   cannot catch it.  After the call the routing and grouping arrays are read back from
   the workspace (moe_workspace_routing says where they are) and compared with the
   oracle: logits within fp32 accumulation error, top-k and weights equal to the oracle's
   routing of those logits, counts / offsets / perm / unique bit-exact against the
   oracle's grouping of that top-k (the batch MoE union of the hakusoku page, section
   "実装済み機能"; deterministic order: the GLM-5.3-Flash vLLM page, section
   "Ampere世代のGPU向けに最適化された独自カーネル群"), and the top-k equal to the oracle's
   own routing on every token that is not a near tie.

2. Activation edge cases.  The int4 path carries each fp16 activation row as three exact
   int8 limbs with one power-of-two scale per row; values far below the row maximum are
   rounded.  Rows with outlier channels 2^12 .. 2^15 above the rest, rows at the largest
   finite fp16 values, rows of fp16 subnormals and rows mixing subnormals with N(0,1)
   values (synth.make_stress_tokens) go through the whole layer and are compared with the
   FP64 oracle at the layer's tolerance, on the decode kernels (T = 1, 8), a 40-token batch
   on the int8 path (5 tokens per expert) and on the tensor-memory kernel (20 tokens per
   expert), and the NVFP4 path.  The layer's weights are scaled by
   powers of two (synth.scale_layer) so that h and y stay inside the fp16 range; the test
   checks that on the oracle's values first.

3. The one-launch decode path (moe_forward_fused): its own routing and grouping read back
   the same way, the whole layer against the oracle and against moe_forward (bit for bit
   with int4 weights), edge-case activations, guard bands and the T > 16 rejection.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a16_quantized_expert_b200 as moe
from gpu_cases import GAP_MIN, W_RTOL, check_y, desc_of, y_to_f64
from w4a16_quantized_expert_b200.device import DeviceLayer

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
E1024 = W["tiny"].with_(E=1024, k=8, name="tiny_e1024")
BATCH = synth.Workload("stress_batch", 40, 1024, 512, 512, 32, 4, 1, 2.5, synth.FMT_INT4, "uniform",
                       synth.BASE_SEED + 40)
# the same batch over 8 experts: 20 tokens per expert, past the int8 path's share
BATCH_TC = BATCH.with_(E=8, name="stress_batch_tc")


def _workload(name):
    return E1024 if name == "tiny_e1024" else W[name]


def ws_routing(dev, ws, T):
    """The routing and grouping arrays moe_forward left in the workspace."""
    r = moe.moe_workspace_routing(dev.handle, T)
    b = ws.cpu().numpy()
    k, E = dev.d["k"], dev.d["E"]

    def a(key, n, dt=np.int32):
        return b[r[key]: r[key] + 4 * n].view(dt).copy()

    out = {"logits": a("logits", T * E, np.float32).reshape(T, E),
           "topk_idx": a("topk_idx", T * k).reshape(T, k),
           "topk_w": a("topk_w", T * k, np.float32).reshape(T, k),
           "counts": a("counts", E), "offsets": a("offsets", E + 1)}
    nu = int(a("n_unique", 1)[0])
    out["perm"] = a("perm", T * k)[: out["offsets"][E]]
    out["unique"] = a("unique", E)[:nu]
    return out


GROUP_CASES = [("decode1", 1, 0.0), ("tiny", 1, 0.0), ("tiny_e1024", 1, 0.0), ("nvfp4_1", 1, 0.0),
               ("decode1", 1, 0.7), ("tiny", 4, 0.0), ("decode8", 8, 0.0), ("nvfp4_16", 16, 0.0),
               ("tiny", 16, 0.0), ("tiny", 17, 0.0), ("tiny", 37, 0.0), ("prefill512", 512, 0.0),
               ("decode8", 8, 0.7), ("tiny", 4, 0.5), ("tiny", 37, 0.5), ("tiny_e1024", 9, 0.0),
               ("tiny_e1024", 40, 0.0)]


@pytest.mark.parametrize("name,T,p", GROUP_CASES)
def test_forward_routing_and_grouping_match_the_oracle(name, T, p):
    w = _workload(name)
    if p:
        w = w.with_(top_p=p)
    host = synth.make_layer(w, experts=[0])     # expert values do not enter routing
    desc = desc_of(w)
    dev = DeviceLayer(desc, host, max_tokens=T)
    x = synth.make_tokens(w, T)
    ws = dev.workspace(T)
    dev.forward(torch.from_numpy(x.copy()).cuda(), ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    g = ws_routing(dev, ws, T)
    _check_routing_arrays(g, host, desc, x, w)
    dev.close()


@pytest.mark.parametrize("name,T", [("decode1", 1), ("tiny", 37)])
def test_host_forward_routing_and_grouping_match_the_oracle(name, T):
    w = _workload(name)
    host = synth.make_layer(w, experts=[0])
    desc = desc_of(w)
    dev = DeviceLayer(desc, host, max_tokens=T)
    x = synth.make_tokens(w, T)
    ws = dev.workspace(T)
    xh = torch.from_numpy(x.copy()).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    dev.forward_host(xh, yh, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    _check_routing_arrays(ws_routing(dev, ws, T), host, desc, x, w)
    dev.close()


def _check_routing_arrays(g, host, desc, x, w):
    o = oracle.default()
    T = x.shape[0]
    ref_logits = o.router_logits(x, host["Wr"])
    # logits: fp32 accumulation of the same products
    assert np.abs(g["logits"] - ref_logits).max() <= 1e-5 * np.abs(ref_logits).max() + 1e-6
    # top-k (and top-p) and weights: the oracle's routing of the GPU's own logits
    idx_g, w_g, _, _ = o.route(g["logits"], host["bias"], w.k, desc["scaling"], desc["top_p"])
    assert np.array_equal(g["topk_idx"], idx_g), "top-k differs from the oracle's routing of the same logits"
    kept = idx_g >= 0
    assert np.all(g["topk_w"][~kept] == 0)
    rel = np.abs(g["topk_w"][kept].astype(np.float64) - w_g[kept]) / np.abs(w_g[kept])
    assert rel.max() <= W_RTOL, f"topk_w relative error {rel.max():.3g}"
    # grouping: bit-exact against the oracle's grouping of that top-k
    c, off, perm, uniq = o.group(g["topk_idx"], w.E)
    assert np.array_equal(g["counts"], c), "counts"
    assert np.array_equal(g["offsets"], off), "offsets"
    assert np.array_equal(g["perm"], perm), "perm"
    assert np.array_equal(g["unique"], uniq), "unique"
    # and the top-k is the oracle's own on every token that is not a near tie
    idx_r, _, _, gap = o.route(ref_logits, host["bias"], w.k, desc["scaling"], desc["top_p"])
    keep = gap >= GAP_MIN
    assert keep.sum() >= (T + 1) // 2, f"too many near ties ({int((~keep).sum())}/{T})"
    assert np.array_equal(g["topk_idx"][keep], idx_r[keep])


# ------------------------------------------------------------------ activation edge cases
# (gate/up, down, router) weight factors per kind: h and y inside the fp16 range, and
# router logits of subnormal rows large enough that the scores, not the bias alone, order
# the experts
FACTORS = {"outlier": (2.0 ** -8, 1.0, 1.0), "near_max": (2.0 ** -9, 2.0 ** -2, 1.0),
           "subnormal": (2.0 ** 12, 1.0, 2.0 ** 14), "mixed": (1.0, 1.0, 1.0)}

STRESS_CASES = [(n, T, kind) for n, T in (("decode1", 1), ("stress_batch", 40), ("stress_batch_tc", 40),
                                          ("nvfp4_1", 1))
                for kind in synth.STRESS_KINDS] + \
               [("decode8", 8, "outlier"), ("decode8", 8, "subnormal"), ("decode8", 8, "near_max"),
                ("nvfp4_16", 16, "outlier"), ("nvfp4_16", 16, "subnormal")]


@pytest.mark.parametrize("name,T,kind", STRESS_CASES)
def test_forward_activation_edge_cases(name, T, kind):
    w = {"stress_batch": BATCH, "stress_batch_tc": BATCH_TC}.get(name) or W[name]
    fgu, fd, fr = FACTORS[kind]
    if kind == "subnormal" and w.fmt == synth.FMT_NVFP4:
        fgu *= 8.0     # NVFP4 weights are about 4x smaller than the int4 ones
    x = synth.make_stress_tokens(w, T, kind)
    Wr, bias = synth.make_router(w)
    o = oracle.default()
    logits = o.router_logits(x, synth.scale_layer({"Wr": Wr}, w.fmt, 1.0, 1.0, fr)["Wr"])
    _, _, sel, _ = o.route(logits, bias, w.k, w.scaling)
    experts = np.unique(np.argsort(-sel, axis=1, kind="stable")[:, : w.k + 2])
    host = {"Wr": Wr, "bias": bias}
    host.update(synth.make_experts(w, experts))
    host = synth.scale_layer(host, w.fmt, fgu, fd, fr)
    desc = desc_of(w)
    ref = o.forward(desc, host, x, want_h=True)
    # the construction keeps h and y inside the fp16 range (checked on the oracle's values)
    h_max = max(np.abs(ref["h_assign"]).max(), np.abs(ref["h_shared"]).max())
    assert h_max < 32768 and np.abs(ref["y"]).max() < 32768, (h_max, np.abs(ref["y"]).max())
    dev = DeviceLayer(desc, host, max_tokens=T)
    ws = dev.workspace(T)
    y = dev.forward(torch.from_numpy(x.copy()).cuda(), ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    assert excluded < T, "every token excluded as a near tie"
    print(f"{name} {kind}: excluded {excluded}/{T}, rel err {err:.3g}")
    dev.close()


# ------------------------------------------------------------------ one-launch decode path
@pytest.mark.parametrize("name,T,p", [("decode1", 1, 0.0), ("tiny", 4, 0.0), ("decode8", 8, 0.0),
                                      ("nvfp4_16", 16, 0.0), ("tiny", 16, 0.0), ("decode8", 8, 0.7),
                                      ("tiny", 4, 0.5), ("tiny_e1024", 9, 0.0)])
def test_fused_path_routing_and_grouping_match_the_oracle(name, T, p):
    """moe_forward_fused routes and groups in its own router tasks and finishing task."""
    w = _workload(name)
    if p:
        w = w.with_(top_p=p)
    host = synth.make_layer(w, experts=[0])
    desc = desc_of(w)
    dev = DeviceLayer(desc, host, max_tokens=T)
    x = synth.make_tokens(w, T)
    ws = dev.workspace(T)
    dev.forward(torch.from_numpy(x.copy()).cuda(), ws, fused=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    _check_routing_arrays(ws_routing(dev, ws, T), host, desc, x, w)
    dev.close()


FUSED_CASES = [("tiny", 1), ("tiny", 2), ("tiny", 3), ("tiny", 4), ("tiny", 9), ("tiny", 15), ("tiny", 16),
               ("decode1", 1), ("decode8", 8), ("nvfp4_1", 1), ("nvfp4_16", 16)]


@pytest.mark.parametrize("name,T", FUSED_CASES)
def test_fused_forward_matches_the_oracle_and_moe_forward(name, T):
    """The whole layer in one launch against the FP64 oracle, and against moe_forward: bit
    for bit with int4 weights, within tolerance with NVFP4; run twice (counters and flags
    left ready for the next call)."""
    w = W[name]
    x = synth.make_tokens(w, T, batch=T)
    if name == "tiny":
        host = synth.make_layer(w)
    else:
        logits = oracle.default().router_logits(x, synth.make_router(w)[0])
        _, _, sel, _ = oracle.default().route(logits, synth.make_router(w)[1], w.k, w.scaling)
        host = synth.make_layer(w, experts=np.unique(np.argsort(-sel, axis=1, kind="stable")[:, : w.k + 2]))
    desc = desc_of(w)
    dev = DeviceLayer(desc, host, max_tokens=max(T, 16))
    xd = torch.from_numpy(x.copy()).cuda()
    ws = dev.workspace(T)
    y_ref = dev.forward(xd, ws)
    for _ in range(2):
        y = dev.forward(xd, ws, fused=True)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
        if w.fmt == synth.FMT_INT4:
            assert torch.equal(y, y_ref), "fused path differs from moe_forward"
        ref = oracle.default().forward(desc, host, x)
        excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"{name} T={T} fused: excluded {excluded}/{T}, rel err {err:.3g}")
    dev.close()


@pytest.mark.parametrize("name,T,kind", [("decode1", 1, "outlier"), ("decode1", 1, "subnormal"),
                                         ("decode8", 8, "near_max"), ("nvfp4_1", 1, "outlier")])
def test_fused_forward_activation_edge_cases(name, T, kind):
    w = W[name]
    fgu, fd, fr = FACTORS[kind]
    if kind == "subnormal" and w.fmt == synth.FMT_NVFP4:
        fgu *= 8.0
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
    ws = dev.workspace(T)
    y = dev.forward(torch.from_numpy(x.copy()).cuda(), ws, fused=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    assert excluded < T
    dev.close()


def test_fused_forward_stays_inside_its_buffers_and_rejects_large_batches():
    w = W["tiny"]
    T = 16
    host = synth.make_layer(w)
    dev = DeviceLayer(desc_of(w), host, max_tokens=32)
    n = moe.moe_workspace_size(dev.handle, T)
    G = 4096
    buf = torch.full((G + n + G,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[G:G + n]
    ws.zero_()
    x = torch.from_numpy(synth.make_tokens(w, T).copy()).cuda()
    yb = torch.full((T + 2, w.H), 0x5A5A, dtype=torch.int16, device="cuda").view(torch.uint16)
    for _ in range(3):
        dev.forward(x, ws, y=yb[1:T + 1], fused=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    b = buf.cpu().numpy()
    assert np.all(b[:G] == 0xA5) and np.all(b[G + n:] == 0xA5), "write outside the workspace"
    yh = yb.view(torch.int16).cpu().numpy()
    assert np.all(yh[0] == 0x5A5A) and np.all(yh[T + 1] == 0x5A5A), "write outside y"
    x17 = torch.from_numpy(synth.make_tokens(w, 17).copy()).cuda()
    ws17 = dev.workspace(17)
    with pytest.raises(moe.MoeError) as e:
        dev.forward(x17, ws17, fused=True)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
    dev.close()
