"""GPU parity: every step of the layer through the C ABI against the FP64 oracle on the
same seeded inputs (see ``gpu_cases.py`` for the comparison rules)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a16_quantized_expert_b200 as moe
from gpu_cases import Case, check_routing, check_weights, check_y, y_to_f64

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module")
def tiny():
    return Case(W["tiny"], max_tokens=64)


# ------------------------------------------------------------------ routing
def _route_from_logits(case, T):
    ws = case.dev.workspace(T)
    ref = case.oracle_forward()
    li = torch.from_numpy(ref["logits"]).cuda()
    idx, w, lo = case.dev.route(None, T, ws, logits_in=li, want_logits=True)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"]), "topk_idx differs"
    check_weights(w.cpu().numpy(), ref["topk_w"].astype(np.float64))
    assert np.array_equal(lo.cpu().numpy(), ref["logits"]), "logits_out copy"
    return ref


def test_route_bitexact_from_oracle_logits_tiny(tiny):
    _route_from_logits(tiny, tiny.T)


@pytest.mark.parametrize("name,T", [("decode8", 8), ("nvfp4_16", 16), ("tiny", 37)])
def test_route_bitexact_from_oracle_logits(name, T):
    w = W[name]
    case = Case(w, T=T, experts="routed") if name != "tiny" else Case(w, T=T)
    _route_from_logits(case, T)


@pytest.mark.parametrize("E,k,pattern", [(256, 8, "ties"), (256, 8, "all_equal"), (37, 5, "ties"),
                                          (5, 2, "ties"), (200, 32, "ties"), (256, 1, "random")])
def test_route_single_token_bitexact(E, k, pattern):
    """One token (the whole-CTA top-k and the direct grouping): top-k indices, their order
    and the grouping bit-exact, weights within 1e-6, from oracle logits full of ties
    (values on a coarse grid, or all equal), so the lower-index rule decides often."""
    rng = np.random.default_rng(E * 100 + k)
    if pattern == "all_equal":
        logits = np.zeros((1, E), np.float32)
    elif pattern == "ties":
        logits = (rng.integers(-4, 5, (1, E)) * 0.25).astype(np.float32)
    else:
        logits = rng.standard_normal((1, E)).astype(np.float32)
    w = synth.WORKLOADS["tiny"].with_(E=E, k=k)
    host = {"Wr": np.zeros((E, 256), np.float32), "bias": np.zeros(E, np.float32)}
    if pattern == "ties":   # a bias on the same grid: selection ties among unequal scores
        host["bias"] = (rng.integers(-2, 3, E) * 0.125).astype(np.float32)
    host.update(synth.make_experts(w, experts=[]))
    from w4a16_quantized_expert_b200.device import DeviceLayer
    desc = oracle.desc_of(w)
    dev = DeviceLayer(desc, host, max_tokens=1)
    ws = dev.workspace(1)
    idx, wt, _ = dev.route(None, 1, ws, logits_in=torch.from_numpy(logits).cuda())
    torch.cuda.synchronize()
    r_idx, r_w, _, _ = oracle.default().route(logits, host["bias"], k, float(np.float32(w.scaling)))
    assert np.array_equal(idx.cpu().numpy(), r_idx)
    check_weights(wt.cpu().numpy(), r_w.astype(np.float64))
    counts, offsets, perm, unique, nu = dev.group(idx, 1, ws)
    c_ref, o_ref, p_ref, u_ref = oracle.default().group(r_idx, E)
    assert np.array_equal(counts.cpu().numpy(), c_ref) and np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy()[: len(p_ref)], p_ref)
    assert int(nu.item()) == len(u_ref) and np.array_equal(unique.cpu().numpy()[: len(u_ref)], u_ref)
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK
    dev.close()


def test_route_gemv_logits(tiny):
    T = tiny.T
    ws = tiny.dev.workspace(T)
    idx, w, lo = tiny.dev.route(tiny.x_dev, T, ws, want_logits=True)
    ref = tiny.oracle_forward()
    lo = lo.cpu().numpy()
    assert np.abs(lo - ref["logits"]).max() <= 1e-5 * np.abs(ref["logits"]).max() + 1e-6
    keep = ref["gap"] >= 1e-4
    assert np.array_equal(idx.cpu().numpy()[keep], ref["topk_idx"][keep])


@pytest.mark.parametrize("name,T", [("tiny", 17), ("tiny", 37), ("tiny", 64), ("decode8", 40),
                                    ("prefill512", 512)])
def test_route_logits_batches(name, T):
    """Batches of several token tiles (the GEMM-tiled router): logits within fp32
    accumulation error of the FP64 oracle's, and top-k indices and weights identical to
    the oracle's routing of the GPU's own logits."""
    case = Case(W[name], T=T, experts=[0])
    ws = case.dev.workspace(T)
    idx, w, lo = case.dev.route(case.x_dev, T, ws, want_logits=True)
    torch.cuda.synchronize()
    o = oracle.default()
    ref = o.router_logits(case.x, case.router[0])
    lo = lo.cpu().numpy()
    assert np.abs(lo - ref).max() <= 1e-5 * np.abs(ref).max() + 1e-6
    r_idx, r_w, _, _ = o.route(lo, case.router[1], case.w.k, case.desc["scaling"])
    assert np.array_equal(idx.cpu().numpy(), r_idx), "top-k of the GPU logits"
    check_weights(w.cpu().numpy(), r_w.astype(np.float64))


# ------------------------------------------------------------------ adaptive top-p
@pytest.mark.parametrize("name,T,p", [("tiny", 4, 0.5), ("tiny", 37, 0.5), ("decode8", 8, 0.7),
                                      ("nvfp4_16", 16, 0.7)])
def test_route_topp_bitexact_from_oracle_logits(name, T, p):
    """Fed the oracle's fp32 logits, the GPU's top-p routing (kept experts, their order,
    the -1 tail) is the oracle's, weights within 1e-6."""
    w = W[name].with_(top_p=p)
    case = Case(w, T=T, experts=[0])
    ref = case.oracle_forward()
    ws = case.dev.workspace(T)
    li = torch.from_numpy(ref["logits"]).cuda()
    idx, wt, _ = case.dev.route(None, T, ws, logits_in=li, want_logits=True)
    torch.cuda.synchronize()
    check_routing(idx.cpu().numpy(), wt.cpu().numpy(), ref["topk_idx"], ref["topk_w"].astype(np.float64))
    assert (ref["topk_idx"] == -1).any(), "the case drops some experts"


@pytest.mark.parametrize("name,T,p", [("tiny", 4, 0.5), ("tiny", 37, 0.5), ("decode1", 1, 0.7),
                                      ("decode8", 8, 0.7), ("nvfp4_16", 16, 0.7)])
def test_forward_topp(name, T, p):
    """The whole layer with adaptive top-p against the oracle (tokens near a top-k or a
    top-p decision excluded, as for plain top-k)."""
    w = W[name].with_(top_p=p)
    case = Case(w, T=T, experts="routed") if name != "tiny" else Case(w, T=T, max_tokens=64)
    y, _ = _forward(case)
    ref = case.oracle_forward()
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"{name} top-p {p}: excluded {excluded}/{T}, kept {(ref['topk_idx'] >= 0).sum()}/{ref['topk_idx'].size}, rel err {err:.3g}")


# ------------------------------------------------------------------ grouping
@pytest.mark.parametrize("T,k,E,mode", [(4, 2, 16, "rand"), (1, 8, 256, "rand"), (16, 8, 256, "rand"),
                                        (512, 8, 256, "rand"), (40, 4, 16, "hot"), (9, 3, 1024, "rand"),
                                        (16, 8, 256, "drop"), (300, 8, 256, "drop")])
def test_group_bitexact(T, k, E, mode):
    rng = np.random.default_rng(T * 1000 + E)
    if mode == "hot":
        idx = np.stack([np.concatenate([[0], rng.choice(np.arange(1, E), k - 1, replace=False)])
                        for _ in range(T)]).astype(np.int32)
    else:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    if mode == "drop":   # top-p tails: entries past a random count per token are -1
        for t in range(T):
            idx[t, int(rng.integers(1, k + 1)):] = -1
    w = synth.WORKLOADS["tiny"].with_(E=E, k=k)
    host = {"Wr": np.zeros((E, 256), np.float32), "bias": np.zeros(E, np.float32)}
    host.update(synth.make_experts(w, experts=[]))
    from w4a16_quantized_expert_b200.device import DeviceLayer
    dev = DeviceLayer(oracle.desc_of(w), host, max_tokens=T)
    ws = dev.workspace(T)
    counts, offsets, perm, unique, nu = dev.group(torch.from_numpy(idx).cuda(), T, ws)
    c_ref, o_ref, p_ref, u_ref = oracle.default().group(idx, E)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy()[: len(p_ref)], p_ref)
    n = int(nu.item())
    assert n == len(u_ref) and np.array_equal(unique.cpu().numpy()[:n], u_ref)
    assert moe.moe_get_device_status(dev.handle) == moe.MOE_OK


def test_group_out_of_range_index_is_reported_not_faulted(tiny):
    idx = torch.tensor([[0, 99], [3, -2], [5, 6], [7, 1]], dtype=torch.int32, device="cuda")
    ws = tiny.dev.workspace(4)
    counts, offsets, perm, unique, nu = tiny.dev.group(idx, 4, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(tiny.dev.handle) == moe.MOE_ERR_DEVICE_BOUNDS
    assert int(offsets[-1].item()) == 6        # the two bad assignments were dropped


# ------------------------------------------------------------------ experts
def _ffn_vs_oracle(case, T):
    ref = case.oracle_forward()
    ws = case.dev.workspace(T)
    offsets = torch.from_numpy(ref["offsets"]).cuda()
    perm = torch.from_numpy(ref["perm"]).cuda()
    ya, ys = case.dev.expert_ffn(case.x_dev, T, offsets, perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(case.dev.handle) == moe.MOE_OK
    ya = ya.cpu().numpy().astype(np.float64)
    scale = np.abs(ref["y_assign"]).max()
    err = np.abs(ya - ref["y_assign"]).max() / scale
    assert err <= 4e-3, f"y_assign error {err:.3g}"
    if case.desc["n_shared"]:
        ys = ys.cpu().numpy().astype(np.float64)
        err = np.abs(ys - ref["y_shared"]).max() / np.abs(ref["y_shared"]).max()
        assert err <= 4e-3, f"y_shared error {err:.3g}"
    return ref


def test_expert_ffn_tiny(tiny):
    _ffn_vs_oracle(tiny, tiny.T)


@pytest.mark.parametrize("name,T", [("decode8", 8), ("nvfp4_16", 16), ("nvfp4_1", 1)])
def test_expert_ffn(name, T):
    _ffn_vs_oracle(Case(W[name], T=T, experts="routed"), T)


@pytest.mark.parametrize("T", [33, 49, 64])
def test_expert_ffn_batches(T):
    """The staged expert step on both batch paths (E = 16, k = 2: T = 33 the int8 path,
    its x limbs made by the staged call itself; T = 49 and 64 the tensor-memory kernel)."""
    _ffn_vs_oracle(Case(W["tiny"], T=T, max_tokens=64, batch=T), T)


def test_combine_tiny(tiny):
    T = tiny.T
    ref = tiny.oracle_forward()
    ya = torch.from_numpy(ref["y_assign"].astype(np.float32)).cuda()
    ys = torch.from_numpy(ref["y_shared"].astype(np.float32)).cuda()
    w = torch.from_numpy(ref["topk_w"]).cuda()
    y = tiny.dev.combine(ya, ys, w, T)
    check_y(y_to_f64(y), ref["y"], np.full(T, 1.0))


# ------------------------------------------------------------------ fused layer
def _forward(case, T=None):
    T = case.T if T is None else T
    ws = case.dev.workspace(T)
    y = case.dev.forward(case.x_dev[:T], ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(case.dev.handle) == moe.MOE_OK
    return y, ws


def test_forward_tiny(tiny):
    y, _ = _forward(tiny)
    ref = tiny.oracle_forward()
    check_y(y_to_f64(y), ref["y"], ref["gap"])


@pytest.mark.parametrize("name", ["decode1", "decode8", "nvfp4_1", "nvfp4_16"])
def test_forward_full_size(name):
    case = Case(W[name], experts="routed")
    y, _ = _forward(case)
    ref = case.oracle_forward()
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"{name}: excluded {excluded}/{case.T}, rel err {err:.3g}")


def test_forward_prefill512_sampled():
    """~16 tokens per expert (the tensor-memory kernel's 32-token items): every fourth
    token and the last against the oracle, so that nearly every (expert, token chunk) item
    holds a checked token."""
    case = Case(W["prefill512"])
    y, _ = _forward(case)
    tokens = list(range(0, 512, 4)) + [511]
    ref = case.oracle_forward(tokens=tokens)
    excluded, err = check_y(y_to_f64(y)[tokens], ref["y"], ref["gap"])
    print(f"prefill512 sampled: excluded {excluded}/{len(tokens)}, rel err {err:.3g}")


def test_forward_batch128():
    """About 4 tokens per expert at full size (the int8 path's 8-token items, some experts
    with two items): every token against the oracle."""
    case = Case(W["batch128"])
    y, _ = _forward(case)
    ref = case.oracle_forward(tokens=list(range(128)))
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"batch128: excluded {excluded}/128, rel err {err:.3g}")


def test_forward_prefill2048_sampled():
    """About 64 tokens per expert: 64-token items, several per expert row tile; every
    sixteenth token and the last against the oracle."""
    case = Case(W["prefill2048"])
    y, _ = _forward(case)
    tokens = list(range(0, 2048, 16)) + [2047]
    ref = case.oracle_forward(tokens=tokens)
    excluded, err = check_y(y_to_f64(y)[tokens], ref["y"], ref["gap"])
    print(f"prefill2048 sampled: excluded {excluded}/{len(tokens)}, rel err {err:.3g}")


@pytest.mark.parametrize("E,k,T", [(8, 2, 64),    # 16 tokens per expert: the tensor-memory kernel
                                   (32, 4, 48)])  # 6 tokens per expert: the int8 path
def test_forward_full_T_at_the_decode_shape(E, k, T):
    """Every token of a batch at H = 6144, I = 2048 (the stage counts and ring wrap-around
    of the full-size layer) against the oracle, on both batch paths."""
    case = Case(W["decode1"].with_(E=E, k=k, T=T, name=f"full_T_{E}_{k}_{T}"))
    y, _ = _forward(case)
    ref = case.oracle_forward()
    excluded, err = check_y(y_to_f64(y), ref["y"], ref["gap"])
    print(f"E={E} k={k} T={T}: excluded {excluded}/{T}, rel err {err:.3g}")


# (E = 16, k = 2: up to T = 48, six tokens per expert, the int8 path's 8-token items; from
# T = 49 the tensor-memory kernel)
@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 33, 48, 49, 64])
def test_forward_ragged_T(tiny, T):
    case = Case(W["tiny"], T=T, max_tokens=64, batch=T)
    y, _ = _forward(case)
    ref = case.oracle_forward()
    check_y(y_to_f64(y), ref["y"], ref["gap"])


def test_forward_T0_is_noop(tiny):
    ws = tiny.dev.workspace(0)
    y = torch.zeros((0, 256), dtype=torch.uint16, device="cuda")
    moe.moe_forward(tiny.dev.handle, tiny.x_dev.data_ptr(), 0, y.data_ptr(), ws.data_ptr(), ws.numel(), 0)


def test_staged_equals_fused(tiny):
    T = tiny.T
    ws = tiny.dev.workspace(T)
    y_fused = tiny.dev.forward(tiny.x_dev, ws)
    idx, w, _ = tiny.dev.route(tiny.x_dev, T, ws)
    counts, offsets, perm, unique, nu = tiny.dev.group(idx, T, ws)
    ya, ys = tiny.dev.expert_ffn(tiny.x_dev, T, offsets, perm, ws)
    y_staged = tiny.dev.combine(ya, ys, w, T)
    torch.cuda.synchronize()
    a, b = y_to_f64(y_fused), y_to_f64(y_staged)
    assert np.abs(a - b).max() <= 1e-3 * np.abs(a).max()


def test_determinism_bit_identical():
    case = Case(W["decode8"], experts="routed")
    y1, ws = _forward(case)
    y2 = case.dev.forward(case.x_dev, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_forward_host_matches_forward(tiny):
    T = tiny.T
    ws = tiny.dev.workspace(T)
    y_dev = tiny.dev.forward(tiny.x_dev, ws)
    xh = torch.from_numpy(tiny.x.copy()).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    tiny.dev.forward_host(xh, yh, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_dev.cpu(), yh)


def test_forward_host_pipelined_calls_share_a_workspace(tiny):
    """Consecutive host-buffer calls through two handles that share one workspace (mapped
    page-locked x fetched by the first kernel of each launch chain, one staging buffer):
    every y equals the device-buffer forward of its own tokens, for mapped page-locked y
    (written by the last kernel), pageable y and pageable x (staged copies), eagerly and
    replayed from a CUDA graph."""
    T = tiny.T
    other = tiny.dev.clone_weights()
    ws = tiny.dev.workspace(T)
    xs = [synth.make_tokens(tiny.w, T, batch=10 + b) for b in range(6)]
    refs = []
    for i, x in enumerate(xs):
        dev = tiny.dev if i % 2 == 0 else other
        refs.append(dev.forward(torch.from_numpy(x.copy()).cuda(), ws).cpu())
    torch.cuda.synchronize()
    xh = [torch.from_numpy(x.copy()).pin_memory() if i != 4 else torch.from_numpy(x.copy()) for i, x in enumerate(xs)]
    yh = [torch.zeros_like(x).pin_memory() if i != 3 else torch.zeros_like(x) for i, x in enumerate(xh)]
    stream = torch.cuda.Stream()
    for i in range(len(xs)):
        (tiny.dev if i % 2 == 0 else other).forward_host(xh[i], yh[i], ws, stream=stream)
    stream.synchronize()
    for i in range(len(xs)):
        assert torch.equal(yh[i], refs[i]), f"eager call {i}"
    # the same calls (mapped x and y only) captured once and replayed twice, with new x
    # contents written into the same host buffers before the second replay
    for y in yh:
        y.zero_()
    xh[4] = xh[4].pin_memory()
    yg = [torch.zeros_like(x).pin_memory() for x in xh]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(len(xs)):
            (tiny.dev if i % 2 == 0 else other).forward_host(xh[i], yg[i], ws, stream=stream)
    n = len(xs)
    for rep in range(2):
        for y in yg:
            y.zero_()
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        for i in range(n):   # (the two handles hold the same weights)
            assert torch.equal(yg[i], refs[(i + rep) % n]), f"graph call {i}, replay {rep}"
        # the second replay reads new contents of the same host buffers
        rotated = [xh[(i + 1) % n].clone() for i in range(n)]
        for i in range(n):
            xh[i].copy_(rotated[i])
    del g
    assert moe.moe_get_device_status(tiny.dev.handle) == moe.MOE_OK
    other.close()


# ------------------------------------------------------------------ special shapes
def _special(E, k, n_shared, scaling, fmt=0, bias_hot=None, T=6, H=None, I=None):
    H0, I0 = (256, 128) if fmt == 0 else (512, 256)
    H, I = H or H0, I or I0
    w = synth.Workload("special", T, H, I, I, E, k, n_shared, scaling, fmt, "uniform", 99)
    host = synth.make_layer(w)
    if bias_hot is not None:
        host["bias"] = np.full(E, -1.0, np.float32)
        host["bias"][bias_hot] = 1.0
    case = Case.__new__(Case)
    case.w, case.T, case.desc = w, T, oracle.desc_of(w)
    case.x = synth.make_tokens(w, T)
    case.host = host
    from w4a16_quantized_expert_b200.device import DeviceLayer
    case.dev = DeviceLayer(case.desc, host, max_tokens=T)
    case.x_dev = torch.from_numpy(case.x.copy()).cuda()
    return case


@pytest.mark.parametrize("E,k,n_shared,scaling,fmt,hot", [
    (1, 1, 0, 1.0, 0, None),       # dense SwiGLU special case
    (8, 8, 1, 2.5, 0, None),       # k = E: every expert on every token
    (16, 4, 0, 2.5, 0, [3, 5, 7, 9]),   # every token on the same four experts
    (32, 8, 1, 2.5, 1, None),      # NVFP4 with a small shape
    (5, 2, 1, 1.0, 0, None),       # E not a multiple of 32
])
def test_forward_special_shapes(E, k, n_shared, scaling, fmt, hot):
    case = _special(E, k, n_shared, scaling, fmt, hot)
    y, _ = _forward(case)
    ref = oracle.default().forward(case.desc, case.host, case.x)
    check_y(y_to_f64(y), ref["y"], ref["gap"])


@pytest.mark.parametrize("E,k,n_shared,fmt,T,H,I", [
    (32, 8, 1, 1, 40, None, None),   # NVFP4, several token tiles
    (5, 2, 1, 0, 50, None, None),    # one partial expert tile
    (40, 4, 1, 0, 70, None, None),   # a full and a partial expert tile
    (16, 2, 1, 0, 33, 320, 192),     # H with a partial limb block, ~4 tokens per expert (int8 path)
    (4, 2, 1, 0, 33, 320, 192),      # ~16 tokens per expert, int4 rows not multiples of 128 (f16 path)
    (4, 2, 1, 0, 100, None, None),   # ~50 tokens per expert: 64-token items on tcgen05, ragged
    (8, 2, 1, 0, 200, 512, 256),     # the same with several 64-token items per expert
])
def test_forward_special_batches(E, k, n_shared, fmt, T, H, I):
    case = _special(E, k, n_shared, 2.5, fmt, None, T=T, H=H, I=I)
    y, _ = _forward(case)
    ref = oracle.default().forward(case.desc, case.host, case.x)
    check_y(y_to_f64(y), ref["y"], ref["gap"])


def test_device_wait_timeout_is_reported(tiny):
    moe.moe_debug_wait_timeout(tiny.dev.handle, 1 << 20, 0)
    assert moe.moe_get_device_status(tiny.dev.handle) == moe.MOE_ERR_DEVICE_TIMEOUT
    # the context stays usable
    y, _ = _forward(tiny)
    assert y.shape == (tiny.T, 256)


def test_handles_with_different_expert_counts_coexist(tiny):
    """Kernel launch limits are per function: a later handle with a smaller E must not
    break launches of an earlier handle with a larger one."""
    small = _special(5, 2, 1, 1.0)
    y_small, _ = _forward(small)
    y, _ = _forward(tiny)
    ref = tiny.oracle_forward()
    check_y(y_to_f64(y), ref["y"], ref["gap"])
