"""moe_route_static (routing with the library's static scratch, no workspace) against
moe_route on the same inputs: identical top-k indices, weights and logits, on two calls
in a row (the second call relies on the first one leaving the tile counters at zero).

The file name sorts last so that the test also runs after every other GPU test of the
session has used the library; it passes alone as well."""
import numpy as np
import pytest
import torch

import synth
import w4a16_quantized_expert_b200 as moe
from gpu_cases import Case

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def _pair(case, T, logits_in=None):
    ws = case.dev.workspace(T)
    x = None if logits_in is not None else case.x_dev[:T]
    ref = case.dev.route(x, T, ws, logits_in=logits_in, want_logits=True)
    got = case.dev.route_static(x, T, logits_in=logits_in, want_logits=True)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in ref], [t.cpu().numpy() for t in got]


def _same(ref, got):
    assert np.array_equal(ref[0], got[0]), "topk_idx differs from moe_route"
    assert np.array_equal(ref[1].view(np.uint32), got[1].view(np.uint32)), "topk_w differs"
    assert np.array_equal(ref[2].view(np.uint32), got[2].view(np.uint32)), "logits differ"


@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode8", 8), ("decode1", 1), ("decode8", 64)])
def test_static_route_matches_workspace_route_twice(name, T):
    case = Case(W[name], T=T, experts="routed") if name != "tiny" else Case(W[name], T=T)
    for _ in range(2):
        ref, got = _pair(case, T)
        _same(ref, got)
    assert moe.moe_get_device_status(case.dev.handle) == moe.MOE_OK


def test_static_route_from_logits_twice():
    case = Case(W["tiny"], T=37)
    g = torch.Generator().manual_seed(7)
    li = (torch.randn((37, case.desc["E"]), generator=g) * 3).float().cuda()
    for _ in range(2):
        ref, got = _pair(case, 37, logits_in=li)
        _same(ref, got)


def test_static_route_rejects_oversize():
    case = Case(W["decode8"], T=8, max_tokens=128, experts="routed")
    x = torch.zeros((128, case.desc["H"]), dtype=torch.float16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        case.dev.route_static(x, 65)            # 65 * 256 > 16384 (token, expert) pairs
    assert ei.value.code == moe.MOE_ERR_WORKSPACE
    # the rejected call launched nothing: the next one still matches
    ref, got = _pair(case, 8)
    _same(ref, got)
