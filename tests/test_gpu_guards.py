"""Guard bands: no kernel writes outside the workspace it was given or outside y, and the
host checks reject a workspace that is too small, misaligned or missing (nothing is
launched then)."""
import numpy as np
import pytest
import torch

import synth
import w4a16_quantized_expert_b200 as moe
from gpu_cases import Case

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS
G = 4096   # guard bytes on each side (a multiple of 256: the workspace stays aligned)


@pytest.mark.parametrize("name,T", [("tiny", 4), ("tiny", 37), ("nvfp4_16", 16)])
def test_workspace_and_output_guard_bands(name, T):
    case = Case(W[name], T=T, max_tokens=64, experts=[0, 1, 2, 3]) if name != "tiny" else \
        Case(W[name], T=T, max_tokens=64)
    H = case.desc["H"]
    n = moe.moe_workspace_size(case.dev.handle, T)
    buf = torch.full((G + n + G,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[G:G + n]
    ws.zero_()                                   # the counter header starts at zero
    yb = torch.full((T + 2, H), 0x5A5A, dtype=torch.int16, device="cuda").view(torch.uint16)
    y = yb[1:T + 1]
    x = case.x_dev[:T]
    for _ in range(2):                           # the second call relies on counters left zero
        case.dev.forward(x, ws, y=y)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(case.dev.handle) == moe.MOE_OK
    b = buf.cpu().numpy()
    assert np.all(b[:G] == 0xA5) and np.all(b[G + n:] == 0xA5), "write outside the workspace"
    yh = yb.view(torch.int16).cpu().numpy()
    assert np.all(yh[0] == 0x5A5A) and np.all(yh[T + 1] == 0x5A5A), "write outside y"
    ref = case.dev.forward(x, case.dev.workspace(T))
    torch.cuda.synchronize()
    assert torch.equal(y, ref), "guarded run differs from a plain run"


def test_bad_workspace_is_rejected_before_launch():
    case = Case(W["tiny"], T=4, max_tokens=8)
    T = 4
    n = moe.moe_workspace_size(case.dev.handle, T)
    big = torch.zeros(n + 512, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(case.x_dev)
    h, x = case.dev.handle, case.x_dev.data_ptr()
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward(h, x, T, y.data_ptr(), big.data_ptr(), n - 256)        # too small
    assert e.value.code == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward(h, x, T, y.data_ptr(), big.data_ptr() + 16, n)        # misaligned
    assert e.value.code == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward(h, x, T, y.data_ptr(), None, n)                       # missing
    assert e.value.code == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoeError) as e:
        moe.moe_forward(h, x, 9, y.data_ptr(), big.data_ptr(), n + 512)       # T > max_tokens
    assert e.value.code == moe.MOE_ERR_INVALID_ARG
    # nothing was launched: a normal call still works and the status is clean
    out = case.dev.forward(case.x_dev, case.dev.workspace(T))
    torch.cuda.synchronize()
    assert out.shape == (T, case.desc["H"])
    assert moe.moe_get_device_status(case.dev.handle) == moe.MOE_OK
