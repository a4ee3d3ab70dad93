"""The C-ABI library: it loads without a GPU, exports every symbol ``include/moe.h``
declares, and its host-side validation rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import w4a16_quantized_expert_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_layer_create", "moe_layer_destroy", "moe_workspace_size", "moe_route",
                     "moe_group", "moe_expert_ffn", "moe_combine", "moe_forward"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_python_binding_has_the_same_names():
    for n in declared_functions():
        assert hasattr(moe, n), n


def test_status_strings_and_version():
    assert moe.status_string(moe.MOE_OK) == "MOE_OK"
    assert moe.status_string(moe.MOE_ERR_DEVICE_TIMEOUT) == "MOE_ERR_DEVICE_TIMEOUT"
    assert moe.status_string(99) == "MOE_ERR_UNKNOWN"
    assert moe.moe_version() >= 100


def _desc(**kw):
    d = dict(hidden=256, inter=128, inter_shared=128, n_experts=16, top_k=2, n_shared=1,
             routed_scaling=2.5, format=0, max_tokens=4)
    d.update(kw)
    return moe.moe_layer_desc(**d)


def _weights(fmt=0, n_shared=1, misalign=None, drop=None):
    w = moe.moe_weights()
    for i, f in enumerate(moe.WEIGHT_FIELDS):
        setattr(w, f, 0x100000 + 0x1000 * i)
    if misalign:
        setattr(w, misalign, getattr(w, misalign) + 4)
    if drop:
        setattr(w, drop, None)
    return w


def _create(desc, w):
    h = ctypes.c_void_p()
    rc = moe.lib().moe_layer_create(ctypes.byref(desc), ctypes.byref(w), ctypes.byref(h))
    return rc, h.value


@pytest.mark.parametrize("bad", [
    dict(hidden=0), dict(hidden=96), dict(hidden=16384 + 64), dict(inter=100),
    dict(n_experts=0), dict(n_experts=1025), dict(top_k=0), dict(top_k=33),
    dict(top_k=17), dict(n_shared=2), dict(inter_shared=50), dict(max_tokens=0),
    dict(max_tokens=70000), dict(format=7), dict(routed_scaling=float("nan")),
    dict(format=1, hidden=320), dict(format=1, inter=128), dict(top_p=-0.1), dict(top_p=float("nan")),
])
def test_create_rejects_bad_shapes(bad):
    rc, h = _create(_desc(**bad), _weights())
    assert rc == moe.MOE_ERR_INVALID_ARG and h is None


@pytest.mark.parametrize("field", ["router_w", "gate", "down_scale", "shared_up"])
def test_create_rejects_missing_or_misaligned_pointers(field):
    rc, _ = _create(_desc(), _weights(drop=field))
    assert rc == moe.MOE_ERR_INVALID_ARG
    rc, _ = _create(_desc(), _weights(misalign=field))
    assert rc == moe.MOE_ERR_INVALID_ARG


def test_unused_pointers_may_be_null():
    # int4 without a shared expert ignores the NVFP4 and shared fields; with no GPU the
    # call gets past validation and fails at the first CUDA call instead
    w = _weights()
    for f in moe.WEIGHT_FIELDS:
        if "bscale" in f or "tscale" in f or f.startswith("shared"):
            setattr(w, f, None)
    rc, h = _create(_desc(n_shared=0), w)
    try:
        import torch
        gpu = torch.cuda.is_available()
    except Exception:
        gpu = False
    if not gpu:
        assert rc == moe.MOE_ERR_CUDA and h is None


D, F, TM = moe.MOE_PLAN_DECODE, moe.MOE_PLAN_F16_BATCH, moe.MOE_PLAN_TENSOR_MEMORY
BIG = dict(hidden=6144, inter=2048, inter_shared=2048, n_experts=256, top_k=8, max_tokens=4096)


@pytest.mark.parametrize("fmt,T,shape,plan", [
    (0, 1, BIG, (D, 8, 1)), (0, 16, BIG, (D, 8, 1)),
    (0, 17, BIG, (D, 8, 1)), (0, 128, BIG, (D, 8, 1)), (0, 192, BIG, (D, 8, 1)),  # <= 6 tokens per expert
    (0, 193, BIG, (TM, 32, 1)), (0, 512, BIG, (TM, 32, 1)),                       # tensor-memory kernel
    (0, 1152, BIG, (TM, 32, 1)), (0, 1153, BIG, (TM, 64, 1)), (0, 2048, BIG, (TM, 64, 1)),  # > 36 per expert
    (1, 1, BIG, (D, 8, 0)), (1, 16, BIG, (D, 8, 0)), (1, 17, BIG, (F, 32, 0)),     # NVFP4
    (2, 1, BIG, (D, 8, 1)), (2, 2048, BIG, (D, 8, 1)), (3, 512, BIG, (D, 8, 1)),   # int8, int2
    (0, 48, dict(hidden=256, inter=128, inter_shared=128, n_experts=16, top_k=2, max_tokens=64), (D, 8, 1)),
    (0, 49, dict(hidden=256, inter=128, inter_shared=128, n_experts=16, top_k=2, max_tokens=64), (TM, 32, 1)),
    (0, 33, dict(hidden=320, inter=192, inter_shared=192, n_experts=4, top_k=2, max_tokens=64), (F, 32, 0)),
    (0, 33, dict(hidden=320, inter=192, inter_shared=192, n_experts=16, top_k=2, max_tokens=64), (D, 8, 1)),
])
def test_plan_of_a_batch(fmt, T, shape, plan):
    """Which expert kernels a batch runs (a host function: no GPU).  The boundaries are the
    measured crossovers: at most 6 tokens per routed expert on the 8-token items, 64-token
    items past 36 tokens per expert, the decode variants for every format up to 16 tokens."""
    assert moe.moe_plan(_desc(format=fmt, **shape), T) == plan


def test_plan_rejects_bad_arguments():
    with pytest.raises(moe.MoeError):
        moe.moe_plan(_desc(), 0)
    with pytest.raises(moe.MoeError):
        moe.moe_plan(_desc(), 5)            # max_tokens = 4
    with pytest.raises(moe.MoeError):
        moe.moe_plan(_desc(hidden=100), 1)  # not a multiple of 64


def test_null_handle_and_out_of_range_T():
    L = moe.lib()
    assert L.moe_workspace_size(None, 1) == 0
    assert L.moe_forward(None, None, 1, None, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(None, None, 1, None, None, None, None, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_destroy(None) == moe.MOE_OK
    assert L.moe_workspace_routing(None, 1, None) == moe.MOE_ERR_INVALID_ARG
    st = ctypes.c_int(0)
    assert L.moe_get_device_status(None, ctypes.byref(st)) == moe.MOE_ERR_INVALID_ARG


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of moe_layer_desc and moe_weights have the C header's sizes and
    field offsets (compiled with the host C compiler)."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no host C compiler")
    fields = [f for f, _ in moe.moe_layer_desc._fields_]
    wfields = [f for f, _ in moe.moe_weights._fields_]
    rfields = [f for f, _ in moe.moe_ws_routing._fields_]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe.h"', "int main(void) {",
             '  printf("%zu %zu %zu\\n", sizeof(moe_layer_desc), sizeof(moe_weights), sizeof(moe_ws_routing));']
    lines += [f'  printf("%zu\\n", offsetof(moe_layer_desc, {f}));' for f in fields]
    lines += [f'  printf("%zu\\n", offsetof(moe_weights, {f}));' for f in wfields]
    lines += [f'  printf("%zu\\n", offsetof(moe_ws_routing, {f}));' for f in rfields]
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split()
    sizes, offs = [int(v) for v in out[:3]], [int(v) for v in out[3:]]
    assert sizes == [ctypes.sizeof(moe.moe_layer_desc), ctypes.sizeof(moe.moe_weights),
                     ctypes.sizeof(moe.moe_ws_routing)]
    py = [getattr(moe.moe_layer_desc, f).offset for f in fields] + \
         [getattr(moe.moe_weights, f).offset for f in wfields] + \
         [getattr(moe.moe_ws_routing, f).offset for f in rfields]
    assert offs == py


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle and has no CPU compute path."""
    pkg = os.path.join(ROOT, "w4a16_quantized_expert_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "liboracle" not in txt, f
