"""Shared helpers of the GPU parity tests: seeded workloads on the device, the oracle on
the same inputs, and the comparison rules.

Comparison rules (the layer's stated tolerances):
* expert indices, grouping arrays: bit-exact when the router is fed the oracle's fp32
  logits;
* combine weights: relative error <= 1e-6;
* outputs: max |gpu - oracle| <= 4e-3 * max |oracle| over tokens whose k-th vs (k+1)-th
  selection-score gap is >= 1e-4 (closer tokens may legitimately route differently
  because the GPU accumulates the router logits in fp32; they are excluded and counted).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from w4a16_quantized_expert_b200.device import DeviceLayer

TOL = 4e-3
GAP_MIN = 1e-4
W_RTOL = 1e-6


def desc_of(w):
    d = oracle.desc_of(w)
    d["scaling"] = float(np.float32(w.scaling))   # the ABI carries an fp32 scaling factor
    d["top_p"] = float(np.float32(d.get("top_p", 0.0)))   # and an fp32 top-p
    return d


class Case:
    """A workload with its host layer, device layer and tokens."""

    def __init__(self, w, T=None, max_tokens=None, experts="all", batch=0):
        self.w = w
        self.T = w.T if T is None else T
        self.desc = desc_of(w)
        self.x = synth.make_tokens(w, self.T, batch=batch)
        self.router = synth.make_router(w)
        if experts == "routed":
            # generate only the experts the oracle routes to (plus neighbours of near ties)
            logits = oracle.default().router_logits(self.x, self.router[0])
            idx, _, sel, gap = oracle.default().route(logits, self.router[1], w.k, self.desc["scaling"])
            order = np.argsort(-sel, axis=1, kind="stable")[:, : w.k + 2]
            experts = np.unique(order)
        elif isinstance(experts, str):   # "all"
            experts = None
        self.host = {"Wr": self.router[0], "bias": self.router[1]}
        self.host.update(synth.make_experts(w, experts))
        self.dev = DeviceLayer(self.desc, self.host, max_tokens=max_tokens or max(self.T, 1))
        self.x_dev = torch.from_numpy(self.x.copy()).cuda()

    def oracle_forward(self, logits_in=None, tokens=None, want_h=False):
        o = oracle.default()
        if tokens is None:
            return o.forward(self.desc, self.host, self.x, logits_in=logits_in, want_h=want_h)
        outs = [o.forward_token(self.desc, self.host, self.x[t]) for t in tokens]
        return {"y": np.stack([r["y"] for r in outs]), "gap": np.array([r["gap"] for r in outs]),
                "topk_idx": np.stack([r["topk_idx"] for r in outs]),
                "topk_w": np.stack([r["topk_w"] for r in outs])}


def y_to_f64(y: torch.Tensor) -> np.ndarray:
    return y.cpu().numpy().view(np.float16).astype(np.float64)


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, gap: np.ndarray, tol: float = TOL):
    """Returns (excluded token count, relative error) and asserts the tolerance."""
    keep = gap >= GAP_MIN
    assert np.isfinite(y_gpu[keep]).all(), "non-finite outputs"
    scale = np.abs(y_ref[keep]).max() if keep.any() else 1.0
    err = np.abs(y_gpu[keep] - y_ref[keep]).max() / scale if keep.any() else 0.0
    assert err <= tol, f"max|gpu-oracle| = {err:.3g} * max|oracle| > {tol}"
    return int((~keep).sum()), float(err)


def check_routing(idx_gpu, w_gpu, idx_ref, w_ref):
    """Top-k (and top-p) routing: indices bit-exact (-1 = dropped by top-p), weights
    within W_RTOL relative where kept and exactly zero where dropped."""
    assert np.array_equal(idx_gpu, idx_ref), "topk_idx differs"
    kept = idx_ref >= 0
    assert np.all(w_gpu[~kept] == 0)
    rel = np.abs(w_gpu[kept].astype(np.float64) - w_ref[kept]) / np.abs(w_ref[kept])
    assert rel.max() <= W_RTOL, f"topk_w relative error {rel.max():.3g}"


def check_weights(w_gpu: np.ndarray, w_ref: np.ndarray):
    rel = np.abs(w_gpu.astype(np.float64) - w_ref) / np.abs(w_ref)
    assert rel.max() <= W_RTOL, f"topk_w relative error {rel.max():.3g}"
