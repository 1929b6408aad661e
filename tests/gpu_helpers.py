"""Shared helpers of the GPU parity tests: device copies of the seeded inputs,
numpy views for the oracle, and the tolerances (stated once, here)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances. bf16 layer output: max|err| <= 2e-2 * max|ref|. fp32 router
# probabilities and renormalised weights: <= 1e-5 relative. aux loss: <= 1e-4
# relative. fp32 layers (CUDA-core FFMA, fp32 accumulation over K <= 4096
# terms): max|err| <= 1e-4 * max|ref|.
TOL_BF16_OUT = 2e-2
TOL_F32_OUT = 1e-4
TOL_PROB_REL = 1e-5
TOL_AUX_REL = 1e-4


def np32(t: torch.Tensor) -> np.ndarray:
    """float32 numpy copy (exact for bf16 and fp32 tensors)."""
    return t.detach().to("cpu", torch.float32).numpy()


def npi(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


class ExpertWeights:
    """[E, r, c] torch weights seen by the oracle one expert at a time."""

    def __init__(self, w: torch.Tensor):
        self.w = w

    def __getitem__(self, e):
        return self.w[e].to(torch.float32).numpy()

    def __len__(self):
        return self.w.shape[0]


def max_err_ratio(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    m = np.max(np.abs(ref)) if ref.size else 0.0
    if m == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref)) / m)


def rel_err(got, ref, floor=0.0) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = np.maximum(np.abs(ref), floor)
    den = np.where(den == 0, 1.0, den)
    return float(np.max(np.abs(got - ref) / den))


def device_inputs(inp, dev="cuda"):
    d = {"x": inp.x.to(dev), "wg": inp.wg.to(dev), "w1": inp.w1.to(dev), "w2": inp.w2.to(dev),
         "w3": None if inp.w3 is None else inp.w3.to(dev),
         "bias": None if inp.bias is None else inp.bias.to(dev)}
    return d


def new_ws(nbytes: int, dev="cuda") -> torch.Tensor:
    from mixture_experts_routing_route_b200 import _abi
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
    _abi.moe_workspace_init(ws)
    return ws


def check_topk_end_to_end(g_idx, route_ref, eps=1e-3):
    """End-to-end top-k check against the oracle's own routing.

    On tokens the oracle does not flag as near-ties (k-th and (k+1)-th logits
    at least eps apart) the selected SET must be the oracle's. Inside the set
    the order may differ only where two selected logits are closer than eps
    (another float summation order can swap them); the GPU's order must be
    non-increasing in the oracle's logits up to eps. The exact order is
    checked separately, stage-chained on the GPU's own logits."""
    g = np.asarray(g_idx, dtype=np.int64)
    ref = np.asarray(route_ref["topk_idx"], dtype=np.int64)
    ok = ~np.asarray(route_ref["near_tie"])
    assert np.array_equal(np.sort(g[ok], axis=1), np.sort(ref[ok], axis=1)), "top-k set differs"
    lg = np.take_along_axis(np.asarray(route_ref["logits"], np.float64), g, axis=1)
    assert np.all(lg[:, :-1] >= lg[:, 1:] - eps), "top-k order not descending"
    return int(np.sum(np.any(g[ok] != ref[ok], axis=1)))
