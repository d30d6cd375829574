"""Helpers shared by the GPU parity tests: build seeded cases, run the CUDA
path through the C ABI, and compare with the CPU oracle.

Parity rules (the layer's stated bar):
  - top-k indices equal the oracle's as a set on every row whose oracle logit
    gap (k-th largest minus (k+1)-th largest) exceeds 1e-4;
  - on rows with a smaller gap several selections are correct: the GPU's
    choice must lie within 1e-4 of the k-th logit, and the output is then
    compared with the oracle rerun on the GPU's selection;
  - the output (bf16) against the oracle's double result: relative L2
    <= 5e-3 and max-abs <= 2e-2 over the whole [rows, H] tensor.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import moe_inputs as mi
import oracle

REL_L2_TOL = 5e-3
MAX_ABS_TOL = 2e-2
GAP = 1e-4
W_ATOL = 2e-5      # routing weights: fp32 softmax of fp32 logits
GS_ATOL = 1e-5     # shared-gate sigmoid


@dataclass
class Case:
    dims: mi.LayerDims
    layer: mi.Layer
    x: np.ndarray                 # uint16 [rows, H]
    logits: np.ndarray            # oracle float64 [rows, E]
    residual: np.ndarray | None = None


def needed_experts(logits: np.ndarray, k: int, margin: float = 1e-3) -> set:
    srt = -np.sort(-logits, axis=1)
    kth = srt[:, k - 1:k]
    rows, cols = np.nonzero(logits >= kth - margin)
    return set(cols.tolist())


def build_case(dims: mi.LayerDims, rows: int, seed: int = 0, router_bias: bool = False,
               stream: int | None = None, all_experts: bool = False, layer: mi.Layer | None = None,
               residual: bool = False) -> Case:
    x = mi.make_x(dims, rows, seed=seed, stream=rows if stream is None else stream)
    if layer is None:
        rw, g, b = mi.make_router(dims, seed, router_bias)
        logits, _, _, _ = oracle.router_topk(dims, x, rw, g, router_bias=b)
        experts = None if all_experts else needed_experts(logits, dims.top_k)
        layer = mi.make_layer(dims, seed=seed, router_bias=router_bias, experts=experts)
    logits, _, _, _ = oracle.router_topk(dims, x, layer.router_w, layer.shared_gate,
                                         router_bias=layer.router_bias)
    missing = needed_experts(logits, dims.top_k) - set(layer.generated)
    assert not missing, f"layer lacks weights of experts {sorted(missing)[:8]}"
    res = mi.make_residual(dims, rows, seed=seed, stream=rows) if residual else None
    return Case(dims, layer, x, logits, res)


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def device_weights(layer: mi.Layer, device="cuda") -> dict:
    return {
        "router_w": bf16_tensor(layer.router_w, device),
        "shared_gate": bf16_tensor(layer.shared_gate, device),
        "expert_w8": torch.from_numpy(layer.expert_w8).to(device),
        "expert_scales": torch.from_numpy(layer.expert_scales).to(device),
        "shared_w8": torch.from_numpy(layer.shared_w8).to(device),
        "shared_scales": torch.from_numpy(layer.shared_scales).to(device),
        "router_bias": None if layer.router_bias is None else torch.from_numpy(layer.router_bias).to(device),
    }


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_routing(case: Case, gpu_idx: np.ndarray, gpu_w: np.ndarray | None = None,
                  gpu_gs: np.ndarray | None = None, oracle_w=None, oracle_gs=None):
    """Assert the GPU routing is valid; returns the number of near-tie rows."""
    k = case.dims.top_k
    L = case.logits
    E = L.shape[1]
    srt = -np.sort(-L, axis=1)
    gap = srt[:, k - 1] - srt[:, k] if k < E else np.full(L.shape[0], np.inf)
    ref_idx = np.argsort(-L, axis=1, kind="stable")[:, :k]
    near = 0
    for t in range(L.shape[0]):
        g = gpu_idx[t]
        assert len(set(g.tolist())) == k, f"row {t}: repeated experts {g}"
        assert np.all((g >= 0) & (g < E)), f"row {t}: expert id out of range {g}"
        if gap[t] > GAP:
            assert set(g.tolist()) == set(ref_idx[t].tolist()), f"row {t}: {sorted(g)} != {sorted(ref_idx[t])}"
        else:
            near += 1
            assert np.all(L[t, g] >= srt[t, k - 1] - GAP), f"row {t}: choice outside the tie band"
        # descending order, up to near-ties inside the top-k
        lv = L[t, g]
        assert np.all(np.diff(lv) <= GAP), f"row {t}: not in descending logit order"
    if gpu_w is not None and oracle_w is not None:
        # match by expert id
        for t in range(L.shape[0]):
            ref = dict(zip(ref_idx[t].tolist(), oracle_w[t].tolist()))
            if gap[t] > GAP:
                for e, wv in zip(gpu_idx[t].tolist(), gpu_w[t].tolist()):
                    assert abs(wv - ref[e]) <= W_ATOL, f"row {t} expert {e}: w {wv} vs {ref[e]}"
        assert np.allclose(gpu_w.sum(axis=1), 1.0, atol=1e-5)
    if gpu_gs is not None and oracle_gs is not None:
        assert np.max(np.abs(gpu_gs - oracle_gs)) <= GS_ATOL
    return near


def compare_output(case: Case, gpu_out: np.ndarray, gpu_idx: np.ndarray):
    """Oracle rerun on the GPU's (validated) routing; assert the tolerances.
    Returns (rel_l2, max_abs)."""
    L = case.layer
    ref = oracle.moe_forward(case.dims, case.x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                             L.shared_scales, L.shared_gate, residual=case.residual,
                             router_bias=L.router_bias, forced_idx=gpu_idx, want_logits=False)
    err = gpu_out - ref.out
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref.out), 1e-300))
    mx = float(np.max(np.abs(err))) if err.size else 0.0
    assert np.all(np.isfinite(gpu_out)), "non-finite output"
    assert rel <= REL_L2_TOL, f"relative L2 {rel:.3e} > {REL_L2_TOL}"
    assert mx <= MAX_ABS_TOL, f"max-abs {mx:.3e} > {MAX_ABS_TOL}"
    return rel, mx
