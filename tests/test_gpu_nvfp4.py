"""The layer with NVFP4 experts (moe_ffn_forward_nvfp4) against the oracle's
NVFP4 layer, through the C ABI, on the GPU.

The weights are moe_inputs' NVFP4 storage of the seeded fp32 draws (codes
and block scales bit-identical to the oracle's own quantiser).  The GPU's
routing comes from the same router kernel (moe_router_topk on the same
inputs); it is validated against the oracle's logits, and the oracle layer
is rerun on it.  Every output element is compared at the FP8 path's
tolerances (relative L2 5e-3, max-abs 2e-2); rows run in chunks of up to 4,
so the row counts below cover one chunk, several, and a ragged last one.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


def _case(dims, rows, seed, all_experts=False):
    x = mi.make_x(dims, rows, seed=seed, stream=700 + rows)
    rw, g, _ = mi.make_router(dims, seed)
    logits, _, _, _ = oracle.router_topk(dims, x, rw, g)
    experts = None if all_experts else P.needed_experts(logits, dims.top_k)
    layer = mi.make_layer_nvfp4(dims, seed=seed, experts=experts)
    return x, layer, logits


def _dev(layer):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return {"router_w": P.bf16_tensor(layer.router_w), "shared_gate": P.bf16_tensor(layer.shared_gate),
            "w4": t(layer.expert_w4), "sf": t(layer.expert_sf), "gs": t(layer.expert_gs),
            "sw4": t(layer.shared_w4), "ssf": t(layer.shared_sf), "sgs": t(layer.shared_gs)}


def _run(dims, x, layer, residual=None):
    rows = x.shape[0]
    dev = _dev(layer)
    xt = P.bf16_tensor(x)
    ws = moe.alloc_workspace(dims, rows)
    out = torch.full((rows, dims.hidden), float("nan"), dtype=torch.bfloat16, device="cuda")
    res = None if residual is None else P.bf16_tensor(residual)
    moe.ffn_forward_nvfp4(dims, xt, dev["router_w"], dev["w4"], dev["sf"], dev["gs"], dev["sw4"], dev["ssf"],
                          dev["sgs"], dev["shared_gate"], out, ws, residual=res)
    idx = torch.empty(rows, dims.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(rows, dims.top_k, dtype=torch.float32, device="cuda")
    gs = torch.empty(rows, dtype=torch.float32, device="cuda")
    moe.router_topk(dims, xt, dev["router_w"], dev["shared_gate"], idx, w, gs, ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == moe.MOE_OK
    return P.bf16_to_f64(out), idx.cpu().numpy()


def _check(dims, x, layer, logits, got, idx, residual=None):
    case = P.Case(dims, None, x, logits)
    P.check_routing(case, idx)
    ref = oracle.moe_forward_nvfp4(dims, x, layer.router_w, layer.expert_w4, layer.expert_sf, layer.expert_gs,
                                   layer.shared_w4, layer.shared_sf, layer.shared_gs, layer.shared_gate,
                                   residual=residual, forced_idx=idx, want_logits=False)
    err = got - ref.out
    rel = float(np.linalg.norm(err) / np.linalg.norm(ref.out))
    assert np.all(np.isfinite(got))
    assert rel <= P.REL_L2_TOL, f"relative L2 {rel:.3e}"
    assert float(np.max(np.abs(err))) <= P.MAX_ABS_TOL
    return rel


@pytest.mark.parametrize("rows", [1, 4, 9])
def test_nvfp4_tiny(rows):
    d = mi.TINY
    x, layer, logits = _case(d, rows, seed=21, all_experts=True)
    got, idx = _run(d, x, layer)
    _check(d, x, layer, logits, got, idx)


@pytest.mark.parametrize("rows", [1, 3])
def test_nvfp4_qwen36_35b(rows):
    d = mi.QWEN36_35B_A3B
    x, layer, logits = _case(d, rows, seed=22)
    got, idx = _run(d, x, layer)
    _check(d, x, layer, logits, got, idx)


@pytest.mark.parametrize("rows", [1, 2])
def test_nvfp4_qwen35_397b(rows):
    d = mi.QWEN35_397B_A17B
    x, layer, logits = _case(d, rows, seed=23)
    got, idx = _run(d, x, layer)
    _check(d, x, layer, logits, got, idx)


def test_nvfp4_residual_and_batch_invariance():
    """A residual joins before the one rounding; a row's bits do not depend on
    the other rows of the call."""
    d = mi.QWEN36_35B_A3B
    x, layer, logits = _case(d, 5, seed=24)
    res = mi.make_residual(d, 5, seed=24, stream=5)
    got, idx = _run(d, x, layer, residual=res)
    _check(d, x, layer, logits, got, idx, residual=res)
    for t in (0, 4):
        one, _ = _run(d, x[t:t + 1], layer, residual=res[t:t + 1])
        assert np.array_equal(one[0], got[t])


@pytest.mark.parametrize("dims,rows", [
    # I > 1024: 72 scale blocks a down row (the lanes' blocks past 64); H/32 = 12 chunks, fewer than
    # the lanes; Is != I; two chunks of rows
    (mi.LayerDims(hidden=384, n_experts=12, top_k=3, inter=1152, shared_inter=640), 5),
    (mi.LayerDims(hidden=256, n_experts=16, top_k=16, inter=128, shared_inter=128), 2),   # k = E
    (mi.LayerDims(hidden=128, n_experts=1, top_k=1, inter=128, shared_inter=128), 1),     # one expert
    (mi.LayerDims(hidden=8192, n_experts=4, top_k=2, inter=128, shared_inter=256), 3),    # 256 chunks: two load rounds
])
def test_nvfp4_odd_shapes(dims, rows):
    x, layer, logits = _case(dims, rows, seed=25, all_experts=True)
    got, idx = _run(dims, x, layer)
    _check(dims, x, layer, logits, got, idx)


def test_nvfp4_rows_zero_is_noop():
    d = mi.TINY
    layer = mi.make_layer_nvfp4(d, seed=26)
    dev = _dev(layer)
    ws = moe.alloc_workspace(d, 1)
    x = torch.empty(0, d.hidden, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, d.hidden, dtype=torch.bfloat16, device="cuda")
    moe.ffn_forward_nvfp4(d, x, dev["router_w"], dev["w4"], dev["sf"], dev["gs"], dev["sw4"], dev["ssf"],
                          dev["sgs"], dev["shared_gate"], out, ws)
    torch.cuda.synchronize()
