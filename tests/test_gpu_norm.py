"""GPU parity of the layer behind its RMSNorm (moe_ffn_forward_norm) against
the oracle's RMSNorm followed by the layer with the residual join, through
the C ABI.

On the decode path the norm runs inside the decode-step kernel; on the
grouped-GEMM paths a norm kernel runs first.  Both compute the mean square
and the scaling in double and round x once to bf16, as the oracle does, so
the routing is checked against the oracle's logits on the oracle's x.  Also:
the update in place of the residual stream, and a chain of layers where each
layer's output is the next one's input.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")

EPS = 1e-6


def norm_weight(d, seed=0):
    g = torch.Generator().manual_seed(1000 + seed)
    w = 1.0 + 0.1 * torch.randn(d.hidden, generator=g)
    return w.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def residual_rows(d, rows, seed=0):
    return mi.make_residual(d, rows, seed=seed, stream=500 + rows)


def check_norm(d, layer, dev, resid, nw, path, inplace=False):
    rows = resid.shape[0]
    r = P.bf16_tensor(resid)
    out = r if inplace else torch.empty(rows, d.hidden, dtype=torch.bfloat16, device="cuda")
    ws = moe.alloc_workspace(d, rows)
    moe.ffn_forward_norm(d, r, P.bf16_tensor(nw), EPS, dev["router_w"], dev["expert_w8"], dev["expert_scales"],
                         dev["shared_w8"], dev["shared_scales"], dev["shared_gate"], out, ws,
                         router_bias=dev["router_bias"], path=path)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == moe.MOE_OK
    _, xb = oracle.rmsnorm(resid, nw, EPS)
    logits, oidx, ow, ogs = oracle.router_topk(d, xb, layer.router_w, layer.shared_gate,
                                               router_bias=layer.router_bias)
    case = P.Case(d, layer, xb, logits, residual=resid)
    # the output is checked against the oracle rerun on the routing the GPU took
    # (validated against the oracle's logits by check_routing)
    gout = P.bf16_to_f64(out)
    gidx = _gpu_routing(d, dev, xb, layer)
    P.check_routing(case, gidx)
    return P.compare_output(case, gout, gidx)


def _gpu_routing(d, dev, xb, layer):
    """The GPU router on the oracle's x (the same bf16 values the kernels use)."""
    rows = xb.shape[0]
    idx = torch.empty(rows, d.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(rows, d.top_k, dtype=torch.float32, device="cuda")
    gs = torch.empty(rows, dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(d, rows)
    moe.router_topk(d, P.bf16_tensor(xb), dev["router_w"], dev["shared_gate"], idx, w, gs, ws,
                    router_bias=dev["router_bias"])
    torch.cuda.synchronize()
    return idx.cpu().numpy()


@pytest.mark.parametrize("path", [moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL_NARROW, moe.MOE_PATH_PREFILL])
@pytest.mark.parametrize("rows", [1, 3, 6])
def test_norm_tiny_every_path(path, rows):
    d = mi.TINY
    layer = mi.make_layer(d, seed=2)
    dev = P.device_weights(layer)
    check_norm(d, layer, dev, residual_rows(d, rows, 2), norm_weight(d, 2), path)


@pytest.mark.parametrize("rows", [1, 2, 4])
def test_norm_35b_decode(rows):
    d = mi.QWEN36_35B_A3B
    resid = residual_rows(d, rows)
    nw = norm_weight(d)
    rw, g, _ = mi.make_router(d, 0)
    _, xb = oracle.rmsnorm(resid, nw, EPS)
    lg, _, _, _ = oracle.router_topk(d, xb, rw, g)
    layer = mi.make_layer(d, seed=0, experts=P.needed_experts(lg, d.top_k))
    dev = P.device_weights(layer)
    check_norm(d, layer, dev, resid, nw, moe.MOE_PATH_DECODE)


def test_norm_in_place_and_bias():
    d = mi.LayerDims(hidden=512, n_experts=32, top_k=4, inter=256, shared_inter=256)
    layer = mi.make_layer(d, seed=4, router_bias=True)
    dev = P.device_weights(layer)
    for path in (moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL_NARROW):
        check_norm(d, layer, dev, residual_rows(d, 3, 4), norm_weight(d, 4), path, inplace=True)


def test_norm_chain_of_layers():
    """Three layers, each updating the residual stream in place: r <- r +
    layer_l(rmsnorm(r) * w_l); compared with the oracle applying the same
    three steps to its own (rounded) outputs."""
    d = mi.TINY
    rows = 2
    layers = [mi.make_layer(d, seed=10 + l) for l in range(3)]
    devs = [P.device_weights(L) for L in layers]
    nws = [norm_weight(d, 10 + l) for l in range(3)]
    r0 = residual_rows(d, rows, 9)
    r = P.bf16_tensor(r0)
    ws = moe.alloc_workspace(d, rows)
    for L, dev, nw in zip(layers, devs, nws):
        moe.ffn_forward_norm(d, r, P.bf16_tensor(nw), EPS, dev["router_w"], dev["expert_w8"], dev["expert_scales"],
                             dev["shared_w8"], dev["shared_scales"], dev["shared_gate"], r, ws)
    torch.cuda.synchronize()
    got = P.bf16_to_f64(r)
    ref = r0
    for L, nw in zip(layers, nws):
        res = oracle.moe_forward_norm(d, ref, nw, EPS, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                                      L.shared_scales, L.shared_gate)
        ref = oracle.round_to_bf16(res.out)
    refd = oracle.bf16_bits_to_f64(ref)
    rel = np.linalg.norm(got - refd) / np.linalg.norm(refd)
    assert rel <= P.REL_L2_TOL and np.max(np.abs(got - refd)) <= 3 * P.MAX_ABS_TOL
