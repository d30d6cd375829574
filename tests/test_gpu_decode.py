"""GPU parity of the decode path against the CPU oracle, through the C ABI.

Covers the tiny workload, the Qwen3.6-35B-A3B-shaped layer at rows 1, 2, 8,
16, 32, 64, and the Qwen3.5-397B-A17B-shaped layer at rows 1 and 32 (all at
full size), plus odd shapes, residual, router bias, repeated calls on one
workspace, batch invariance, rows = 0 and the router-only entry point.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


@pytest.fixture(scope="session")
def layer35():
    return mi.make_layer(mi.QWEN36_35B_A3B, seed=0)


@pytest.fixture(scope="session")
def dev35(layer35):
    return P.device_weights(layer35)


def run_forward(case, dev=None, path=moe.MOE_PATH_DECODE, residual_inplace=False):
    d = case.dims
    dev = dev or P.device_weights(case.layer)
    rows = case.x.shape[0]
    x = P.bf16_tensor(case.x)
    res = P.bf16_tensor(case.residual) if case.residual is not None else None
    out = res if (residual_inplace and res is not None) else torch.empty(rows, d.hidden, dtype=torch.bfloat16,
                                                                          device="cuda")
    idx = torch.empty(rows, d.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(rows, d.top_k, dtype=torch.float32, device="cuda")
    gs = torch.empty(rows, dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(d, rows)
    moe.ffn_forward_path(d, x, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                         dev["shared_scales"], dev["shared_gate"], out, ws, path=path, residual=res,
                         router_bias=dev["router_bias"], topk_idx=idx, topk_w=w, shared_gate_sig=gs)
    torch.cuda.synchronize()
    return P.bf16_to_f64(out), idx.cpu().numpy(), w.cpu().numpy(), gs.cpu().numpy()


def check(case, dev=None, **kw):
    out, idx, w, gs = run_forward(case, dev, **kw)
    _, oidx, ow, ogs = oracle.router_topk(case.dims, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    return P.compare_output(case, out, idx)


def test_tiny():
    d = mi.TINY
    case = P.build_case(d, 4, all_experts=True)
    check(case)


@pytest.mark.parametrize("rows", [1, 2, 8, 16, 32, 64])
def test_qwen36_35b_decode(rows, layer35, dev35):
    case = P.build_case(mi.QWEN36_35B_A3B, rows, layer=layer35)
    rel, mx = check(case, dev35)
    assert rel < 5e-3


@pytest.fixture(scope="session")
def case397():
    d = mi.QWEN35_397B_A17B
    rw, g, _ = mi.make_router(d, 0)
    need = set()
    xs = {r: mi.make_x(d, r, seed=0, stream=r) for r in (1, 32)}
    for r, x in xs.items():
        lg, _, _, _ = oracle.router_topk(d, x, rw, g)
        need |= P.needed_experts(lg, d.top_k)
    layer = mi.make_layer(d, seed=0, experts=need)
    return layer, P.device_weights(layer)


@pytest.mark.parametrize("rows", [1, 32])
def test_qwen35_397b_decode(rows, case397):
    layer, dev = case397
    case = P.build_case(mi.QWEN35_397B_A17B, rows, layer=layer)
    check(case, dev)


@pytest.mark.parametrize("dims,rows", [
    (mi.LayerDims(hidden=384, n_experts=12, top_k=3, inter=256, shared_inter=128), 5),
    (mi.LayerDims(hidden=640, n_experts=40, top_k=7, inter=384, shared_inter=640), 3),
    (mi.LayerDims(hidden=256, n_experts=16, top_k=16, inter=128, shared_inter=128), 2),   # k = E
    (mi.LayerDims(hidden=128, n_experts=1, top_k=1, inter=128, shared_inter=128), 1),     # one expert
    (mi.LayerDims(hidden=8192, n_experts=4, top_k=2, inter=128, shared_inter=256), 3),    # two K segments
    (mi.LayerDims(hidden=256, n_experts=33, top_k=5, inter=1152, shared_inter=128), 9),   # I > 1024
])
def test_odd_shapes(dims, rows):
    case = P.build_case(dims, rows, all_experts=True)
    check(case)


@pytest.mark.parametrize("rows", [1, 2])
def test_max_experts_and_top_k(rows):
    """E = 1024 and k = 32, the most the library takes: the one-warp top-k
    over tagged logits (the chunk candidates would not fit), and at 2 rows
    more routed pairs than lanes (the bitmask list of distinct experts)."""
    d = mi.LayerDims(hidden=256, n_experts=1024, top_k=32, inter=128, shared_inter=128)
    case = P.build_case(d, rows)
    check(case)


@pytest.mark.parametrize("dims,rows", [
    (mi.LayerDims(hidden=1024, n_experts=256, top_k=8, inter=256, shared_inter=256), 1),   # chunk ranks, ranked merge
    (mi.LayerDims(hidden=1024, n_experts=256, top_k=8, inter=256, shared_inter=256), 3),   # experts shared by rows
    (mi.LayerDims(hidden=1024, n_experts=512, top_k=10, inter=256, shared_inter=256), 2),  # merge by rounds
    (mi.LayerDims(hidden=512, n_experts=64, top_k=32, inter=128, shared_inter=128), 1),    # k = 32: a whole chunk
])
def test_exact_logit_ties_take_the_lower_expert_first(dims, rows):
    """Experts 2i and 2i+1 share one router row, so their logits are equal
    bit for bit in any summation order.  Equal logits keep ascending expert
    order: where 2i+1 is chosen, 2i is chosen just before it with the same
    weight; where only one of the pair is chosen, it is 2i."""
    seed = 31
    rw, g, _ = mi.make_router(dims, seed)
    rw[1::2] = rw[0::2]
    x = mi.make_x(dims, rows, seed=seed, stream=rows)
    logits, _, _, _ = oracle.router_topk(dims, x, rw, g)
    layer = mi.make_layer(dims, seed=seed, experts=P.needed_experts(logits, dims.top_k))
    layer.router_w[1::2] = layer.router_w[0::2]
    case = P.build_case(dims, rows, seed=seed, layer=layer)
    out, idx, w, gs = run_forward(case)
    _, _, ow, ogs = oracle.router_topk(dims, case.x, layer.router_w, layer.shared_gate)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)
    for t in range(rows):
        pos = {int(e): i for i, e in enumerate(idx[t])}
        for e, i in pos.items():
            if e % 2 == 1:
                assert pos.get(e - 1) == i - 1, f"row {t}: expert {e} at {i} without {e - 1} just before it"
                assert w[t, i] == w[t, i - 1]


def test_residual_and_router_bias():
    d = mi.LayerDims(hidden=512, n_experts=32, top_k=4, inter=256, shared_inter=256)
    case = P.build_case(d, 6, router_bias=True, all_experts=True, residual=True)
    check(case)


def test_residual_in_place():
    d = mi.TINY
    case = P.build_case(d, 4, all_experts=True, residual=True)
    check(case, residual_inplace=True)


@pytest.mark.parametrize("path", ["decode", "auto"])
def test_rows_64_max_decode_tile_then_rows_1_on_same_workspace(layer35, dev35, path):
    """Counters left by one call must not disturb the next (different rows;
    through AUTO, 64 rows take the prefill path and 1 row the decode path)."""
    d = mi.QWEN36_35B_A3B
    ws = moe.alloc_workspace(d, 64)
    pcode = moe.MOE_PATH_DECODE if path == "decode" else moe.MOE_PATH_AUTO
    outs = []
    for rows in (64, 1, 64):
        case = P.build_case(d, rows, layer=layer35)
        x = P.bf16_tensor(case.x)
        out = torch.empty(rows, d.hidden, dtype=torch.bfloat16, device="cuda")
        moe.ffn_forward_path(d, x, dev35["router_w"], dev35["expert_w8"], dev35["expert_scales"],
                             dev35["shared_w8"], dev35["shared_scales"], dev35["shared_gate"], out, ws, path=pcode)
        torch.cuda.synchronize()
        assert moe.device_status(ws) == moe.MOE_OK
        outs.append(out.clone())
    assert torch.equal(outs[0], outs[2])


def test_batch_invariance_bitwise(layer35, dev35):
    """Row r of an 8-row call equals a 1-row call on row r, bit for bit."""
    d = mi.QWEN36_35B_A3B
    case = P.build_case(d, 8, layer=layer35)
    out8, idx8, w8, _ = run_forward(case, dev35)
    for r in range(8):
        one = P.Case(d, layer35, case.x[r:r + 1].copy(), case.logits[r:r + 1])
        out1, idx1, w1, _ = run_forward(one, dev35)
        assert np.array_equal(out1[0], out8[r])
        assert np.array_equal(idx1[0], idx8[r]) and np.array_equal(w1[0], w8[r])


def test_rows_zero_is_noop():
    d = mi.TINY
    L = mi.make_layer(d, seed=0)
    dev = P.device_weights(L)
    x = torch.empty(0, d.hidden, dtype=torch.bfloat16, device="cuda")
    out = torch.full((1, d.hidden), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = moe.alloc_workspace(d, 1)
    moe.ffn_forward(d, x, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                    dev["shared_scales"], dev["shared_gate"], out, ws)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


@pytest.mark.parametrize("dims,rows", [(mi.TINY, 4), (mi.QWEN36_35B_A3B, 64), (mi.QWEN35_397B_A17B, 32)])
def test_router_topk_entry_point(dims, rows):
    rw, g, _ = mi.make_router(dims, 0)
    x = mi.make_x(dims, rows, seed=0, stream=rows)
    logits, oidx, ow, ogs = oracle.router_topk(dims, x, rw, g)
    idx = torch.empty(rows, dims.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(rows, dims.top_k, dtype=torch.float32, device="cuda")
    gs = torch.empty(rows, dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(dims, rows)
    moe.router_topk(dims, P.bf16_tensor(x), P.bf16_tensor(rw), P.bf16_tensor(g), idx, w, gs, ws)
    torch.cuda.synchronize()
    case = P.Case(dims, None, x, logits)
    P.check_routing(case, idx.cpu().numpy(), w.cpu().numpy(), gs.cpu().numpy(), ow, ogs)


def test_paths_in_turn_on_one_workspace(layer35, dev35):
    """Decode steps, the router-only entry and the grouped path (its router
    kernel below 64 rows) called in turn on one workspace give, bit for bit,
    what each gives on a fresh workspace: the decode step leaves its
    per-expert unit counts set between calls, and the router kernel's
    token-group counts must not start from them."""
    d = mi.QWEN36_35B_A3B
    c1 = P.build_case(d, 1, layer=layer35)
    c8 = P.build_case(d, 8, layer=layer35)
    x1, x8 = P.bf16_tensor(c1.x), P.bf16_tensor(c8.x)

    def decode(ws):
        out = torch.empty(1, d.hidden, dtype=torch.bfloat16, device="cuda")
        moe.ffn_forward_path(d, x1, dev35["router_w"], dev35["expert_w8"], dev35["expert_scales"],
                             dev35["shared_w8"], dev35["shared_scales"], dev35["shared_gate"], out, ws,
                             path=moe.MOE_PATH_DECODE)
        return out

    def route(ws):
        idx = torch.empty(8, d.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(8, d.top_k, dtype=torch.float32, device="cuda")
        gs = torch.empty(8, dtype=torch.float32, device="cuda")
        moe.router_topk(d, x8, dev35["router_w"], dev35["shared_gate"], idx, w, gs, ws)
        return idx, w

    def narrow(ws):
        out = torch.empty(8, d.hidden, dtype=torch.bfloat16, device="cuda")
        moe.ffn_forward_path(d, x8, dev35["router_w"], dev35["expert_w8"], dev35["expert_scales"],
                             dev35["shared_w8"], dev35["shared_scales"], dev35["shared_gate"], out, ws,
                             path=moe.MOE_PATH_PREFILL_NARROW)
        return out

    ref_d, ref_r, ref_n = decode(moe.alloc_workspace(d, 8)), route(moe.alloc_workspace(d, 8)), \
        narrow(moe.alloc_workspace(d, 8))
    ws = moe.alloc_workspace(d, 8)
    for _ in range(3):  # both parities of the decode step's counter sets
        got_d = decode(ws)
        got_r = route(ws)
        got_n = narrow(ws)
        torch.cuda.synchronize()
        assert moe.device_status(ws) == moe.MOE_OK
        assert torch.equal(got_d, ref_d)
        assert torch.equal(got_r[0], ref_r[0]) and torch.equal(got_r[1], ref_r[1])
        assert torch.equal(got_n, ref_n)
