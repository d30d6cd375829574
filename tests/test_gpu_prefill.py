"""GPU parity of the prefill path (token permute -> tcgen05 FP8 grouped GEMMs
-> unpermute), with 128-row token tiles and with the narrow tiling (128
weight rows x up to 32 token rows), against the CPU oracle, through the C ABI.

Small shapes are checked on every row; the 4096-row Qwen3.6-35B-A3B-shaped
prefill (router bias for uneven expert loads) is checked on its routing for
every row and on the output of sampled rows, which the oracle computes one
by one (rows are independent in the layer).
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


def run(case, path, dev=None):
    d = case.dims
    dev = dev or P.device_weights(case.layer)
    rows = case.x.shape[0]
    out = torch.empty(rows, d.hidden, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(rows, d.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(rows, d.top_k, dtype=torch.float32, device="cuda")
    gs = torch.empty(rows, dtype=torch.float32, device="cuda")
    ws = moe.alloc_workspace(d, rows)
    res = P.bf16_tensor(case.residual) if case.residual is not None else None
    moe.ffn_forward_path(d, P.bf16_tensor(case.x), dev["router_w"], dev["expert_w8"], dev["expert_scales"],
                         dev["shared_w8"], dev["shared_scales"], dev["shared_gate"], out, ws, path=path,
                         residual=res, router_bias=dev["router_bias"], topk_idx=idx, topk_w=w, shared_gate_sig=gs)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == moe.MOE_OK
    return P.bf16_to_f64(out), idx.cpu().numpy(), w.cpu().numpy(), gs.cpu().numpy()


@pytest.mark.parametrize("dims,rows,bias", [
    (mi.TINY, 4, False),
    (mi.TINY, 100, True),
    (mi.LayerDims(hidden=512, n_experts=32, top_k=4, inter=256, shared_inter=256), 300, True),
    (mi.LayerDims(hidden=256, n_experts=16, top_k=2, inter=128, shared_inter=256), 130, False),   # I != Is
    (mi.LayerDims(hidden=768, n_experts=12, top_k=3, inter=384, shared_inter=128), 200, True),
])
def test_prefill_small_shapes(dims, rows, bias):
    case = P.build_case(dims, rows, router_bias=bias, all_experts=True, residual=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL)
    _, oidx, ow, ogs = oracle.router_topk(dims, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


@pytest.mark.parametrize("dims,rows", [
    (mi.LayerDims(hidden=1024, n_experts=256, top_k=8, inter=256, shared_inter=256), 130),   # top-8 kept per row
    (mi.LayerDims(hidden=512, n_experts=128, top_k=10, inter=128, shared_inter=128), 200),   # top-16 kept
    (mi.LayerDims(hidden=512, n_experts=64, top_k=32, inter=128, shared_inter=128), 129),    # top-32 kept
])
def test_exact_logit_ties_take_the_lower_expert_first(dims, rows):
    """The tensor-core router of the token-tile paths: experts 2i and 2i+1
    share one router row, so their logits are equal bit for bit.  Equal
    logits keep ascending expert order even when a larger logit is inserted
    above them later: where 2i+1 is chosen, 2i is chosen just before it with
    the same weight."""
    seed = 32
    rw, g, _ = mi.make_router(dims, seed)
    rw[1::2] = rw[0::2]
    x = mi.make_x(dims, rows, seed=seed, stream=rows)
    logits, _, _, _ = oracle.router_topk(dims, x, rw, g)
    layer = mi.make_layer(dims, seed=seed, experts=P.needed_experts(logits, dims.top_k))
    layer.router_w[1::2] = layer.router_w[0::2]
    case = P.build_case(dims, rows, seed=seed, layer=layer)
    for path in (moe.MOE_PATH_PREFILL, moe.MOE_PATH_PREFILL_NARROW):
        out, idx, w, gs = run(case, path)
        _, _, ow, ogs = oracle.router_topk(dims, case.x, layer.router_w, layer.shared_gate)
        P.check_routing(case, idx, w, gs, ow, ogs)
        P.compare_output(case, out, idx)
        for t in range(rows):
            pos = {int(e): i for i, e in enumerate(idx[t])}
            for e, i in pos.items():
                if e % 2 == 1:
                    assert pos.get(e - 1) == i - 1, f"row {t}: expert {e} at {i} without {e - 1} just before it"
                    assert w[t, i] == w[t, i - 1]


def test_auto_path_switch():
    d = mi.TINY
    assert moe.auto_path(d, moe.MOE_AUTO_DECODE_MAX_ROWS) == moe.MOE_PATH_DECODE
    assert moe.auto_path(d, moe.MOE_AUTO_DECODE_MAX_ROWS + 1) == moe.MOE_PATH_PREFILL_NARROW
    big = moe.MOE_AUTO_NARROW_MAX_PAIRS * d.n_experts // d.top_k + 1
    assert moe.auto_path(d, big) == moe.MOE_PATH_PREFILL
    for rows in (moe.MOE_AUTO_DECODE_MAX_ROWS + 1, big):
        case = P.build_case(d, rows, all_experts=True)
        out, idx, _, _ = run(case, moe.MOE_PATH_AUTO)
        P.compare_output(case, out, idx)


@pytest.mark.parametrize("rows", [16, 32, 64])
def test_qwen36_35b_auto_at_multi_row_decode_counts(rows):
    # every row against the oracle, on the path AUTO takes
    d = mi.QWEN36_35B_A3B
    case = P.build_case(d, rows)
    out, idx, w, gs = run(case, moe.MOE_PATH_AUTO)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


def test_qwen36_35b_prefill_4096_rows_every_row():
    """The 4096-token prefill workload (per-expert router bias: uneven loads,
    the busiest expert over twenty 128-row tiles, every expert's last tile
    ragged), every output element of every row against the oracle."""
    d = mi.QWEN36_35B_A3B
    rows = 4096
    case = P.build_case(d, rows, router_bias=True, all_experts=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    counts = np.bincount(idx.ravel(), minlength=d.n_experts)
    assert counts.max() > 16 * 128 and counts.max() > 4 * counts.mean()
    assert np.count_nonzero(counts % 128) > 100          # ragged last tiles
    P.compare_output(case, out, idx)


@pytest.mark.parametrize("rows", [128, 512, 1024])
def test_qwen36_35b_auto_every_row(rows):
    """The 35B layer at 128, 512 and 1024 rows through AUTO (the narrow
    grouped GEMMs there), every row against the oracle."""
    d = mi.QWEN36_35B_A3B
    assert moe.auto_path(d, rows) == moe.MOE_PATH_PREFILL_NARROW
    case = P.build_case(d, rows, all_experts=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_AUTO)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


def test_prefill_router_more_than_256_experts():
    # the router takes the experts in passes of 256 accumulator columns
    d = mi.LayerDims(hidden=256, n_experts=300, top_k=5, inter=128, shared_inter=128)
    case = P.build_case(d, 130, router_bias=True, residual=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


def test_qwen35_397b_prefill_every_row():
    # 512 experts (two router passes), top-10, I = Is = 1024, uneven loads
    d = mi.QWEN35_397B_A17B
    rows = 96
    case = P.build_case(d, rows, router_bias=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


@pytest.mark.parametrize("dims,rows", [
    (mi.LayerDims(hidden=384, n_experts=12, top_k=3, inter=256, shared_inter=128), 150),
    (mi.LayerDims(hidden=640, n_experts=20, top_k=4, inter=128, shared_inter=256), 100),
])
def test_prefill_hidden_odd_multiple_of_128(dims, rows):
    # H/128 odd: the down GEMM's last 256-column tile is half empty
    case = P.build_case(dims, rows, router_bias=True, all_experts=True, residual=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL)
    _, oidx, ow, ogs = oracle.router_topk(dims, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


# ---------------------------------------------------------------- narrow grouped GEMMs
# Weight rows as the MMA's M (128) and up to 32 rows of one group as its N.

@pytest.mark.parametrize("dims,rows,bias", [
    (mi.TINY, 4, False),
    (mi.TINY, 300, True),     # several 32-row tiles per group, uneven loads
    (mi.LayerDims(hidden=512, n_experts=32, top_k=4, inter=256, shared_inter=256), 70, True),
    (mi.LayerDims(hidden=256, n_experts=16, top_k=2, inter=128, shared_inter=256), 45, False),   # I != Is
    (mi.LayerDims(hidden=384, n_experts=12, top_k=3, inter=256, shared_inter=128), 33, True),    # H/128 odd
    (mi.LayerDims(hidden=640, n_experts=20, top_k=4, inter=384, shared_inter=128), 17, False),
])
def test_narrow_small_shapes(dims, rows, bias):
    case = P.build_case(dims, rows, router_bias=bias, all_experts=True, residual=True)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL_NARROW)
    _, oidx, ow, ogs = oracle.router_topk(dims, case.x, case.layer.router_w, case.layer.shared_gate,
                                          router_bias=case.layer.router_bias)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


@pytest.mark.parametrize("rows", [1, 2, 8, 16, 32, 64])
def test_qwen36_35b_narrow(rows):
    d = mi.QWEN36_35B_A3B
    case = P.build_case(d, rows)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL_NARROW)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


def test_qwen35_397b_narrow_rows_32():
    d = mi.QWEN35_397B_A17B
    case = P.build_case(d, 32)
    out, idx, w, gs = run(case, moe.MOE_PATH_PREFILL_NARROW)
    _, oidx, ow, ogs = oracle.router_topk(d, case.x, case.layer.router_w, case.layer.shared_gate)
    P.check_routing(case, idx, w, gs, ow, ogs)
    P.compare_output(case, out, idx)


def test_narrow_matches_wide_tiles_on_the_same_routing():
    # both tilings compute each (row, column) with the same per-K-block
    # promotion; only the tensor cores' summation inside a K block may differ
    d = mi.LayerDims(hidden=512, n_experts=32, top_k=4, inter=256, shared_inter=256)
    case = P.build_case(d, 150, router_bias=True, all_experts=True)
    dev = P.device_weights(case.layer)
    a, ia, _, _ = run(case, moe.MOE_PATH_PREFILL, dev)
    b, ib, _, _ = run(case, moe.MOE_PATH_PREFILL_NARROW, dev)
    assert np.array_equal(ia, ib)
    rel = np.linalg.norm(a - b) / np.linalg.norm(a)
    assert rel < 2e-3, rel
