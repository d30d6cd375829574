"""The workspace-free entry point (moe_ffn_forward_static) against the
workspace entry point (moe_ffn_forward), through the C ABI, on the GPU.

The static variant serves callers that cannot allocate device memory; it
runs the same kernels on a scratch array built into the library.  Two calls
in a row must each match the workspace call (the array keeps the previous
call's contents, which must not leak into the next result).  This file sorts
last so that a run stopping at the first failure has run everything else.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


def _inputs(dims, rows, seed, layer=None):
    layer = layer or mi.make_layer(dims, seed=seed)
    dev = P.device_weights(layer)
    xs = [P.bf16_tensor(mi.make_x(dims, rows, seed=seed, stream=100 + i)) for i in range(2)]
    return dev, xs


def _run_both(dims, dev, x):
    rows = x.shape[0]
    ws = moe.alloc_workspace(dims, rows)
    ref = torch.empty(rows, dims.hidden, dtype=torch.bfloat16, device="cuda")
    moe.ffn_forward(dims, x, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                    dev["shared_scales"], dev["shared_gate"], ref, ws)
    got = torch.full((rows, dims.hidden), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.ffn_forward_static(dims, x, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                           dev["shared_scales"], dev["shared_gate"], got)
    torch.cuda.synchronize()
    return P.bf16_to_f64(ref), P.bf16_to_f64(got)


def _check_close(ref, got):
    err = got - ref
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    assert np.all(np.isfinite(got))
    assert rel <= P.REL_L2_TOL and np.max(np.abs(err)) <= P.MAX_ABS_TOL
    assert np.array_equal(ref, got)   # the same kernels on the same inputs


# AUTO's three paths: (35B, 1) the decode kernels; (TINY, 4), (35B, 8), (TINY, 100) the narrow
# grouped GEMMs; (TINY, 300) the grouped GEMMs with 128-row tiles
@pytest.mark.parametrize("dims,rows", [(mi.TINY, 4), (mi.QWEN36_35B_A3B, 1), (mi.QWEN36_35B_A3B, 8), (mi.TINY, 100),
                                       (mi.TINY, 300)])
def test_static_scratch_matches_workspace_two_calls_in_a_row(dims, rows):
    dev, xs = _inputs(dims, rows, seed=5)
    for x in xs:                      # two calls in a row on different inputs
        ref, got = _run_both(dims, dev, x)
        _check_close(ref, got)


def test_static_scratch_rejects_shapes_beyond_its_size():
    d = mi.QWEN35_397B_A17B
    rows = 128
    assert moe.workspace_bytes(d, rows) > moe.static_scratch_bytes()
    x = torch.zeros(rows, d.hidden, dtype=torch.bfloat16, device="cuda")
    dummy8 = torch.zeros(16, dtype=torch.uint8, device="cuda")
    dummyf = torch.zeros(4, dtype=torch.float32, device="cuda")
    dummyb = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(rows, d.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.ffn_forward_static(d, x, dummyb, dummy8, dummyf, dummy8, dummyf, dummyb, out)
    assert e.value.status == moe.MOE_EWORKSPACE


def test_static_timeout_is_reported_and_not_erased_by_the_next_call():
    """A bounded wait that runs out on the scratch array (a 2 ms wait on an
    mbarrier nothing completes) shows up as MOE_ETIMEOUT through
    moe_static_device_status, even after another static call, and is
    reported once."""
    d = mi.TINY
    dev, xs = _inputs(d, 4, seed=6)
    assert moe.static_device_status() == moe.MOE_OK
    moe.debug_wait_timeout_static(2000)
    out = torch.empty(4, d.hidden, dtype=torch.bfloat16, device="cuda")
    moe.ffn_forward_static(d, xs[0], dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                           dev["shared_scales"], dev["shared_gate"], out)
    assert moe.static_device_status() == moe.MOE_ETIMEOUT
    assert moe.static_device_status() == moe.MOE_OK
    assert moe.status() == moe.MOE_OK
    ref, got = _run_both(d, dev, xs[1])        # the array still serves correct calls
    _check_close(ref, got)
