"""The host-buffer entry point (moe_ffn_forward_host) against the device
entry point (moe_ffn_forward), through the C ABI, on the GPU.

x and out live in pinned host memory: a kernel reads x over the host link
and the forward's kernels store out straight into the host buffer.  The
result must be the device call's, bit for bit (the same kernels on the same
inputs), for every path AUTO takes, and a host buffer rewritten between two
calls must be read afresh.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


def _device_call(dims, dev, x, ws):
    out = torch.empty(x.shape[0], dims.hidden, dtype=torch.bfloat16, device="cuda")
    moe.ffn_forward(dims, x, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                    dev["shared_scales"], dev["shared_gate"], out, ws)
    return out


def _host_call(dims, dev, x_host, out_host, ws):
    moe.ffn_forward_host(dims, x_host, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                         dev["shared_scales"], dev["shared_gate"], out_host, ws)


# AUTO's three paths: (35B, 1), (35B, 3) the decode step; (TINY, 4), (TINY, 100) the narrow
# grouped GEMMs; (TINY, 300) the grouped GEMMs with 128-row tiles
@pytest.mark.parametrize("dims,rows", [(mi.QWEN36_35B_A3B, 1), (mi.QWEN36_35B_A3B, 3), (mi.TINY, 4),
                                       (mi.TINY, 100), (mi.TINY, 300)])
def test_host_buffers_match_the_device_call(dims, rows):
    layer = mi.make_layer(dims, seed=9)
    dev = P.device_weights(layer)
    ws = moe.alloc_workspace(dims, rows)
    xs = [P.bf16_tensor(mi.make_x(dims, rows, seed=9, stream=300 + i)) for i in range(3)]
    refs = [P.bf16_to_f64(_device_call(dims, dev, x, ws)) for x in xs]
    # two pinned buffers, then the first one rewritten with the third input
    hx = [torch.empty(rows, dims.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ho = [torch.full((rows, dims.hidden), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    for i, (src, dst) in enumerate([(0, 0), (1, 1), (0, 2)]):
        hx[src].copy_(xs[i].cpu())
        _host_call(dims, dev, hx[src], ho[dst], ws)
        torch.cuda.synchronize()
        got = P.bf16_to_f64(ho[dst])
        assert np.all(np.isfinite(got))
        assert np.array_equal(refs[i], got), f"call {i}"


def test_host_entry_refuses_device_memory():
    d = mi.QWEN36_35B_A3B
    layer = mi.make_layer(d, seed=9)
    dev = P.device_weights(layer)
    ws = moe.alloc_workspace(d, 1)
    x = P.bf16_tensor(mi.make_x(d, 1, seed=9, stream=1))
    out = torch.empty(1, d.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        _host_call(d, dev, x, out, ws)
    assert e.value.status == moe.MOE_EINVAL
