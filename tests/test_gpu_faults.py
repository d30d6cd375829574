"""Failure detection on the GPU without faulting it: a bounded wait that runs
out is reported through the workspace status word, the context stays usable,
and the host-side error knob is sticky until reset."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import parity as P

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


def tiny_forward(ws):
    d = mi.TINY
    case = P.build_case(d, 4, all_experts=True)
    dev = P.device_weights(case.layer)
    out = torch.empty(4, d.hidden, dtype=torch.bfloat16, device="cuda")
    moe.ffn_forward(d, P.bf16_tensor(case.x), dev["router_w"], dev["expert_w8"], dev["expert_scales"],
                    dev["shared_w8"], dev["shared_scales"], dev["shared_gate"], out, ws)
    torch.cuda.synchronize()
    idx = np.argsort(-case.logits, axis=1, kind="stable")[:, :d.top_k].astype(np.int32)
    return case, P.bf16_to_f64(out), idx


def test_bounded_wait_reports_timeout_and_context_survives():
    d = mi.TINY
    ws = moe.alloc_workspace(d, 4)
    assert moe.device_status(ws) == moe.MOE_OK
    moe.debug_wait_timeout(ws, 2000)            # 2 ms on an mbarrier nobody completes
    assert moe.device_status(ws) == moe.MOE_ETIMEOUT
    assert moe.status() == moe.MOE_OK           # a device-side timeout is not a CUDA error
    moe.workspace_init(ws)
    assert moe.device_status(ws) == moe.MOE_OK
    case, out, idx = tiny_forward(ws)
    P.compare_output(case, out, idx)
    assert moe.device_status(ws) == moe.MOE_OK


def test_injected_fault_is_sticky_then_reset_recovers():
    d = mi.TINY
    ws = moe.alloc_workspace(d, 4)
    moe.reset_status()
    moe.debug_inject_fault(1)
    with pytest.raises(moe.MoeError) as e:
        tiny_forward(ws)
    assert e.value.status == moe.MOE_ECUDA
    with pytest.raises(moe.MoeError):
        tiny_forward(ws)                          # sticky
    moe.reset_status()
    moe.workspace_init(ws)
    case, out, idx = tiny_forward(ws)
    P.compare_output(case, out, idx)


def test_host_checks_on_gpu_tensors():
    d = mi.TINY
    L = mi.make_layer(d, seed=0)
    dev = P.device_weights(L)
    x = P.bf16_tensor(mi.make_x(d, 4))
    out = torch.empty(4, d.hidden, dtype=torch.bfloat16, device="cuda")
    small = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.ffn_forward(d, x, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                        dev["shared_scales"], dev["shared_gate"], out, small)
    assert e.value.status == moe.MOE_EWORKSPACE
    ws = moe.alloc_workspace(d, 4)
    xm = torch.empty(4 * d.hidden + 1, dtype=torch.bfloat16, device="cuda")[1:].view(4, d.hidden)
    with pytest.raises(moe.MoeError) as e:
        moe.ffn_forward(d, xm, dev["router_w"], dev["expert_w8"], dev["expert_scales"], dev["shared_w8"],
                        dev["shared_scales"], dev["shared_gate"], out, ws)
    assert e.value.status == moe.MOE_EINVAL
    assert moe.status() == moe.MOE_OK
