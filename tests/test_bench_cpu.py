"""The benchmark's host-side arithmetic and its reference arm, on CPU.

The byte and FLOP counts behind every GB/s and TFLOP/s figure are checked
against totals worked out by hand from the layer's shapes (one expert slab
of 3*I*H e4m3 bytes plus one fp32 scale per 128x128 block; 2 FLOP per
multiply-add), and the reference arm (the CPU oracle timed on the
benchmark's workload) must print one JSON line of the benchmark's contract.
"""
import json
import os
import subprocess
import sys

import moe_inputs as mi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_decode_bytes_35b_rows1():
    # 8 routed experts + the shared one: 9 slabs of 3*512*2048 bytes and
    # 8*16 + 16*4 scales; router 256 x 2048 bf16 + the gate vector; x and out
    slab = 3 * 512 * 2048 + 4 * (8 * 16 + 16 * 4)
    want = 9 * slab + 2 * 256 * 2048 + 2 * 2048 + 2 * 2048 * 2
    assert want == 29_379_328
    assert bench.algorithmic_bytes(mi.QWEN36_35B_A3B, 1, 8)["total"] == want


def test_decode_bytes_397b_rows1():
    slab = 3 * 1024 * 4096 + 4 * (16 * 32 + 32 * 8)
    want = 11 * slab + 2 * 512 * 4096 + 2 * 4096 + 2 * 4096 * 2
    assert want == 142_664_704
    assert bench.algorithmic_bytes(mi.QWEN35_397B_A17B, 1, 10)["total"] == want


def test_decode_bytes_grow_with_rows_only_through_activations():
    d = mi.QWEN36_35B_A3B
    a = bench.algorithmic_bytes(d, 1, 100)["total"]
    b = bench.algorithmic_bytes(d, 64, 100)["total"]
    assert b - a == 63 * 2 * 2048 * 2          # x in and out, bf16


def test_prefill_flops_35b_4096():
    f = bench.prefill_flops(mi.QWEN36_35B_A3B, 4096)
    # per token: 8 routed + 1 shared expert, each 2*(2I*H) + 2*(I*H) FLOP
    per_expert = 2 * 1024 * 2048 + 2 * 512 * 2048
    assert f["gemm_gate_up"] + f["gemm_down"] == 4096 * 9 * per_expert == 231_928_233_984
    assert f["router_topk"] == 4096 * 2 * (256 + 1) * 2048 == 4_311_744_512


def test_executed_flops_pad_each_group_to_128_rows_and_double_for_hi_lo():
    d = mi.LayerDims(hidden=256, n_experts=4, top_k=2, inter=128, shared_inter=128)
    counts = [1, 128, 129, 2]              # routed rows per expert: 260 pairs = 130 tokens
    ex = bench.prefill_executed_flops(d, counts)
    tiles = 1 + 1 + 2 + 1 + 2              # routed groups padded to 128 rows, then the shared 130 rows
    # a tile issues 128 rows x (2I x H) multiply-adds in GEMM1, 128 x (I x H) in
    # GEMM2, each once for hi and once for lo
    assert ex["gemm_gate_up"] == tiles * 128 * (2 * 128) * 256 * 2 * 2 == 234_881_024
    assert ex["gemm_down"] == tiles * 128 * 128 * 256 * 2 * 2 == 117_440_512


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["steps"] == 1 and j["n_gpus"] == 1
    assert j["value"] > 0 and j["unit"] == "GB/s" and j["higher_is_better"] is True
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["e2e"]["value"] == j["value"] and j["e2e"]["h2d_bytes_per_step"] == 0
    assert j["config"]["workload"].startswith("Qwen3.6-35B-A3B-shaped")
