"""Write the oracle's regression fixtures for the tiny workload.

Calls only ``oracle`` and ``moe_inputs``.  The fixture is a regression
record of the oracle itself (it pins nothing on its own): a later change to
the oracle's arithmetic shows up as a mismatch and must then name the
reading of the pages that justifies it.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402


def tiny_record(seed: int = 0) -> dict:
    d = mi.TINY
    L = mi.make_layer(d, seed=seed)
    x = mi.make_x(d, 4, seed=seed)
    r = oracle.moe_forward(d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                           L.shared_scales, L.shared_gate)
    return {
        "workload": "tiny: hidden 256, 16 experts top-2, inter 128, shared inter 128, 4 rows, seed 0",
        "idx": r.idx.tolist(),
        "w": [[float.hex(float(v)) for v in row] for row in r.w],
        "gate_sig": [float.hex(float(v)) for v in r.gate_sig],
        "out_bf16_bits": oracle.round_to_bf16(r.out).astype(int).tolist(),
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_seed0.json")
    with open(path, "w") as f:
        json.dump(tiny_record(0), f, indent=1)
    print("wrote", path)
