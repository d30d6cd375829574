"""Pins of the oracle's NVFP4 expert format (CPU only).

NVFP4 (the expert format of the Qwen3.5-397B-A17B-NVFP4 checkpoint, "The
Config That Launched a Thousand GPUs" page; the format itself is its public
definition, a reading): e2m1 codes, one e4m3 scale per 16 consecutive
elements along the reduction dimension, one fp32 scale per matrix.  Each
part is pinned against something other than the oracle itself:

- the e2m1 codec against ml_dtypes' float4_e2m1fn (all 16 codes; rounding
  of random, tie and saturating values);
- the quantiser against the input generator's library casts (torch e4m3,
  ml_dtypes e2m1), bit for bit, and against the closed-form error bound of
  round-to-nearest on the e2m1 grid;
- the layout (nibble order, scale indexing, per-matrix tensor scales, slab
  offsets) against the FP8 layer, already pinned: on weights that both
  formats represent exactly, the two oracle layers must agree bit for bit;
- the routed layer against its dense brute force.
"""
import ml_dtypes
import numpy as np
import pytest

import moe_inputs as mi
import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def test_e2m1_decode_matches_ml_dtypes_on_all_codes():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_decode(c) for c in range(16)])
    assert np.array_equal(ours, lib)
    assert np.array_equal(np.signbit(ours), np.signbit(lib))
    assert ours.max() == 6.0 and sorted(set(np.abs(ours))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_matches_ml_dtypes_rounding():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.normal(0, 3, 4000), rng.uniform(-8, 8, 4000),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 7.0, 100.0, -0.25, -5.0, -9.0,
                                  0.0, -0.0, 1e-9, -1e-9])]).astype(np.float32)
    lib = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0x0F
    ours = np.array([oracle.e2m1_encode(float(a)) for a in v], dtype=np.uint8)
    assert np.array_equal(ours, lib)


@pytest.mark.parametrize("case", ["normal", "zero_blocks", "all_zero", "wide_rows"])
def test_nvfp4_quantiser_matches_library_casts(case):
    import torch
    w = mi._normal((128, 256), 0.02, 11, "nvfp4_pin", 0)
    if case == "zero_blocks":
        w[:, 16:48] = 0.0
        w[5, :] = 0.0
    elif case == "all_zero":
        w = torch.zeros_like(w)
    elif case == "wide_rows":
        w = w * torch.logspace(-6, 2, 128).reshape(128, 1).to(torch.float32)
    q, sf, gs = mi.encode_nvfp4(w)
    q2, sf2, gs2 = oracle.quantize_nvfp4(w.numpy())
    assert np.array_equal(q, q2) and np.array_equal(sf, sf2) and np.float32(gs) == np.float32(gs2)


def _dequant(q, sf, gs, cols):
    lo, hi = q & 0x0F, q >> 4
    codes = np.empty((q.shape[0], cols), dtype=np.uint8)
    codes[:, 0::2], codes[:, 1::2] = lo, hi
    vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    scale = sf.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return vals * np.repeat(scale, 16, axis=1) * np.float64(gs), codes


def test_nvfp4_dequantisation_error_is_within_half_an_e2m1_step():
    w = mi._normal((128, 512), 0.02, 12, "nvfp4_bound", 0).numpy().astype(np.float64)
    q, sf, gs = oracle.quantize_nvfp4(w.astype(np.float32))
    dq, _ = _dequant(q, sf, gs, 512)
    unit = np.repeat(sf.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1) * gs
    a = np.abs(w) / unit                                   # the scaled magnitude the code rounds
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))  # e2m1 grid spacing there
    bound = np.where(a <= 6, step / 2, a - 6) * unit * (1 + 1e-6) + 1e-30
    assert np.all(np.abs(w - dq) <= bound)
    # the block scale keeps every block's largest element within one e4m3 rounding of 6
    assert np.all(a.reshape(128, 32, 16).max(axis=2)[sf != 0] <= 6 * 1.0625 + 1e-9)


def _exact_pair(rng, R, C):
    """NVFP4 bytes whose values an FP8 matrix with a power-of-two block scale
    holds exactly: e2m1 codes at random, block scales 2^-3..2^3, gs = 2^-10."""
    codes = rng.integers(0, 16, size=(R, C), dtype=np.uint8)
    q4 = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    k = rng.integers(-3, 4, size=(R, C // 16))
    sf = np.array([[oracle.e4m3_encode(2.0 ** e) for e in row] for row in k], dtype=np.uint8)
    gs = np.float32(2.0 ** -10)
    vals = np.array([[oracle.e2m1_decode(c) for c in row] for row in codes]) * np.repeat(2.0 ** k, 16, axis=1)
    q8 = np.array([[oracle.e4m3_encode(v) for v in row] for row in vals], dtype=np.uint8)  # scale 2^-10
    assert np.array_equal(np.array([[oracle.e4m3_decode(c) for c in row] for row in q8]), vals)
    s8 = np.full((R // 128, C // 128), 2.0 ** -10, dtype=np.float32)
    return q4, sf, gs, q8, s8


def test_nvfp4_layer_equals_fp8_layer_on_weights_both_hold_exactly():
    d = mi.TINY
    H, I, Is, E = d.hidden, d.inter, d.shared_inter, d.n_experts
    rng = np.random.default_rng(5)
    rw, g, _ = mi.make_router(d, 5)

    def slab(inter):
        a13 = _exact_pair(rng, 2 * inter, H)
        a2 = _exact_pair(rng, H, inter)
        w4 = np.concatenate([a13[0].ravel(), a2[0].ravel()])
        sf = np.concatenate([a13[1].ravel(), a2[1].ravel()])
        gs = np.array([a13[2], a2[2]], dtype=np.float32)
        w8 = np.concatenate([a13[3].ravel(), a2[3].ravel()])
        s8 = np.concatenate([a13[4].ravel(), a2[4].ravel()])
        return w4, sf, gs, w8, s8

    ex = [slab(I) for _ in range(E)]
    sh = slab(Is)
    x = mi.make_x(d, 3, seed=5)
    f8 = oracle.moe_forward(d, x, rw, np.stack([e[3] for e in ex]), np.stack([e[4] for e in ex]), sh[3], sh[4], g)
    f4 = oracle.moe_forward_nvfp4(d, x, rw, np.stack([e[0] for e in ex]), np.stack([e[1] for e in ex]),
                                  np.stack([e[2] for e in ex]), sh[0], sh[1], sh[2], g)
    assert np.array_equal(f8.idx, f4.idx)
    assert np.array_equal(f8.out, f4.out)          # the same values in the same order
    assert np.abs(f8.out).max() > 0


def test_nvfp4_dense_brute_force_equals_routed():
    d = mi.TINY
    layer = mi.make_layer_nvfp4(d, seed=6)
    x = mi.make_x(d, 4, seed=6)
    args = (d, x, layer.router_w, layer.expert_w4, layer.expert_sf, layer.expert_gs, layer.shared_w4,
            layer.shared_sf, layer.shared_gs, layer.shared_gate)
    r = oracle.moe_forward_nvfp4(*args)
    b = oracle.moe_forward_nvfp4(*args, dense=True)
    assert np.array_equal(r.idx, b.idx)
    assert np.max(np.abs(r.out - b.out)) <= 1e-12 * np.max(np.abs(r.out))


def test_nvfp4_layer_is_close_to_the_fp8_layer_of_the_same_weights():
    """Sanity of the whole chain on the seeded weights: both formats quantise
    the same fp32 draws, so the two layers differ by quantisation noise only
    (e2m1 keeps ~2 significant bits against e4m3's 4)."""
    d = mi.TINY
    l8 = mi.make_layer(d, seed=7)
    l4 = mi.make_layer_nvfp4(d, seed=7)
    x = mi.make_x(d, 4, seed=7)
    f8 = oracle.moe_forward(d, x, l8.router_w, l8.expert_w8, l8.expert_scales, l8.shared_w8, l8.shared_scales,
                            l8.shared_gate)
    f4 = oracle.moe_forward_nvfp4(d, x, l4.router_w, l4.expert_w4, l4.expert_sf, l4.expert_gs, l4.shared_w4,
                                  l4.shared_sf, l4.shared_gs, l4.shared_gate)
    assert np.array_equal(f8.idx, f4.idx)          # the router is the same bf16 layer
    rel = np.linalg.norm(f4.out - f8.out) / np.linalg.norm(f8.out)
    assert 1e-3 < rel < 0.25
