"""Pins for the CPU oracle, each against something other than the oracle.

- e4m3 codec: every one of the 256 codes against torch's float8_e4m3fn
  decode (a library routine) and against the OCP E4M3 table's landmark
  values; the encoder against torch's round-to-nearest-even cast, including
  every exact midpoint between neighbouring codes, and saturation at 448.
- bf16: all 65,536 patterns against torch's bf16 decode; the rounding
  function against torch's fp32->bf16 cast on fp32-exact inputs.
- block quantiser: the half-ulp-times-scale bound, and bit equality with the
  input generator's torch-based encoder.
- top-k: brute force by a stable sort; k = E reduces to a plain softmax
  (scipy); weights sum to one; ties go to the lower expert index.
- one expert: a numpy float64 SwiGLU built from torch-decoded weights.
- the layer: with E = 1, k = 1 and a zero gate vector it reduces to
  expert(x) + expert_shared(x)/2; the routed result equals the dense,
  all-experts evaluation masked to the top-k; a hand-derived case with
  exact dyadic outputs.
- the shared-expert gate: hand cases with g . x = +2, -2, -2.5, 3.5 against
  scipy's logistic function (a flipped sign or a dot product with another
  vector fails), and random gate vectors against numpy's float64 dot.
- the router-only entry equals the layer's own routing (logits, experts,
  weights, gate) on the tiny and 35B-A3B-shaped layers.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import moe_inputs as mi
import oracle


# ------------------------------------------------------------------ e4m3

def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(mine) & np.isnan(ref)
    assert np.all((mine == ref) | both_nan)
    # exactly two NaN codes (S.1111.111), no infinities
    assert set(np.flatnonzero(np.isnan(mine)).tolist()) == {0x7F, 0xFF}
    assert not np.any(np.isinf(mine))


def test_e4m3_landmarks_from_ocp_table():
    # OCP 8-bit FP spec, E4M3 column
    assert oracle.e4m3_decode(0x7E) == 448.0                    # max normal S.1111.110
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6                # min normal S.0001.000
    assert oracle.e4m3_decode(0x07) == 0.875 * 2.0 ** -6        # max subnormal S.0000.111
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9                # min subnormal S.0000.001
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0xB8) == -1.0
    assert oracle.e4m3_decode(0x80) == 0.0 and math.copysign(1, oracle.e4m3_decode(0x80)) < 0


def _finite_codes():
    return [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_e4m3_encode_roundtrip_every_finite_code():
    for c in _finite_codes():
        v = oracle.e4m3_decode(c)
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_e4m3_encode_matches_torch_rne_including_midpoints():
    pos = sorted(oracle.e4m3_decode(c) for c in range(0x00, 0x7F))
    mids = [(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])]
    rng = np.random.default_rng(1)
    rand = (rng.standard_normal(20000) * rng.choice([1e-3, 0.05, 1, 30, 200], 20000)).tolist()
    vals = [v for v in pos + mids + rand if abs(v) < 464]
    vals = vals + [-v for v in vals]
    v32 = np.array(vals, dtype=np.float32)          # all chosen values are fp32-exact or fp32 draws
    ref = torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_encode(float(v)) for v in v32], dtype=np.uint8)
    assert np.array_equal(mine, ref)
    # midpoints resolve to the even code
    for a, m in zip(pos[:-1], mids):
        c = oracle.e4m3_encode(m)
        assert c % 2 == 0


def test_e4m3_encode_saturates():
    assert oracle.e4m3_encode(449.0) == 0x7E
    assert oracle.e4m3_encode(1e6) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F


# ------------------------------------------------------------------ bf16

def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = oracle.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    both_nan = np.isnan(mine) & np.isnan(ref)
    assert np.all((mine == ref) | both_nan)


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(20000) * rng.choice([1e-30, 1e-3, 1, 1e5, 1e30], 20000)).astype(np.float32)
    # exact ties between neighbouring bf16 values: low 16 bits = 0x8000
    ties = (rng.integers(0, 2 ** 31, 2000, dtype=np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    v = np.concatenate([v, ties.view(np.float32)])
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = oracle.round_to_bf16(v.astype(np.float64))
    assert np.array_equal(mine, ref)
    assert oracle.f64_to_bf16(1e39) == 0x7F80     # overflow to +inf


# ------------------------------------------------------------ quantiser

def _ulp_e4m3(q):
    a = np.abs(q)
    out = np.full(a.shape, 2.0 ** -9)
    n = a >= 2.0 ** -6
    out[n] = 2.0 ** (np.floor(np.log2(a[n])) - 3)
    return out


def test_quantise_dequantise_within_half_ulp_times_scale():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((256, 384)) * 0.02).astype(np.float32)
    w[0:128, 0:128] = 0.0                            # an all-zero block
    w[128:256, 256:384] *= 1e-4                      # a block in the subnormal-heavy range
    q, s = oracle.quantize_blocks(w)
    assert s[0, 0] == 1.0 and np.all(q[0:128, 0:128] == 0)
    dec = np.array([oracle.e4m3_decode(int(c)) for c in range(256)])
    qv = dec[q]
    S = np.kron(s.astype(np.float64), np.ones((128, 128)))
    err = np.abs(qv * S - w.astype(np.float64))
    bound = 0.5 * _ulp_e4m3(qv) * S
    # the quotient w/s is formed in fp32, so allow its own rounding on top
    assert np.all(err <= bound * (1 + 1e-6) + np.abs(w) * 2.0 ** -23)
    # each block's largest magnitude maps to 448
    for bi in range(2):
        for bj in range(3):
            blk = np.abs(qv[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128])
            if s[bi, bj] != 1.0:
                assert blk.max() == 448.0


def test_oracle_quantiser_matches_input_generator_bit_for_bit():
    g = torch.Generator().manual_seed(4)
    w = torch.randn(384, 256, generator=g) * 0.02
    q1, s1 = mi.encode_e4m3_blocks(w)
    q2, s2 = oracle.quantize_blocks(w.numpy())
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


# ----------------------------------------------------------------- top-k

def test_topk_brute_force_and_invariants():
    rng = np.random.default_rng(5)
    for E, k in [(16, 2), (256, 8), (512, 10), (7, 7)]:
        for _ in range(20):
            l = rng.standard_normal(E)
            idx, w = oracle.topk(l, k)
            order = np.lexsort((np.arange(E), -l))[:k]   # stable: (-l, e)
            assert np.array_equal(idx, order)
            assert abs(w.sum() - 1.0) < 1e-12
            assert np.all(np.diff(w) <= 0)
            ref = scipy.special.softmax(l[order])
            assert np.allclose(w, ref, rtol=1e-13, atol=0)


def test_topk_full_softmax_when_k_equals_E():
    l = np.array([0.3, -1.2, 2.5, 0.0, 0.7])
    idx, w = oracle.topk(l, 5)
    full = scipy.special.softmax(l)
    assert np.allclose(w, full[idx], rtol=1e-14)


def test_topk_ties_prefer_lower_index():
    l = np.array([1.0, 3.0, 3.0, 2.0, 3.0])
    idx, w = oracle.topk(l, 2)
    assert idx.tolist() == [1, 2]
    assert w.tolist() == [0.5, 0.5]


# ------------------------------------------------------------ one expert

def _dequant(q, s):
    dec = torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return dec * np.kron(s.astype(np.float64), np.ones((128, 128)))


def _numpy_swiglu(slab, scales, H, I, x):
    w13q = slab[: 2 * I * H].reshape(2 * I, H)
    w2q = slab[2 * I * H:].reshape(H, I)
    n13 = (2 * I // 128) * (H // 128)
    s13 = scales[:n13].reshape(2 * I // 128, H // 128)
    s2 = scales[n13:].reshape(H // 128, I // 128)
    W13, W2 = _dequant(w13q, s13), _dequant(w2q, s2)
    gu = W13 @ x
    g, u = gu[:I], gu[I:]
    h = g * scipy.special.expit(g) * u
    return W2 @ h


@pytest.mark.parametrize("H,I", [(256, 128), (384, 256)])
def test_expert_ffn_matches_numpy_swiglu(H, I):
    d = mi.LayerDims(hidden=H, n_experts=1, top_k=1, inter=I, shared_inter=I)
    slab, sc = mi.expert_slab(d, seed=7, e=0)
    x = np.random.default_rng(6).standard_normal(H)
    y = oracle.expert_ffn(slab, sc, H, I, x)
    ref = _numpy_swiglu(slab, sc, H, I, x)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------- the layer

def test_single_expert_layer_reduces_to_dense_swiglu():
    """E = 1, k = 1, zero gate vector: out = expert_0(x) + sigmoid(0) * shared(x)."""
    d = mi.LayerDims(hidden=256, n_experts=1, top_k=1, inter=128, shared_inter=256)
    L = mi.make_layer(d, seed=8)
    gate0 = np.zeros_like(L.shared_gate)
    x = mi.make_x(d, 3, seed=8)
    r = oracle.moe_forward(d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                           L.shared_scales, gate0)
    xd = oracle.bf16_bits_to_f64(x)
    for t in range(3):
        ref = (_numpy_swiglu(L.expert_w8[0], L.expert_scales[0], 256, 128, xd[t])
               + 0.5 * _numpy_swiglu(L.shared_w8, L.shared_scales, 256, 256, xd[t]))
        assert np.allclose(r.out[t], ref, rtol=1e-12, atol=1e-13)
    assert np.all(r.idx == 0) and np.all(r.w == 1.0) and np.all(r.gate_sig == 0.5)


@pytest.mark.parametrize("dims,rows,bias", [
    (mi.TINY, 4, False),
    (mi.TINY, 4, True),
    (mi.LayerDims(hidden=384, n_experts=12, top_k=3, inter=256, shared_inter=128), 3, False),
])
def test_routed_equals_dense_masked(dims, rows, bias):
    L = mi.make_layer(dims, seed=0, router_bias=bias)
    x = mi.make_x(dims, rows, seed=0)
    res = mi.make_residual(dims, rows, seed=0)
    args = (dims, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8, L.shared_scales,
            L.shared_gate)
    a = oracle.moe_forward(*args, residual=res, router_bias=L.router_bias)
    b = oracle.moe_forward_dense(*args, residual=res, router_bias=L.router_bias)
    assert np.array_equal(a.idx, b.idx)
    rel = np.linalg.norm(a.out - b.out) / np.linalg.norm(a.out)
    assert rel <= 1e-12
    assert np.allclose(a.w.sum(axis=1), 1.0, atol=1e-12)


def test_forced_routing_equals_own_routing():
    d = mi.TINY
    L = mi.make_layer(d, seed=1)
    x = mi.make_x(d, 4, seed=1)
    args = (d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8, L.shared_scales,
            L.shared_gate)
    a = oracle.moe_forward(*args)
    b = oracle.moe_forward(*args, forced_idx=a.idx)
    assert np.array_equal(a.out, b.out) and np.array_equal(a.w, b.w)


# ------------------------------------------------------- hand-derived case

def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _slab_from_fp32(w13, w2):
    q13, s13 = oracle.quantize_blocks(w13)
    q2, s2 = oracle.quantize_blocks(w2)
    return (np.concatenate([q13.ravel(), q2.ravel()]), np.concatenate([s13.ravel(), s2.ravel()]))


def test_hand_derived_layer():
    """H = I = Is = 128, E = 4, k = 2, one row.

    Every 128x128 block holds a 112 somewhere, so its scale is 112/448 = 0.25
    exactly and the entries {0, +-0.25, +-0.5, +-112} are codes {0, +-1, +-2,
    +-448}: the dequantised weights are exact.  x = e_0 + 2 e_1.

    Router rows give logits [1, 3, 3, 2]: the top-2 is the tie {1, 2}, which
    resolves to order [1, 2] with weights 1/2, 1/2.  The gate vector has
    g.x = 2 - 2 = 0, so sigmoid = 1/2.  silu(112) = 112 in double (exp(-112)
    vanishes next to 1) and silu(-112) is below 1e-46.

    expert 1: gate_0 = 112 x_0 = 112, up_0 = 0.5 x_1 = 1      -> h_0 = 112
              gate_1 = -112, up_1 = 0.25                       -> h_1 ~ -7e-48
              y_0 = 0.25 h_0 = 28, y_1 = -0.5 h_0 = -56, y_2 = 112 h_1 ~ 0
    expert 2: gate_0 = 112, up_0 = -0.5 x_0 = -0.5             -> h_0 = -56
              y_0 = 0.5 h_0 = -28, y_3 = 0.25 h_0 = -14
    shared:   gate_0 = 112, up_0 = 0.25 x_1 = 0.5              -> h_0 = 56
              y_0 = 0.5 h_0 = 28, y_4 = -0.25 h_0 = -14
    experts 0 and 3 are not selected but would put 112*112*112 into out[5].

    out = (y1 + y2)/2 + y_shared/2 = [14, -28, ~0, -7, -7, 0, ...]; with the
    residual r_0 = 1 the first entry becomes 15.
    """
    H = I = 128
    d = mi.LayerDims(hidden=H, n_experts=4, top_k=2, inter=I, shared_inter=I)
    x = np.zeros((1, H), dtype=np.float32)
    x[0, 0], x[0, 1] = 1.0, 2.0
    rw = np.zeros((4, H), dtype=np.float32)
    rw[0, :2] = [1, 0]
    rw[1, :2] = [1, 1]
    rw[2, :2] = [3, 0]
    rw[3, :2] = [0, 1]
    g = np.zeros(H, dtype=np.float32)
    g[0], g[1] = 2.0, -1.0

    def expert(kind):
        w13 = np.zeros((2 * I, H), dtype=np.float32)
        w2 = np.zeros((H, I), dtype=np.float32)
        w13[0, 0] = 112.0
        if kind == 1:
            w13[1, 0] = -112.0
            w13[I + 0, 1] = 0.5
            w13[I + 1, 0] = 0.25
            w13[2 * I - 1, H - 1] = 112.0
            w2[0, 0], w2[1, 0], w2[2, 1] = 0.25, -0.5, 112.0
        elif kind == 2:
            w13[I + 0, 0] = -0.5
            w13[2 * I - 1, H - 1] = 112.0
            w2[0, 0], w2[3, 0], w2[H - 1, I - 1] = 0.5, 0.25, 112.0
        elif kind == "shared":
            w13[I + 0, 1] = 0.25
            w13[2 * I - 1, H - 1] = 112.0
            w2[0, 0], w2[4, 0], w2[H - 1, I - 1] = 0.5, -0.25, 112.0
        else:  # masked experts
            w13[I + 0, 0] = 112.0
            w2[5, 0] = 112.0
        return _slab_from_fp32(w13, w2)

    slabs = [expert(0), expert(1), expert(2), expert(3)]
    w8 = np.stack([s[0] for s in slabs])
    sc = np.stack([s[1] for s in slabs])
    assert np.all(sc == 0.25)
    sw8, ssc = expert("shared")
    r = oracle.moe_forward(d, _bf16(x), _bf16(rw), w8, sc, sw8, ssc, _bf16(g))
    assert r.logits[0].tolist() == [1.0, 3.0, 3.0, 2.0]
    assert r.idx[0].tolist() == [1, 2] and r.w[0].tolist() == [0.5, 0.5]
    assert r.gate_sig[0] == 0.5
    out = r.out[0]
    assert out[0] == 14.0 and out[1] == -28.0 and out[3] == -7.0 and out[4] == -7.0
    assert abs(out[2]) < 1e-40 and out[5] == 0.0
    assert np.all(out[6:] == 0.0)
    res = np.zeros((1, H), dtype=np.float32)
    res[0, 0] = 1.0
    r2 = oracle.moe_forward(d, _bf16(x), _bf16(rw), w8, sc, sw8, ssc, _bf16(g), residual=_bf16(res))
    assert r2.out[0, 0] == 15.0 and r2.out[0, 1] == -28.0
    dn = oracle.moe_forward_dense(d, _bf16(x), _bf16(rw), w8, sc, sw8, ssc, _bf16(g))
    assert np.array_equal(dn.out[0, :2], out[:2])


def test_router_bias_shifts_selection():
    """A bias of +100 on one expert forces it into every row's top-k."""
    d = mi.TINY
    L = mi.make_layer(d, seed=2)
    x = mi.make_x(d, 4, seed=2)
    bias = np.zeros(d.n_experts, dtype=np.float32)
    bias[11] = 100.0
    r = oracle.moe_forward(d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                           L.shared_scales, L.shared_gate, router_bias=bias)
    assert np.all(r.idx[:, 0] == 11)
    r0 = oracle.moe_forward(d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                            L.shared_scales, L.shared_gate)
    assert np.allclose(r.logits - r0.logits, bias[None, :], atol=1e-12)


# ------------------------------------------------------- regression record

def test_oracle_reproduces_its_tiny_regression_record():
    import json
    import os
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, os.path.join(here, "golden"))
    import make_golden
    with open(os.path.join(here, "golden", "tiny_seed0.json")) as f:
        stored = json.load(f)
    assert make_golden.tiny_record(0) == stored


# ------------------------------------------------------- shared-expert gate

def _gate_case(gate_entries):
    """H = I = Is = 128, E = 2, k = 1, one row x = e_0 + 2 e_1 (exact bf16).

    Router rows give logits [1, 0], so expert 0 is chosen with weight 1.
    Every 128x128 block holds a 112, so its scale is 0.25 and the entries
    used are exact codes.  Expert 0: gate_0 = 112 x_0, up_0 = 0.25 x_1 = 0.5,
    h_0 = silu(112) * 0.5 = 56, y_0 = 0.5 * 56 = 28.  Shared expert: gate_0 =
    112 x_0, up_0 = 0.5 x_1 = 1, h_0 = 112, y_1 = 0.25 * 112 = 28.  So
    out = [28, sigmoid(z) * 28, 0, ...] with z = g . x set by the gate
    vector's first two entries.
    """
    H = I = 128
    d = mi.LayerDims(hidden=H, n_experts=2, top_k=1, inter=I, shared_inter=I)
    x = np.zeros((1, H), dtype=np.float32)
    x[0, 0], x[0, 1] = 1.0, 2.0
    rw = np.zeros((2, H), dtype=np.float32)
    rw[0, 0] = 1.0
    g = np.zeros(H, dtype=np.float32)
    g[0], g[1] = gate_entries

    def slab(up_val, y_row, y_val):
        w13 = np.zeros((2 * I, H), dtype=np.float32)
        w2 = np.zeros((H, I), dtype=np.float32)
        w13[0, 0] = 112.0
        w13[I + 0, 1] = up_val
        w13[2 * I - 1, H - 1] = 112.0     # sets every W13 block's scale to 0.25
        w2[y_row, 0] = y_val
        w2[H - 1, I - 1] = 112.0          # and the W2 block's
        return _slab_from_fp32(w13, w2)

    e0 = slab(0.25, 0, 0.5)
    e1 = slab(0.0, 2, 112.0)              # never chosen
    sh = slab(0.5, 1, 0.25)
    w8 = np.stack([e0[0], e1[0]])
    sc = np.stack([e0[1], e1[1]])
    return d, _bf16(x), _bf16(rw), w8, sc, sh[0], sh[1], _bf16(g)


@pytest.mark.parametrize("entries,z", [((1.0, 0.5), 2.0), ((0.0, -1.0), -2.0), ((-3.0, 0.25), -2.5),
                                       ((0.5, 1.5), 3.5)])
def test_shared_gate_sigmoid_at_nonzero_z(entries, z):
    """sigmoid(g . x) with g . x != 0, against scipy's logistic function: a
    flipped sign (sigmoid(-z)), a dropped factor or a dot product with
    another vector (the router row gives 1 here) fails."""
    d, x, rw, w8, sc, sw8, ssc, g = _gate_case(entries)
    r = oracle.moe_forward(d, x, rw, w8, sc, sw8, ssc, g)
    want = scipy.special.expit(z)
    assert r.idx[0].tolist() == [0] and r.w[0].tolist() == [1.0]
    assert abs(r.gate_sig[0] - want) <= 1e-15
    assert abs(r.gate_sig[0] - scipy.special.expit(-z)) > 0.1      # the sign matters here
    assert r.out[0, 0] == 28.0
    assert abs(r.out[0, 1] - want * 28.0) <= 1e-13
    assert np.all(r.out[0, 2:] == 0.0)
    _, _, _, gs = oracle.router_topk(d, x, rw, g)
    assert abs(gs[0] - want) <= 1e-15


def test_shared_gate_against_numpy_dot():
    """Random gate vectors (tiny layer, 4 rows): the oracle's gate equals
    scipy.expit of numpy's float64 dot product of the bf16-decoded x and g."""
    d = mi.TINY
    L = mi.make_layer(d, seed=3)
    x = mi.make_x(d, 4, seed=3)
    g = mi._bf16_bits(torch.randn(d.hidden, generator=torch.Generator().manual_seed(11)) * 0.05)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    gd = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    z = xd @ gd
    assert np.all(np.abs(z) > 0.05)
    r = oracle.moe_forward(d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                           L.shared_scales, g)
    assert np.allclose(r.gate_sig, scipy.special.expit(z), rtol=0, atol=1e-14)


def _router_vs_forward(d, L, x, bias=None):
    lg, idx, w, gs = oracle.router_topk(d, x, L.router_w, L.shared_gate, router_bias=bias)
    r = oracle.moe_forward(d, x, L.router_w, L.expert_w8, L.expert_scales, L.shared_w8,
                           L.shared_scales, L.shared_gate, router_bias=bias)
    assert np.array_equal(lg, r.logits)
    assert np.array_equal(idx, r.idx)
    assert np.array_equal(w, r.w)
    assert np.array_equal(gs, r.gate_sig)


def test_router_entry_equals_forward_routing_tiny():
    """The router-only entry (the reference routing of every GPU test) gives
    the same logits, experts, weights and gate as the layer's own routing."""
    d = mi.TINY
    L = mi.make_layer(d, seed=0, router_bias=True)
    x = mi.make_x(d, 6, seed=0)
    _router_vs_forward(d, L, x)
    _router_vs_forward(d, L, x, L.router_bias)


def test_router_entry_equals_forward_routing_35b():
    d = mi.QWEN36_35B_A3B
    x = mi.make_x(d, 2, seed=0, stream=2)
    rw, g, _ = mi.make_router(d, 0)
    lg, idx, _, _ = oracle.router_topk(d, x, rw, g)
    L = mi.make_layer(d, seed=0, experts=set(idx.ravel().tolist()))
    _router_vs_forward(d, L, x)


# ------------------------------------------------------------------ RMSNorm

def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_rmsnorm_hand_cases():
    """Cases with exact results: a row of 2s has mean square 4, so with eps = 0
    x = w exactly and with eps = 12 x = 2 w / 4 = w / 2 exactly (an eps added after
    the root, or a mean over H - 1, fails); a row (8, 0, ..., 0) of H = 128
    has mean square 1/2, so x_0 = 8 sqrt(2) w_0, whose nearest bf16 is 11.3125."""
    H = 128
    w = _bf16_bits(np.linspace(-3.0, 3.0, H))
    wd = oracle.bf16_bits_to_f64(w)
    r = _bf16_bits(np.full((2, H), 2.0))
    r[1] = _bf16_bits(np.full(H, -2.0))
    xd, xb = oracle.rmsnorm(r, w, 0.0)
    assert np.array_equal(xd[0], wd) and np.array_equal(xd[1], -wd)
    assert np.array_equal(xb[0], w)
    xd, _ = oracle.rmsnorm(r[:1], w, 12.0)
    assert np.array_equal(xd[0], wd / 2.0)
    one = _bf16_bits(np.ones(H))
    r2 = np.zeros((1, H), dtype=np.uint16)
    r2[0, 0] = _bf16_bits([8.0])[0]
    xd, xb = oracle.rmsnorm(r2, one, 0.0)
    assert abs(xd[0, 0] - 8.0 * math.sqrt(2.0)) <= 1e-14
    assert oracle.bf16_to_f64(int(xb[0, 0])) == 11.3125
    assert np.all(xd[0, 1:] == 0.0)


def test_rmsnorm_matches_torch_float64():
    """Random residual rows against torch's rms_norm in float64 (a library
    routine)."""
    H, rows, eps = 384, 5, 1e-6
    g = torch.Generator().manual_seed(3)
    r = _bf16_bits((torch.randn(rows, H, generator=g) * 3.0).numpy())
    w = _bf16_bits((1.0 + 0.1 * torch.randn(H, generator=g)).numpy())
    xd, xb = oracle.rmsnorm(r, w, eps)
    rt = torch.from_numpy(oracle.bf16_bits_to_f64(r))
    wt = torch.from_numpy(oracle.bf16_bits_to_f64(w))
    ref = torch.nn.functional.rms_norm(rt, (H,), weight=wt, eps=eps).numpy()
    assert np.allclose(xd, ref, rtol=1e-14, atol=0.0)
    assert np.array_equal(xb, oracle.round_to_bf16(xd))
