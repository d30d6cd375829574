"""Numerics behind the prefill path's activation format (CPU only).

The prefill path feeds activations to FP8 tensor cores.  The layer's
tolerance (relative L2 <= 5e-3 against the exact layer) rules out a single
e4m3 code per activation: three mantissa bits give a few percent error per
element.  The reading taken is a two-term split with one shared fp32 scale
per (row, 128-column block):

    s = amax/448,  q_hi = e4m3(v/s),  q_lo = e4m3(v/s - q_hi),  v ~ s*(q_hi + q_lo)

Because both terms share s, one accumulator takes both products.  This test
measures one 35B-shaped expert (H = 2048, I = 512) three ways with the
oracle's own e4m3 codec and numpy matmuls on the dequantised weights.
"""
import numpy as np
import scipy.special
import torch

import moe_inputs as mi
import oracle

_DEC = np.array([oracle.e4m3_decode(c) for c in range(256)])


def _enc(a):
    return np.array([oracle.e4m3_encode(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def _single(v):
    b = v.reshape(v.shape[0], -1, 128)
    s = np.abs(b).max(axis=2, keepdims=True) / 448.0
    s[s == 0] = 1.0
    return (_DEC[_enc(b / s)] * s).reshape(v.shape)


def _hilo(v):
    b = v.reshape(v.shape[0], -1, 128)
    s = np.abs(b).max(axis=2, keepdims=True) / 448.0
    s[s == 0] = 1.0
    hi = _DEC[_enc(b / s)]
    lo = _DEC[_enc(b / s - hi)]
    return ((hi + lo) * s).reshape(v.shape)


def test_single_fp8_activations_fail_and_hilo_split_passes():
    d = mi.QWEN36_35B_A3B
    H, I = d.hidden, d.inter
    slab, sc = mi.expert_slab(d, seed=0, e=0)
    n13 = (2 * I // 128) * (H // 128)
    dec = lambda q, s: (torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn)
                        .to(torch.float64).numpy() * np.kron(s.astype(np.float64), np.ones((128, 128))))
    W13 = dec(slab[: 2 * I * H].reshape(2 * I, H), sc[:n13].reshape(2 * I // 128, H // 128))
    W2 = dec(slab[2 * I * H:].reshape(H, I), sc[n13:].reshape(H // 128, I // 128))
    x = oracle.bf16_bits_to_f64(mi.make_x(d, 8, seed=0))

    def layer(fx, fh):
        gu = fx(x) @ W13.T
        h = gu[:, :I] * scipy.special.expit(gu[:, :I]) * gu[:, I:]
        return fh(h) @ W2.T

    exact = layer(lambda v: v, lambda v: v)
    rel = lambda y: np.linalg.norm(y - exact) / np.linalg.norm(exact)
    e_single = rel(layer(_single, _single))
    e_hilo = rel(layer(_hilo, _hilo))
    assert e_single > 5e-3          # misses the tolerance on its own
    assert e_hilo < 2e-3            # leaves room for the bf16 output rounding


def _e5m2(a):
    import ml_dtypes
    return np.asarray(a, dtype=np.float32).astype(ml_dtypes.float8_e5m2).astype(np.float64)


def test_bf16_splits_exactly_into_three_e5m2_terms():
    """The decode step feeds x to the tensor cores as three e5m2 terms per value
    after a power-of-two scale that puts the block's largest magnitude in
    [2^14, 2^15): t1 = e5m2(x'), t2 = e5m2(x' - t1), t3 = e5m2(x' - t1 - t2),
    each difference taken in fp32 as the kernel does.  Every bf16 value with
    x' >= 2^-9 (within 2^23 of the block maximum) is then exactly t1 + t2 + t3;
    below that the sum is within 2^-17 of x', i.e. under 2^-31 of the block
    maximum.  Checked over every positive bf16 pattern in [2^-24, 2^15) (the
    split is odd in x, and scaling by a power of two is exact)."""
    bits = np.arange(0x3380, 0x4700, dtype=np.uint32)  # bf16 patterns from 2^-24 up to 2^15
    xs = (bits << 16).view(np.float32).astype(np.float64)
    xs = xs[xs < 2.0 ** 15]
    t1 = _e5m2(xs)
    r1 = (xs.astype(np.float32) - t1.astype(np.float32)).astype(np.float64)
    t2 = _e5m2(r1)
    r2 = (r1.astype(np.float32) - t2.astype(np.float32)).astype(np.float64)
    t3 = _e5m2(r2)
    err = np.abs(t1 + t2 + t3 - xs)
    big = xs >= 2.0 ** -9
    assert np.all(err[big] == 0.0)
    assert np.all(err[~big] <= 2.0 ** -17)
    assert np.any(err[~big] > 0.0)  # the bound is reached: the floor is real


def test_fp32_splits_into_eight_e5m2_terms():
    """The decode step feeds h (fp32) to the tensor cores as eight e5m2 terms
    per value after a power-of-two scale that puts the block's largest
    magnitude in [2^14, 2^15): t_k = e5m2(h' - t_1 - ... - t_(k-1)), each
    difference taken in fp32 as the kernel does.  The terms sum exactly to h'
    for every fp32 value with h' >= 2^7 (within 2^8 of the block maximum),
    and to within 2^-17 of h' below that, i.e. under 2^-31 of the block
    maximum.  Checked on random fp32 mantissas at every exponent of the scaled
    range and below it."""
    rng = np.random.default_rng(5)
    mant = rng.integers(0, 1 << 23, size=4000, dtype=np.uint32)
    exps = np.arange(127 - 30, 127 + 15, dtype=np.uint32)  # 2^-30 .. 2^14
    bits = (exps[:, None] << 23) | mant[None, :]
    hs = bits.ravel().view(np.float32).astype(np.float64)
    r = hs.astype(np.float32)
    total = np.zeros_like(hs)
    for _ in range(8):
        t = _e5m2(r)
        total += t
        r = (r - t.astype(np.float32)).astype(np.float32)
    err = np.abs(total - hs)
    big = hs >= 2.0 ** 7
    assert np.all(err[big] == 0.0)
    assert np.all(err[~big] <= 2.0 ** -17)
