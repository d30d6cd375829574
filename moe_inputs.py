"""Seeded synthetic inputs for one top-k MoE FFN layer step.

This module is the one thing the CUDA path's tests/benchmark and the CPU
oracle share.  It draws the random tensors and stores them in the layer's
input formats; it computes nothing of the layer itself (no routing, no
GEMV, no activation, no blend).

Shapes and value distributions follow the workloads the reference pages
describe (Qwen3.6-35B-A3B blueprint page: 256 experts top-8 with a shared
expert, FP8 weights in 128x128 blocks; Qwen3.5-397B-A17B config page:
hidden 4096, 512 experts, 10 per token):

  x            bf16 [T, H]   ~ N(0, 1)
  router_w     bf16 [E, H]   ~ N(0, 0.02)
  shared_gate  bf16 [H]      ~ N(0, 0.02)
  router_bias  fp32 [E]      ~ N(0, 1)    (prefill workload only: uneven loads)
  expert e     W13 [2I, H] and W2 [H, I] drawn fp32 ~ N(0, 0.02), stored as
               e4m3 codes with one fp32 scale per 128x128 block
  shared       same with Is in place of I

Weight storage: one slab per expert, ``[W13 (2I x H) | W2 (H x I)]`` bytes,
row-major with the reduction dimension contiguous; scales ``[s13 (2I/128 x
H/128) | s2 (H/128 x I/128)]``.  The stored format is produced with
torch's own e4m3 conversion (a library cast, round-to-nearest-even) of
w / s with s = amax/448 per block; the oracle has its own, independent
quantiser, and a test checks that the two agree bit for bit.

NVFP4 experts (make_layer_nvfp4; the 397B-A17B checkpoint's expert format):
the same fp32 weights stored as e2m1 codes packed two to a byte (element 2j
in the low nibble of byte j), one e4m3 scale per 16 consecutive elements of
a row and one fp32 scale per matrix, through library casts (torch's e4m3,
ml_dtypes' e2m1, both round-to-nearest-even); the oracle has its own
quantiser, checked against these bytes.  Slab per expert: codes ``[W13 (2I x
H/2) | W2 (H x I/2)]``, scales ``[W13 (2I x H/16) | W2 (H x I/16)]``, tensor
scales ``[gs13, gs2]``.

Every tensor has its own generator, seeded from (seed, tensor name, index),
so any single expert can be regenerated alone; tests that only need the
experts a routing touches generate just those and leave the others zero.

bf16 tensors are returned as numpy uint16 bit patterns, codes as uint8,
scales and bias as float32.
"""
from __future__ import annotations

import hashlib
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class LayerDims:
    hidden: int        # H
    n_experts: int     # E
    top_k: int         # k
    inter: int         # I
    shared_inter: int  # Is

    @property
    def expert_bytes(self) -> int:
        return 3 * self.inter * self.hidden

    @property
    def expert_nscales(self) -> int:
        H, I = self.hidden, self.inter
        return (2 * I // 128) * (H // 128) + (H // 128) * (I // 128)

    @property
    def shared_bytes(self) -> int:
        return 3 * self.shared_inter * self.hidden

    @property
    def shared_nscales(self) -> int:
        H, I = self.hidden, self.shared_inter
        return (2 * I // 128) * (H // 128) + (H // 128) * (I // 128)


# Named workloads (dims, default row counts, router bias on/off).
TINY = LayerDims(hidden=256, n_experts=16, top_k=2, inter=128, shared_inter=128)
QWEN36_35B_A3B = LayerDims(hidden=2048, n_experts=256, top_k=8, inter=512, shared_inter=512)
QWEN35_397B_A17B = LayerDims(hidden=4096, n_experts=512, top_k=10, inter=1024, shared_inter=1024)

WORKLOADS = {
    "tiny": dict(dims=TINY, rows=[4], router_bias=False),
    "qwen3.6-35b-a3b-decode": dict(dims=QWEN36_35B_A3B, rows=[1], router_bias=False),
    "qwen3.6-35b-a3b-multiseq": dict(dims=QWEN36_35B_A3B, rows=[2, 8, 16, 32, 64], router_bias=False),
    "qwen3.5-397b-a17b-decode": dict(dims=QWEN35_397B_A17B, rows=[1, 32], router_bias=False),
    "qwen3.6-35b-a3b-prefill": dict(dims=QWEN36_35B_A3B, rows=[4096], router_bias=True),
}


def _seed(seed: int, name: str, index: int = 0) -> int:
    h = hashlib.sha256(f"{seed}/{name}/{index}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _normal(shape, std: float, seed: int, name: str, index: int = 0) -> torch.Tensor:
    g = torch.Generator().manual_seed(_seed(seed, name, index))
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def encode_e4m3_blocks(w: torch.Tensor):
    """Store an fp32 [R, C] matrix (R, C multiples of 128) as e4m3 codes with
    one fp32 scale per 128x128 block: s = amax/448 (1 for an all-zero block),
    codes = torch's e4m3 cast of w/s (quotient in fp32)."""
    R, C = w.shape
    b = w.reshape(R // 128, 128, C // 128, 128)
    amax = b.abs().amax(dim=(1, 3))
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    q = (b / s[:, None, :, None]).to(torch.float8_e4m3fn)
    return q.reshape(R, C).view(torch.uint8).numpy().copy(), s.numpy().copy()


def encode_nvfp4(w: torch.Tensor):
    """Store an fp32 [R, C] matrix (C a multiple of 16) as NVFP4: gs =
    amax/(448*6) (1 for an all-zero matrix); per 16 elements of a row, the
    scale code = torch's e4m3 cast of amax16/(6*gs); element codes =
    ml_dtypes' e2m1 cast of w/(e4m3(scale)*gs) (divisor and quotient in fp32;
    0 under a zero scale).  -> (packed codes uint8 [R, C/2], scale codes uint8
    [R, C/16], gs float)."""
    import ml_dtypes

    R, C = w.shape
    amax = float(w.abs().max())
    gs = np.float32(1.0) if amax == 0.0 else np.float32(amax) / np.float32(448.0 * 6.0)
    b = w.reshape(R, C // 16, 16)
    bmax = b.abs().amax(dim=2)
    sf = (bmax / torch.tensor(np.float32(6.0) * gs, dtype=torch.float32)).to(torch.float8_e4m3fn)
    div = sf.to(torch.float32) * torch.tensor(gs, dtype=torch.float32)
    q = torch.where(div[:, :, None] == 0, torch.zeros_like(b), b / div[:, :, None])
    codes = q.numpy().astype(ml_dtypes.float4_e2m1fn).view(np.uint8).reshape(R, C) & 0x0F
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed.copy(), sf.view(torch.uint8).numpy().copy(), float(gs)


def expert_slab(dims: LayerDims, seed: int, e: int, inter: int | None = None, name: str = "expert"):
    """(codes uint8 [3*I*H], scales fp32 [n]) for one expert (e = -1: shared)."""
    H = dims.hidden
    I = inter if inter is not None else dims.inter
    w13 = _normal((2 * I, H), 0.02, seed, name + ".w13", e)
    w2 = _normal((H, I), 0.02, seed, name + ".w2", e)
    q13, s13 = encode_e4m3_blocks(w13)
    q2, s2 = encode_e4m3_blocks(w2)
    return (np.concatenate([q13.reshape(-1), q2.reshape(-1)]),
            np.concatenate([s13.reshape(-1), s2.reshape(-1)]))


@dataclass
class Layer:
    dims: LayerDims
    seed: int
    router_w: np.ndarray       # uint16 [E, H]
    shared_gate: np.ndarray    # uint16 [H]
    expert_w8: np.ndarray      # uint8  [E, 3*I*H]
    expert_scales: np.ndarray  # fp32   [E, nscales]
    shared_w8: np.ndarray      # uint8  [3*Is*H]
    shared_scales: np.ndarray  # fp32   [nscales_shared]
    router_bias: np.ndarray | None = None   # fp32 [E]
    generated: frozenset = field(default_factory=frozenset)  # experts with drawn weights


def make_router(dims: LayerDims, seed: int, router_bias: bool = False):
    rw = _bf16_bits(_normal((dims.n_experts, dims.hidden), 0.02, seed, "router"))
    g = _bf16_bits(_normal((dims.hidden,), 0.02, seed, "shared_gate"))
    b = _normal((dims.n_experts,), 1.0, seed, "router_bias").numpy().copy() if router_bias else None
    return rw, g, b


def make_layer(dims: LayerDims, seed: int = 0, router_bias: bool = False, experts=None,
               threads: int | None = None) -> Layer:
    """All weights of one layer.  ``experts``: iterable of expert ids to draw
    (default: all); the rest are left as zero codes with unit scales."""
    rw, g, b = make_router(dims, seed, router_bias)
    E = dims.n_experts
    ids = list(range(E)) if experts is None else sorted(set(int(e) for e in experts))
    w8 = np.zeros((E, dims.expert_bytes), dtype=np.uint8)
    sc = np.ones((E, dims.expert_nscales), dtype=np.float32)

    def one(e):
        q, s = expert_slab(dims, seed, e)
        w8[e] = q
        sc[e] = s

    nthr = threads or min(32, os.cpu_count() or 1)
    if ids:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(one, ids))
    sq, ss = expert_slab(dims, seed, -1, inter=dims.shared_inter, name="shared")
    return Layer(dims, seed, rw, g, w8, sc, sq, ss, b, frozenset(ids))


def expert_slab_nvfp4(dims: LayerDims, seed: int, e: int, inter: int | None = None, name: str = "expert"):
    """(packed codes uint8 [3*I*H/2], scale codes uint8 [3*I*H/16], tensor
    scales fp32 [2]) for one expert (e = -1: shared): the same fp32 weights as
    expert_slab, stored as NVFP4."""
    H = dims.hidden
    I = inter if inter is not None else dims.inter
    w13 = _normal((2 * I, H), 0.02, seed, name + ".w13", e)
    w2 = _normal((H, I), 0.02, seed, name + ".w2", e)
    q13, f13, g13 = encode_nvfp4(w13)
    q2, f2, g2 = encode_nvfp4(w2)
    return (np.concatenate([q13.reshape(-1), q2.reshape(-1)]), np.concatenate([f13.reshape(-1), f2.reshape(-1)]),
            np.array([g13, g2], dtype=np.float32))


@dataclass
class LayerNvfp4:
    dims: LayerDims
    seed: int
    router_w: np.ndarray       # uint16 [E, H]
    shared_gate: np.ndarray    # uint16 [H]
    expert_w4: np.ndarray      # uint8  [E, 3*I*H/2]  packed e2m1 codes
    expert_sf: np.ndarray      # uint8  [E, 3*I*H/16] e4m3 scale codes
    expert_gs: np.ndarray      # fp32   [E, 2]
    shared_w4: np.ndarray      # uint8  [3*Is*H/2]
    shared_sf: np.ndarray      # uint8  [3*Is*H/16]
    shared_gs: np.ndarray      # fp32   [2]
    router_bias: np.ndarray | None = None
    generated: frozenset = field(default_factory=frozenset)


def make_layer_nvfp4(dims: LayerDims, seed: int = 0, router_bias: bool = False, experts=None,
                     threads: int | None = None) -> LayerNvfp4:
    """make_layer's weights stored as NVFP4 experts (the router, gate and
    bias are the same).  Experts not drawn are zero codes and scales with unit
    tensor scales."""
    rw, g, b = make_router(dims, seed, router_bias)
    E, H, I = dims.n_experts, dims.hidden, dims.inter
    ids = list(range(E)) if experts is None else sorted(set(int(e) for e in experts))
    w4 = np.zeros((E, 3 * I * H // 2), dtype=np.uint8)
    sf = np.zeros((E, 3 * I * H // 16), dtype=np.uint8)
    gs = np.ones((E, 2), dtype=np.float32)

    def one(e):
        w4[e], sf[e], gs[e] = expert_slab_nvfp4(dims, seed, e)

    nthr = threads or min(32, os.cpu_count() or 1)
    if ids:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(one, ids))
    sw, ssf, sgs = expert_slab_nvfp4(dims, seed, -1, inter=dims.shared_inter, name="shared")
    return LayerNvfp4(dims, seed, rw, g, w4, sf, gs, sw, ssf, sgs, b, frozenset(ids))


def make_x(dims: LayerDims, rows: int, seed: int = 0, stream: int = 0) -> np.ndarray:
    """Activation rows x, bf16 bits [rows, H], ~ N(0, 1); each (seed, stream)
    gives an independent batch."""
    return _bf16_bits(_normal((rows, dims.hidden), 1.0, seed, "x", stream))


def make_residual(dims: LayerDims, rows: int, seed: int = 0, stream: int = 0) -> np.ndarray:
    return _bf16_bits(_normal((rows, dims.hidden), 1.0, seed, "residual", stream))
