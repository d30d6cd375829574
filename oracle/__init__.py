"""CPU oracle of one top-k MoE FFN layer step (double precision, plain C).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by the CPU-baseline leg of ``bench.py``.  The product package never
imports it.  This wrapper only marshals numpy arrays into the C library
``moe_oracle.c``; all arithmetic lives there.

Arrays use these dtypes: bf16 values are passed as their uint16 bit patterns,
e4m3 codes as uint8, scales as float32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_moe.so")


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` into ``liboracle_moe.so`` beside it (gcc -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("shared_inter", ctypes.c_int32)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_quantize_blocks.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, P]
        lib.oracle_topk.argtypes = [P, ctypes.c_int32, ctypes.c_int32, P, P]
        lib.oracle_router_topk.argtypes = [ctypes.POINTER(_Dims), P, ctypes.c_int32, P, P, P, P, P, P, P]
        lib.oracle_expert_ffn.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, P, P]
        lib.oracle_moe_forward.argtypes = [ctypes.POINTER(_Dims), P, ctypes.c_int32, P, P, P, P, P,
                                           P, P, P, P, P, P, P, P, P, ctypes.c_int32]
        lib.oracle_rmsnorm.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_double, P, P]
        lib.oracle_moe_forward_dense.argtypes = [ctypes.POINTER(_Dims), P, ctypes.c_int32, P, P,
                                                 P, P, P, P, P, P, P, P, P, P, ctypes.c_int32]
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_double]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_quantize_nvfp4.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, P, P]
        lib.oracle_expert_ffn_nvfp4.argtypes = [P, P, P, ctypes.c_int32, ctypes.c_int32, P, P]
        lib.oracle_moe_forward_nvfp4.argtypes = [ctypes.POINTER(_Dims), P, ctypes.c_int32, P, P, P, P, P, P, P,
                                                 P, P, P, P, ctypes.c_int32, P, P, P, P, P, ctypes.c_int32]
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with status {rc}")


# ---------------------------------------------------------------- scalars

def bf16_to_f64(bits: int) -> float:
    return _load().oracle_bf16_to_f64(int(bits))


def f64_to_bf16(v: float) -> int:
    return int(_load().oracle_f64_to_bf16(float(v)))


def e4m3_decode(code: int) -> float:
    return _load().oracle_e4m3_decode(int(code))


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return _load().oracle_e2m1_decode(int(code))


def e2m1_encode(v: float) -> int:
    return int(_load().oracle_e2m1_encode(float(v)))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Element-wise nearest bf16 (ties to even) of a float64 array, as uint16 bits."""
    f = np.vectorize(lambda v: _load().oracle_f64_to_bf16(float(v)), otypes=[np.uint16])
    return f(np.asarray(a, dtype=np.float64))


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    f = np.vectorize(lambda b: _load().oracle_bf16_to_f64(int(b)), otypes=[np.float64])
    return f(np.asarray(a, dtype=np.uint16))


# ---------------------------------------------------------------- arrays

def quantize_blocks(w: np.ndarray):
    """Oracle block quantiser: fp32 [R, C] -> (e4m3 codes uint8 [R, C], fp32 scales [R/128, C/128])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    R, C = w.shape
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty((R // 128, C // 128), dtype=np.float32)
    _check(_load().oracle_quantize_blocks(_ptr(w), R, C, _ptr(q), _ptr(s)), "oracle_quantize_blocks")
    return q, s


def quantize_nvfp4(w: np.ndarray):
    """Oracle NVFP4 quantiser: fp32 [R, C] (C a multiple of 16) -> (packed e2m1
    codes uint8 [R, C/2] (element 2j in the low nibble of byte j), e4m3 block
    scale codes uint8 [R, C/16], fp32 tensor scale)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    R, C = w.shape
    q = np.zeros((R, C // 2), dtype=np.uint8)
    sf = np.empty((R, C // 16), dtype=np.uint8)
    gs = np.empty(1, dtype=np.float32)
    _check(_load().oracle_quantize_nvfp4(_ptr(w), R, C, _ptr(q), _ptr(sf), _ptr(gs)), "oracle_quantize_nvfp4")
    return q, sf, float(gs[0])


def expert_ffn_nvfp4(w4, sf, gs, H: int, I: int, x: np.ndarray) -> np.ndarray:
    """One SwiGLU expert with NVFP4 weights (slab layout of moe_inputs), x float64 [H] -> y [H]."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(H, dtype=np.float64)
    _check(_load().oracle_expert_ffn_nvfp4(_ptr(np.ascontiguousarray(w4, dtype=np.uint8)),
                                           _ptr(np.ascontiguousarray(sf, dtype=np.uint8)),
                                           _ptr(np.ascontiguousarray(gs, dtype=np.float32)), H, I, _ptr(x),
                                           _ptr(y)), "oracle_expert_ffn_nvfp4")
    return y


def moe_forward_nvfp4(d, x, router_w, expert_w4, expert_sf, expert_gs, shared_w4, shared_sf, shared_gs,
                      shared_gate, residual=None, router_bias=None, forced_idx=None, dense=False,
                      want_logits=True, nthreads: int | None = None) -> ForwardResult:
    """The layer with NVFP4 experts in double (routed; or, dense=True, every
    expert under the top-k mask)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows = x.shape[0]
    out = np.empty((rows, d.hidden), dtype=np.float64)
    idx = np.empty((rows, d.top_k), dtype=np.int32)
    w = np.empty((rows, d.top_k), dtype=np.float64)
    gs = np.empty(rows, dtype=np.float64)
    logits = np.empty((rows, d.n_experts), dtype=np.float64) if (want_logits and not dense) else None
    if forced_idx is not None:
        forced_idx = np.ascontiguousarray(forced_idx, dtype=np.int32)
    dims = _dims(d)
    rc = _load().oracle_moe_forward_nvfp4(
        ctypes.byref(dims), _ptr(x), rows, _ptr(np.ascontiguousarray(router_w, dtype=np.uint16)),
        _ptr(np.ascontiguousarray(expert_w4, dtype=np.uint8)), _ptr(np.ascontiguousarray(expert_sf, dtype=np.uint8)),
        _ptr(np.ascontiguousarray(expert_gs, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_w4, dtype=np.uint8)), _ptr(np.ascontiguousarray(shared_sf, dtype=np.uint8)),
        _ptr(np.ascontiguousarray(shared_gs, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_gate, dtype=np.uint16)),
        _ptr(None if residual is None else np.ascontiguousarray(residual, dtype=np.uint16)),
        _ptr(None if router_bias is None else np.ascontiguousarray(router_bias, dtype=np.float32)),
        _ptr(forced_idx), 1 if dense else 0, _ptr(out), _ptr(idx), _ptr(w), _ptr(gs), _ptr(logits),
        nthreads or os.cpu_count() or 1)
    _check(rc, "oracle_moe_forward_nvfp4")
    return ForwardResult(out, idx, w, gs, logits)


def topk(logits: np.ndarray, k: int):
    """Top-k of one row of logits (float64 [E]) -> (idx int32 [k], w float64 [k])."""
    l = np.ascontiguousarray(logits, dtype=np.float64)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    _check(_load().oracle_topk(_ptr(l), l.shape[0], k, _ptr(idx), _ptr(w)), "oracle_topk")
    return idx, w


def router_topk(d, x, router_w, shared_gate, router_bias=None):
    """Router step alone -> (logits float64 [rows, E], idx int32 [rows, k], w float64 [rows, k],
    gate_sig float64 [rows])."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows = x.shape[0]
    logits = np.empty((rows, d.n_experts), dtype=np.float64)
    idx = np.empty((rows, d.top_k), dtype=np.int32)
    w = np.empty((rows, d.top_k), dtype=np.float64)
    gs = np.empty(rows, dtype=np.float64)
    dims = _dims(d)
    _check(_load().oracle_router_topk(
        ctypes.byref(dims), _ptr(x), rows, _ptr(np.ascontiguousarray(router_w, dtype=np.uint16)),
        _ptr(None if router_bias is None else np.ascontiguousarray(router_bias, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_gate, dtype=np.uint16)), _ptr(logits), _ptr(idx), _ptr(w),
        _ptr(gs)), "oracle_router_topk")
    return logits, idx, w, gs


def expert_ffn(w8: np.ndarray, scales: np.ndarray, H: int, I: int, x: np.ndarray) -> np.ndarray:
    """One SwiGLU expert on one row x (float64 [H]) from its e4m3 slab and block scales."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(H, dtype=np.float64)
    _check(_load().oracle_expert_ffn(_ptr(np.ascontiguousarray(w8, dtype=np.uint8)),
                                     _ptr(np.ascontiguousarray(scales, dtype=np.float32)),
                                     H, I, _ptr(x), _ptr(y)), "oracle_expert_ffn")
    return y


def rmsnorm(resid: np.ndarray, norm_w: np.ndarray, eps: float):
    """RMSNorm of each row of the residual stream (bf16 bits [rows, H]) times
    the norm weight (bf16 bits [H]) -> (x float64 [rows, H] before rounding,
    x as bf16 bits)."""
    r = np.ascontiguousarray(resid, dtype=np.uint16)
    rows, H = r.shape
    xd = np.empty((rows, H), dtype=np.float64)
    xb = np.empty((rows, H), dtype=np.uint16)
    _check(_load().oracle_rmsnorm(H, rows, _ptr(r), _ptr(np.ascontiguousarray(norm_w, dtype=np.uint16)),
                                  float(eps), _ptr(xd), _ptr(xb)), "oracle_rmsnorm")
    return xd, xb


def moe_forward_norm(d, resid, norm_w, eps, router_w, expert_w8, expert_scales, shared_w8, shared_scales,
                     shared_gate, router_bias=None, forced_idx=None, want_logits=True,
                     nthreads: int | None = None) -> ForwardResult:
    """The layer behind its RMSNorm: x = bf16(rmsnorm(resid) * norm_w), out =
    resid + layer(x), in double before the output rounding."""
    _, xb = rmsnorm(resid, norm_w, eps)
    return moe_forward(d, xb, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                       residual=resid, router_bias=router_bias, forced_idx=forced_idx, want_logits=want_logits,
                       nthreads=nthreads)


@dataclass
class ForwardResult:
    out: np.ndarray        # float64 [rows, H], before rounding to bf16
    idx: np.ndarray        # int32 [rows, k], rank order
    w: np.ndarray          # float64 [rows, k]
    gate_sig: np.ndarray   # float64 [rows]
    logits: np.ndarray | None  # float64 [rows, E]


def _dims(d) -> _Dims:
    return _Dims(d.hidden, d.n_experts, d.top_k, d.inter, d.shared_inter)


def moe_forward(d, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                residual=None, router_bias=None, forced_idx=None, want_logits=True,
                nthreads: int | None = None) -> ForwardResult:
    """Routed layer output in double.  ``d`` has hidden/n_experts/top_k/inter/shared_inter."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows = x.shape[0]
    out = np.empty((rows, d.hidden), dtype=np.float64)
    idx = np.empty((rows, d.top_k), dtype=np.int32)
    w = np.empty((rows, d.top_k), dtype=np.float64)
    gs = np.empty(rows, dtype=np.float64)
    logits = np.empty((rows, d.n_experts), dtype=np.float64) if want_logits else None
    if forced_idx is not None:
        forced_idx = np.ascontiguousarray(forced_idx, dtype=np.int32)
    dims = _dims(d)
    rc = _load().oracle_moe_forward(
        ctypes.byref(dims), _ptr(x), rows, _ptr(np.ascontiguousarray(router_w, dtype=np.uint16)),
        _ptr(np.ascontiguousarray(expert_w8, dtype=np.uint8)),
        _ptr(np.ascontiguousarray(expert_scales, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_w8, dtype=np.uint8)),
        _ptr(np.ascontiguousarray(shared_scales, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_gate, dtype=np.uint16)),
        _ptr(None if residual is None else np.ascontiguousarray(residual, dtype=np.uint16)),
        _ptr(None if router_bias is None else np.ascontiguousarray(router_bias, dtype=np.float32)),
        _ptr(forced_idx), _ptr(out), _ptr(idx), _ptr(w), _ptr(gs), _ptr(logits),
        nthreads or os.cpu_count() or 1)
    _check(rc, "oracle_moe_forward")
    return ForwardResult(out, idx, w, gs, logits)


def moe_forward_dense(d, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales,
                      shared_gate, residual=None, router_bias=None,
                      nthreads: int | None = None) -> ForwardResult:
    """Same layer by brute force over all experts with the top-k mask."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows = x.shape[0]
    out = np.empty((rows, d.hidden), dtype=np.float64)
    idx = np.empty((rows, d.top_k), dtype=np.int32)
    w = np.empty((rows, d.top_k), dtype=np.float64)
    gs = np.empty(rows, dtype=np.float64)
    dims = _dims(d)
    rc = _load().oracle_moe_forward_dense(
        ctypes.byref(dims), _ptr(x), rows, _ptr(np.ascontiguousarray(router_w, dtype=np.uint16)),
        _ptr(np.ascontiguousarray(expert_w8, dtype=np.uint8)),
        _ptr(np.ascontiguousarray(expert_scales, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_w8, dtype=np.uint8)),
        _ptr(np.ascontiguousarray(shared_scales, dtype=np.float32)),
        _ptr(np.ascontiguousarray(shared_gate, dtype=np.uint16)),
        _ptr(None if residual is None else np.ascontiguousarray(residual, dtype=np.uint16)),
        _ptr(None if router_bias is None else np.ascontiguousarray(router_bias, dtype=np.float32)),
        _ptr(out), _ptr(idx), _ptr(w), _ptr(gs), nthreads or os.cpu_count() or 1)
    _check(rc, "oracle_moe_forward_dense")
    return ForwardResult(out, idx, w, gs, None)
