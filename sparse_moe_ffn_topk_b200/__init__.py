"""B200 (sm_100a) top-k mixture-of-experts FFN layer: Python binding.

A thin ctypes layer over ``libmoe_ffn_b200.so`` (the C ABI of
``include/moe_ffn.h``).  It only marshals torch tensors into pointers, sizes
and the current CUDA stream; every step of the layer runs in the library's
CUDA kernels.  There is no fallback: if the library is missing the import of
the first function raises.

    import sparse_moe_ffn_topk_b200 as moe
    dims = moe.MoeDims(hidden=2048, n_experts=256, top_k=8, inter=512, shared_inter=512)
    ws = moe.alloc_workspace(dims, max_rows=64)
    moe.ffn_forward(dims, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales,
                    shared_gate, out, ws)

Tensor formats: bf16 activations and router/gate weights as ``torch.bfloat16``
(or their int16/uint16 bit patterns), e4m3 weights as ``torch.uint8`` (or
``torch.float8_e4m3fn``), scales and bias as ``torch.float32``, top-k indices
as ``torch.int32``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_ffn_b200.so")

MOE_OK = 0
MOE_EINVAL = -1
MOE_EUNSUPPORTED = -2
MOE_EWORKSPACE = -3
MOE_ECUDA = -4
MOE_ETIMEOUT = -5

MOE_PATH_AUTO = 0
MOE_PATH_DECODE = 1
MOE_PATH_PREFILL = 2
MOE_PATH_PREFILL_NARROW = 3
MOE_DECODE_MAX_ROWS = 4
MOE_AUTO_DECODE_MAX_ROWS = 3
MOE_AUTO_NARROW_MAX_PAIRS = 32

EXPORTED = ("moe_workspace_bytes", "moe_workspace_init", "moe_router_topk", "moe_ffn_forward",
            "moe_ffn_forward_path", "moe_status", "moe_reset_status", "moe_status_string",
            "moe_debug_inject_fault", "moe_kernel_launches", "moe_auto_path", "moe_ffn_forward_timed",
            "moe_device_status", "moe_debug_wait_timeout", "moe_ffn_forward_static",
            "moe_static_scratch_bytes", "moe_static_device_status", "moe_debug_wait_timeout_static",
            "moe_ffn_forward_norm", "moe_ffn_forward_host", "moe_ffn_forward_nvfp4")


class MoeNvfp4Expert(ctypes.Structure):
    _fields_ = [("w4", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("gs", ctypes.c_void_p)]


class MoeDims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("shared_inter", ctypes.c_int32)]

    def __repr__(self):
        return (f"MoeDims(hidden={self.hidden}, n_experts={self.n_experts}, top_k={self.top_k}, "
                f"inter={self.inter}, shared_inter={self.shared_inter})")


class MoeFp8Expert(ctypes.Structure):
    _fields_ = [("w8", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_moe_ffn_topk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32 = ctypes.c_void_p, ctypes.c_int32
        DP = ctypes.POINTER(MoeDims)
        L.moe_workspace_bytes.argtypes = [DP, I32]
        L.moe_workspace_bytes.restype = ctypes.c_size_t
        L.moe_workspace_init.argtypes = [P, ctypes.c_size_t, P]
        L.moe_router_topk.argtypes = [DP, P, I32, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_ffn_forward.argtypes = [DP, P, I32, P, P, P, ctypes.POINTER(MoeFp8Expert), P, P, P, P, P,
                                      ctypes.c_size_t, P]
        L.moe_ffn_forward_path.argtypes = [DP, P, I32, P, P, P, ctypes.POINTER(MoeFp8Expert), P, P, P, P,
                                           P, ctypes.c_size_t, P, I32, P, P, P]
        L.moe_ffn_forward_norm.argtypes = [DP, P, I32, P, ctypes.c_float, P, P, P, ctypes.POINTER(MoeFp8Expert), P,
                                           P, P, P, ctypes.c_size_t, P, I32]
        L.moe_ffn_forward_host.argtypes = [DP, P, I32, P, P, P, ctypes.POINTER(MoeFp8Expert), P, P, P, P,
                                           ctypes.c_size_t, P]
        L.moe_ffn_forward_nvfp4.argtypes = [DP, P, I32, P, P, P, P, ctypes.POINTER(MoeNvfp4Expert), P, P, P, P, P,
                                            ctypes.c_size_t, P]
        L.moe_kernel_launches.argtypes = [DP, I32, I32]
        L.moe_kernel_launches.restype = I32
        L.moe_auto_path.argtypes = [DP, I32]
        L.moe_auto_path.restype = I32
        L.moe_ffn_forward_timed.argtypes = [DP, P, I32, P, P, P, ctypes.POINTER(MoeFp8Expert), P, P, P, P,
                                            P, ctypes.c_size_t, P, I32, ctypes.POINTER(ctypes.c_void_p), I32]
        L.moe_device_status.argtypes = [P, ctypes.c_size_t, P]
        L.moe_debug_wait_timeout.argtypes = [P, ctypes.c_size_t, I32, P]
        L.moe_ffn_forward_static.argtypes = [DP, P, I32, P, P, P, ctypes.POINTER(MoeFp8Expert), P, P, P, P, P]
        L.moe_static_scratch_bytes.argtypes = []
        L.moe_static_scratch_bytes.restype = ctypes.c_size_t
        L.moe_static_device_status.argtypes = [P]
        L.moe_debug_wait_timeout_static.argtypes = [I32, P]
        L.moe_status.argtypes = []
        L.moe_reset_status.argtypes = []
        L.moe_reset_status.restype = None
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_debug_inject_fault.argtypes = [I32]
        L.moe_debug_inject_fault.restype = None
        _lib = L
    return _lib


# --------------------------------------------------------------- marshalling

def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _rows(x) -> int:
    return int(x.shape[0]) if x.dim() > 1 else 1


def _check(rc: int, what: str):
    if rc != MOE_OK:
        raise MoeError(rc, what)


def _dims(d) -> MoeDims:
    if isinstance(d, MoeDims):
        return d
    return MoeDims(d.hidden, d.n_experts, d.top_k, d.inter, d.shared_inter)


# ------------------------------------------------------------------ the API

def workspace_bytes(dims, max_rows: int) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(_dims(dims)), int(max_rows)))


def workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def alloc_workspace(dims, max_rows: int, device=None) -> torch.Tensor:
    """A zero-filled workspace for calls with rows <= max_rows."""
    n = workspace_bytes(dims, max_rows)
    if n == 0:
        raise MoeError(MOE_EUNSUPPORTED, "moe_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def router_topk(dims, x, router_w, shared_gate, topk_idx, topk_w, shared_gate_sig, ws,
                router_bias=None, stream=None):
    d = _dims(dims)
    _check(lib().moe_router_topk(ctypes.byref(d), _ptr(x), _rows(x), _ptr(router_w), _ptr(router_bias),
                                 _ptr(shared_gate), _ptr(topk_idx), _ptr(topk_w), _ptr(shared_gate_sig),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_router_topk")


def ffn_forward(dims, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                out, ws, residual=None, router_bias=None, stream=None):
    d = _dims(dims)
    sh = MoeFp8Expert(_ptr(shared_w8), _ptr(shared_scales))
    _check(lib().moe_ffn_forward(ctypes.byref(d), _ptr(x), _rows(x), _ptr(router_w), _ptr(expert_w8),
                                 _ptr(expert_scales), ctypes.byref(sh), _ptr(shared_gate), _ptr(out),
                                 _ptr(residual), _ptr(router_bias), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)),
           "moe_ffn_forward")


def ffn_forward_path(dims, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                     out, ws, path=MOE_PATH_AUTO, residual=None, router_bias=None, topk_idx=None,
                     topk_w=None, shared_gate_sig=None, stream=None):
    d = _dims(dims)
    sh = MoeFp8Expert(_ptr(shared_w8), _ptr(shared_scales))
    _check(lib().moe_ffn_forward_path(ctypes.byref(d), _ptr(x), _rows(x), _ptr(router_w), _ptr(expert_w8),
                                      _ptr(expert_scales), ctypes.byref(sh), _ptr(shared_gate), _ptr(out),
                                      _ptr(residual), _ptr(router_bias), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream), int(path),
                                      _ptr(topk_idx), _ptr(topk_w), _ptr(shared_gate_sig)),
           "moe_ffn_forward_path")


def ffn_forward_host(dims, x_host, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                     out_host, ws, router_bias=None, stream=None):
    """ffn_forward with x_host and out_host pinned CPU tensors (bf16 [rows, H]):
    the GPU reads x and writes out over the host link; out_host is complete
    once the stream has passed the call."""
    d = _dims(dims)
    sh = MoeFp8Expert(_ptr(shared_w8), _ptr(shared_scales))
    _check(lib().moe_ffn_forward_host(ctypes.byref(d), _ptr(x_host), _rows(x_host), _ptr(router_w),
                                      _ptr(expert_w8), _ptr(expert_scales), ctypes.byref(sh), _ptr(shared_gate),
                                      _ptr(out_host), _ptr(router_bias), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
           "moe_ffn_forward_host")


def ffn_forward_nvfp4(dims, x, router_w, expert_w4, expert_sf, expert_gs, shared_w4, shared_sf, shared_gs,
                      shared_gate, out, ws, residual=None, router_bias=None, stream=None):
    """The layer with NVFP4 experts (packed e2m1 codes, e4m3 block scales per 16
    elements, fp32 tensor scales [E, 2]); device tensors in moe_inputs' slab
    layout."""
    d = _dims(dims)
    sh = MoeNvfp4Expert(_ptr(shared_w4), _ptr(shared_sf), _ptr(shared_gs))
    _check(lib().moe_ffn_forward_nvfp4(ctypes.byref(d), _ptr(x), _rows(x), _ptr(router_w), _ptr(expert_w4),
                                       _ptr(expert_sf), _ptr(expert_gs), ctypes.byref(sh), _ptr(shared_gate),
                                       _ptr(out), _ptr(residual), _ptr(router_bias), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)),
           "moe_ffn_forward_nvfp4")


def ffn_forward_norm(dims, resid, norm_w, eps, router_w, expert_w8, expert_scales, shared_w8, shared_scales,
                     shared_gate, out, ws, router_bias=None, path=MOE_PATH_AUTO, stream=None):
    """out = resid + layer(bf16(rmsnorm(resid) * norm_w)); out may be resid."""
    d = _dims(dims)
    sh = MoeFp8Expert(_ptr(shared_w8), _ptr(shared_scales))
    _check(lib().moe_ffn_forward_norm(ctypes.byref(d), _ptr(resid), _rows(resid), _ptr(norm_w), float(eps),
                                      _ptr(router_w), _ptr(expert_w8), _ptr(expert_scales), ctypes.byref(sh),
                                      _ptr(shared_gate), _ptr(out), _ptr(router_bias), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream), int(path)),
           "moe_ffn_forward_norm")


def kernel_launches(dims, rows: int, path=MOE_PATH_AUTO) -> int:
    return int(lib().moe_kernel_launches(ctypes.byref(_dims(dims)), int(rows), int(path)))


def auto_path(dims, rows: int) -> int:
    """The MOE_PATH_* that MOE_PATH_AUTO takes for these dims and rows."""
    return int(lib().moe_auto_path(ctypes.byref(_dims(dims)), int(rows)))


def ffn_forward_timed(dims, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                      out, ws, events, path=MOE_PATH_AUTO, residual=None, router_bias=None, stream=None):
    """Forward that records ``events`` (torch.cuda.Event(enable_timing=True), at least
    kernel_launches()+1 of them) around each kernel it launches."""
    d = _dims(dims)
    sh = MoeFp8Expert(_ptr(shared_w8), _ptr(shared_scales))
    for e in events:
        if not e.cuda_event:  # torch creates an event's handle on its first record
            e.record(stream if stream is not None else torch.cuda.current_stream())
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().moe_ffn_forward_timed(ctypes.byref(d), _ptr(x), _rows(x), _ptr(router_w), _ptr(expert_w8),
                                       _ptr(expert_scales), ctypes.byref(sh), _ptr(shared_gate), _ptr(out),
                                       _ptr(residual), _ptr(router_bias), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream), int(path), arr,
                                       len(events)),
           "moe_ffn_forward_timed")


def device_status(ws, stream=None) -> int:
    """Synchronises the stream and returns the workspace's device status word."""
    return int(lib().moe_device_status(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def debug_wait_timeout(ws, limit_us: int, stream=None):
    _check(lib().moe_debug_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), int(limit_us),
                                        _stream(stream)), "moe_debug_wait_timeout")


def ffn_forward_static(dims, x, router_w, expert_w8, expert_scales, shared_w8, shared_scales, shared_gate,
                       out, residual=None, router_bias=None, stream=None):
    """ffn_forward without a workspace: uses the library's built-in scratch
    array (static_scratch_bytes() large); allocates nothing.  Calls that would
    overlap on the GPU must not be issued (they share the array)."""
    d = _dims(dims)
    sh = MoeFp8Expert(_ptr(shared_w8), _ptr(shared_scales))
    _check(lib().moe_ffn_forward_static(ctypes.byref(d), _ptr(x), _rows(x), _ptr(router_w), _ptr(expert_w8),
                                        _ptr(expert_scales), ctypes.byref(sh), _ptr(shared_gate), _ptr(out),
                                        _ptr(residual), _ptr(router_bias), _stream(stream)),
           "moe_ffn_forward_static")


def static_scratch_bytes() -> int:
    return int(lib().moe_static_scratch_bytes())


def static_device_status(stream=None) -> int:
    """Synchronises the stream and returns (then clears, if set) the status
    word of the scratch array that ffn_forward_static uses."""
    return int(lib().moe_static_device_status(_stream(stream)))


def debug_wait_timeout_static(limit_us: int, stream=None):
    _check(lib().moe_debug_wait_timeout_static(int(limit_us), _stream(stream)),
           "moe_debug_wait_timeout_static")


def status() -> int:
    return int(lib().moe_status())


def reset_status():
    lib().moe_reset_status()


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def debug_inject_fault(n: int):
    lib().moe_debug_inject_fault(int(n))


class MoeLayer:
    """Device-resident weights of one layer plus a workspace: ``layer(x) -> out``.

    ``weights`` holds torch tensors (any device; moved to ``device``):
    router_w [E, H] bf16, shared_gate [H] bf16, expert_w8 [E, 3IH] uint8,
    expert_scales [E, n] fp32, shared_w8 [3IsH] uint8, shared_scales [n'] fp32,
    and optionally router_bias [E] fp32.
    """

    def __init__(self, dims, weights: dict, max_rows: int = 64, device="cuda"):
        self.dims = _dims(dims)
        self.device = torch.device(device)
        self.w = {k: (v.to(self.device).contiguous() if v is not None else None) for k, v in weights.items()}
        self.w.setdefault("router_bias", None)
        self.max_rows = int(max_rows)
        self.ws = alloc_workspace(self.dims, self.max_rows, device=self.device)

    def ensure_rows(self, rows: int):
        if rows > self.max_rows:
            self.max_rows = int(rows)
            self.ws = alloc_workspace(self.dims, self.max_rows, device=self.device)

    def __call__(self, x, out=None, residual=None, path=MOE_PATH_AUTO, stream=None):
        self.ensure_rows(_rows(x))
        if out is None:
            out = torch.empty((_rows(x), self.dims.hidden), dtype=torch.bfloat16, device=self.device)
        w = self.w
        ffn_forward_path(self.dims, x, w["router_w"], w["expert_w8"], w["expert_scales"], w["shared_w8"],
                         w["shared_scales"], w["shared_gate"], out, self.ws, path=path, residual=residual,
                         router_bias=w["router_bias"], stream=stream)
        return out
