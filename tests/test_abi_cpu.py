"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol ``include/*.h`` declares, and its host-side checks (dims, nulls,
alignment, workspace size, the fault knob) answer without touching CUDA."""
import ctypes
import glob
import os
import re

import pytest

import moe_inputs as mi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

moe = pytest.importorskip("sparse_moe_ffn_topk_b200")


@pytest.fixture(scope="module")
def L():
    from sparse_moe_ffn_topk_b200 import build
    build.build()
    return moe.lib()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert names, "no declarations found"
    assert names == set(moe.EXPORTED) | (names - set(moe.EXPORTED))
    for n in names:
        assert hasattr(L, n), n


def test_binding_constants_match_header():
    src = open(os.path.join(ROOT, "include", "moe_ffn.h")).read()
    defs = dict(re.findall(r"#define\s+(MOE_[A-Z0-9_]+)\s+(-?\d+)", src))
    assert len(defs) >= 12
    for name, value in defs.items():
        assert getattr(moe, name) == int(value), name


def test_binding_names_match_header():
    assert set(moe.EXPORTED) == declared_symbols()


def D(h=2048, e=256, k=8, i=512, s=512):
    return moe.MoeDims(h, e, k, i, s)


def test_workspace_bytes(L):
    d = D()
    a = moe.workspace_bytes(d, 1)
    b = moe.workspace_bytes(d, 64)
    assert 0 < a < b
    assert moe.workspace_bytes(D(h=2000), 1) == 0          # not a multiple of 128
    assert moe.workspace_bytes(D(k=33, e=64), 1) == 0      # k > 32
    assert moe.workspace_bytes(D(k=9, e=8), 1) == 0        # k > E
    assert moe.workspace_bytes(D(e=1025), 1) == 0          # E > 1024
    assert moe.workspace_bytes(d, -1) == 0


FAKE = 1 << 20  # an aligned, never dereferenced address


def fwd(L, d, rows=1, x=FAKE, out=FAKE + 4096, ws=FAKE, ws_bytes=None, shared=True, path=0):
    sh = moe.MoeFp8Expert(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE)) if shared else None
    if ws_bytes is None:
        ws_bytes = moe.workspace_bytes(d, max(rows, 1))
    P = lambda a: ctypes.c_void_p(a) if a else None
    return L.moe_ffn_forward_path(ctypes.byref(d), P(x), rows, P(FAKE), P(FAKE), P(FAKE),
                                  ctypes.byref(sh) if sh else None, P(FAKE), P(out), None, None, P(ws),
                                  ws_bytes, None, path, None, None, None)


def test_argument_checks_on_host(L):
    d = D()
    assert fwd(L, d, x=0) == moe.MOE_EINVAL
    assert fwd(L, d, x=FAKE + 2) == moe.MOE_EINVAL          # misaligned
    assert fwd(L, d, shared=False) == moe.MOE_EINVAL
    assert fwd(L, d, rows=-1) == moe.MOE_EINVAL
    assert fwd(L, d, path=7) == moe.MOE_EINVAL
    assert fwd(L, d, out=FAKE) == moe.MOE_EINVAL            # out aliases x
    assert fwd(L, D(i=500)) == moe.MOE_EUNSUPPORTED
    assert fwd(L, d, ws_bytes=16) == moe.MOE_EWORKSPACE
    assert fwd(L, d, rows=0) == moe.MOE_OK                   # no-op, no CUDA call
    assert fwd(L, d, rows=0, x=0, out=0, ws=0) == moe.MOE_OK  # empty tensors have null pointers
    assert L.moe_router_topk(ctypes.byref(d), None, 1, None, None, None, None, None, None, None, 0,
                             None) == moe.MOE_EINVAL


def test_paths_and_launch_counts(L):
    d = D()
    assert moe.kernel_launches(d, 0) == 0
    assert moe.kernel_launches(d, moe.MOE_AUTO_DECODE_MAX_ROWS) == 1     # one decode-step kernel
    assert moe.kernel_launches(d, moe.MOE_AUTO_DECODE_MAX_ROWS + 1) == 6
    for path, n in ((moe.MOE_PATH_DECODE, 2), (moe.MOE_PATH_PREFILL, 6), (moe.MOE_PATH_PREFILL_NARROW, 6)):
        assert moe.kernel_launches(d, 5, path) == n                        # decode: 4 rows per launch
    assert moe.kernel_launches(d, 64, moe.MOE_PATH_DECODE) == 64 // moe.MOE_DECODE_MAX_ROWS
    assert moe.kernel_launches(d, 5, 4) == 0                  # no such path
    assert moe.auto_path(d, 1) == moe.MOE_PATH_DECODE
    assert moe.auto_path(d, moe.MOE_AUTO_DECODE_MAX_ROWS + 1) == moe.MOE_PATH_PREFILL_NARROW
    narrow_max = moe.MOE_AUTO_NARROW_MAX_PAIRS * 256 // 8          # rows * k <= pairs * E
    assert moe.auto_path(d, narrow_max) == moe.MOE_PATH_PREFILL_NARROW
    assert moe.auto_path(d, narrow_max + 1) == moe.MOE_PATH_PREFILL
    assert moe.auto_path(D(h=8192), 64) == moe.MOE_PATH_PREFILL  # beyond the narrow GEMMs' K
    assert moe.auto_path(d, 4096) == moe.MOE_PATH_PREFILL
    assert moe.auto_path(d, -1) == moe.MOE_EINVAL
    # the narrow GEMMs hold at most 64 K blocks of scales per item: refused
    # on the host before any device call
    assert fwd(L, D(h=8320), path=moe.MOE_PATH_PREFILL_NARROW) == moe.MOE_EUNSUPPORTED
    assert fwd(L, D(i=8320), path=moe.MOE_PATH_PREFILL_NARROW) == moe.MOE_EUNSUPPORTED


def test_fault_knob_is_sticky_until_reset(L):
    d = D()
    moe.reset_status()
    moe.debug_inject_fault(2)
    assert fwd(L, d, rows=0) == moe.MOE_OK        # first call passes (a no-op)
    assert fwd(L, d, rows=0) == moe.MOE_ECUDA     # second call: the injected loss
    assert moe.status() == moe.MOE_ECUDA
    assert fwd(L, d, rows=0) == moe.MOE_ECUDA     # sticky
    moe.reset_status()
    assert moe.status() == moe.MOE_OK
    assert fwd(L, d, rows=0) == moe.MOE_OK


def test_status_strings(L):
    for c in (0, -1, -2, -3, -4, -99):
        assert isinstance(moe.status_string(c), str) and moe.status_string(c)


def test_dims_match_input_generator():
    for d in (mi.TINY, mi.QWEN36_35B_A3B, mi.QWEN35_397B_A17B):
        assert moe.workspace_bytes(d, 1) > 0


# ------------------------------------------------------------ the static entry

def static_fwd(L, d, rows=1, x=FAKE, out=FAKE + 4096, shared=True):
    sh = moe.MoeFp8Expert(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE)) if shared else None
    P = lambda a: ctypes.c_void_p(a) if a else None
    return L.moe_ffn_forward_static(ctypes.byref(d) if d is not None else None, P(x), rows, P(FAKE), P(FAKE),
                                    P(FAKE), ctypes.byref(sh) if sh else None, P(FAKE), P(out), None, None,
                                    None)


def test_static_scratch_size_matches_header(L):
    src = open(os.path.join(ROOT, "include", "moe_ffn.h")).read()
    assert "16 MiB" in src
    assert moe.static_scratch_bytes() == 16 << 20


def test_static_entry_rejects_on_host_before_any_device_call(L):
    """Every rejection below returns before the scratch address is looked up
    or anything is enqueued (this machine has no GPU: a device call would
    fail with MOE_ECUDA instead)."""
    moe.reset_status()
    d = D()
    assert static_fwd(L, None) == moe.MOE_EINVAL                   # null dims
    assert static_fwd(L, d, rows=-1) == moe.MOE_EINVAL
    assert static_fwd(L, d, x=0) == moe.MOE_EINVAL
    assert static_fwd(L, d, x=FAKE + 8) == moe.MOE_EINVAL          # misaligned
    assert static_fwd(L, d, shared=False) == moe.MOE_EINVAL
    assert static_fwd(L, d, out=FAKE) == moe.MOE_EINVAL            # out aliases x
    assert static_fwd(L, D(i=500)) == moe.MOE_EUNSUPPORTED
    assert static_fwd(L, d, rows=0) == moe.MOE_OK                  # a no-op
    assert static_fwd(L, d, rows=0, x=0, out=0) == moe.MOE_OK
    big = mi.QWEN35_397B_A17B
    dd = moe.MoeDims(big.hidden, big.n_experts, big.top_k, big.inter, big.shared_inter)
    assert moe.workspace_bytes(dd, 128) > moe.static_scratch_bytes()
    assert static_fwd(L, dd, rows=128) == moe.MOE_EWORKSPACE       # beyond the scratch array
    assert moe.status() == moe.MOE_OK                              # nothing above touched CUDA


def test_static_entry_respects_sticky_status_and_fault_knob(L):
    d = D()
    moe.reset_status()
    moe.debug_inject_fault(1)
    assert static_fwd(L, d) == moe.MOE_ECUDA       # the knob fires before anything is enqueued
    assert moe.status() == moe.MOE_ECUDA
    assert static_fwd(L, d) == moe.MOE_ECUDA       # sticky
    assert L.moe_static_device_status(None) == moe.MOE_ECUDA
    moe.reset_status()
    assert moe.status() == moe.MOE_OK


def host_fwd(L, d, rows=1, x=FAKE, out=FAKE + 4096, ws=FAKE, ws_bytes=None):
    sh = moe.MoeFp8Expert(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE))
    if ws_bytes is None:
        ws_bytes = moe.workspace_bytes(d, max(rows, 1))
    P = lambda a: ctypes.c_void_p(a) if a else None
    return L.moe_ffn_forward_host(ctypes.byref(d), P(x), rows, P(FAKE), P(FAKE), P(FAKE), ctypes.byref(sh),
                                  P(FAKE), P(out), None, P(ws), ws_bytes, None)


def test_host_entry_rejects_memory_the_device_cannot_address(L):
    """moe_ffn_forward_host takes pinned host buffers only: ordinary host
    memory (here a ctypes array) is refused on the host, before anything is
    enqueued, as are the forward's own argument errors."""
    moe.reset_status()
    d = D()
    buf = (ctypes.c_uint8 * (2 * 4096 + 16))()
    a = (ctypes.addressof(buf) + 15) // 16 * 16
    assert host_fwd(L, d, x=a, out=a + 4096) == moe.MOE_EINVAL     # not pinned
    assert host_fwd(L, d, x=0) == moe.MOE_EINVAL
    assert host_fwd(L, d, x=FAKE + 2) == moe.MOE_EINVAL            # misaligned
    assert host_fwd(L, d, out=FAKE) == moe.MOE_EINVAL              # out aliases x
    assert host_fwd(L, d, ws_bytes=16) == moe.MOE_EWORKSPACE
    assert host_fwd(L, d, rows=0) == moe.MOE_OK                    # a no-op
    assert moe.status() == moe.MOE_OK


def test_nvfp4_entry_rejects_on_host(L):
    """moe_ffn_forward_nvfp4's argument checks answer on the host."""
    moe.reset_status()
    d = D()
    sh = moe.MoeNvfp4Expert(FAKE, FAKE, FAKE)
    P = lambda a: ctypes.c_void_p(a) if a else None

    def call(x=FAKE, out=FAKE + 4096, gs=FAKE, rows=1, ws_bytes=None, shared=sh):
        wb = moe.workspace_bytes(d, max(rows, 1)) if ws_bytes is None else ws_bytes
        return L.moe_ffn_forward_nvfp4(ctypes.byref(d), P(x), rows, P(FAKE), P(FAKE), P(FAKE), P(gs),
                                       ctypes.byref(shared) if shared else None, P(FAKE), P(out), None, None,
                                       P(FAKE), wb, None)
    assert call(x=0) == moe.MOE_EINVAL
    assert call(x=FAKE + 8) == moe.MOE_EINVAL                    # misaligned
    assert call(gs=FAKE + 2) == moe.MOE_EINVAL                   # tensor scales not 4-byte aligned
    assert call(shared=None) == moe.MOE_EINVAL
    assert call(out=FAKE) == moe.MOE_EINVAL                      # out aliases x
    assert call(rows=-1) == moe.MOE_EINVAL
    assert call(ws_bytes=16) == moe.MOE_EWORKSPACE
    assert call(rows=0) == moe.MOE_OK
    assert moe.status() == moe.MOE_OK
