"""The C-ABI library: it loads, exports every function include/attn.h
declares, and its host-only paths (argument checks, sizes, strings) behave
as documented.  No kernel is launched, so these run without a GPU."""
import ctypes
import os
import re

import pytest

from exact_tiled_attention_39_b200 import attn as A

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from exact_tiled_attention_39_b200 import build
    build.build()
    return A.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert "attn_fwd" in declared and "attn_quantize_mxfp8" in declared
    for name in declared:
        assert hasattr(L, name), f"libattn.so does not export {name}"
    assert set(A.EXPORTED_SYMBOLS) <= set(declared)


def test_version_and_strings(L):
    assert L.attn_abi_version() == 4
    assert A.status_string(0) == "ATTN_OK"
    assert A.status_string(5) == "ATTN_ERR_BAD_SEQLENS"
    assert A.status_string(6) == "ATTN_ERR_TIMEOUT"


def test_workspace_size(L):
    s = A.Shape(16384, 7, 32, 128, 4096)
    n_bf16 = A.workspace_size(s, A.ATTN_BF16)
    n_mx = A.workspace_size(s, A.ATTN_MXFP8)
    max_entries = 16384 // 128 + 7 + 1
    assert n_bf16 >= 256 + 2 * 16 * max_entries
    assert n_mx >= n_bf16 + 3 * 16384 * 32 * 128 + 3 * 16384 * 32 * 4
    n_nv = A.workspace_size(s, A.ATTN_NVFP4)
    # packed E2M1 codes and UE4M3 scales of q and k, exact bf16 v
    assert n_nv >= n_bf16 + 2 * (16384 * 32 * 64 + 16384 * 32 * 8) + 2 * 16384 * 32 * 128
    assert A.workspace_size(s, 3) == 0                              # dtype unsupported
    assert A.workspace_size(A.Shape(16, 1, 1, 96, 16)) == 0       # d unsupported
    assert A.workspace_size(A.Shape(-1, 1, 1, 64, 16)) == 0


def _fwd(L, shape, ptrs=(16, 16, 16, 16, 16), ws=16, ws_bytes=1 << 20, scale=0.125, causal=1,
         dtype=0, cu=None):
    s = shape.c() if shape is not None else None
    q, k, v, o, l = (ctypes.c_void_p(p) if p else None for p in ptrs)
    return L.attn_fwd(q, k, v, cu, o, l, causal, scale, dtype, None,
                      ctypes.byref(s) if s is not None else None,
                      ctypes.c_void_p(ws) if ws else None, ws_bytes)


def test_host_checks_return_before_launch(L):
    ok = A.Shape(256, 1, 2, 64, 256)
    assert _fwd(L, None) == 1                                   # NULL shape
    assert _fwd(L, A.Shape(256, 1, 2, 96, 256)) == 2            # d unsupported
    assert _fwd(L, ok, dtype=7) == 2
    assert _fwd(L, ok, scale=0.0) == 1
    assert _fwd(L, ok, scale=float("nan")) == 1
    assert _fwd(L, ok, causal=2) == 1
    assert _fwd(L, A.Shape(256, 2, 2, 64, 100)) == 1            # dense: T != B*N
    assert _fwd(L, ok, ptrs=(16, 16, 0, 16, 16)) == 1           # NULL v
    assert _fwd(L, ok, ptrs=(16, 24, 16, 16, 16)) == 3          # misaligned k
    assert _fwd(L, ok, ws=0) == 4
    assert _fwd(L, ok, ws_bytes=8) == 4
    assert _fwd(L, A.Shape(0, 0, 2, 64, 0), ptrs=(0, 0, 0, 0, 0)) == 0   # T == 0: no-op


def test_quantize_host_checks(L):
    assert L.attn_quantize_mxfp8(None, None, None, 4, 48, None) == 1     # cols % 32
    assert L.attn_quantize_mxfp8(None, None, None, 0, 64, None) == 0     # empty: no-op
    assert L.attn_quantize_mxfp8(ctypes.c_void_p(16), ctypes.c_void_p(8), ctypes.c_void_p(16),
                                 4, 64, None) == 3


def test_timing_read_without_a_timed_call(L):
    """attn_timing_read reports INVALID_ARG until a call has been timed
    (no GPU needed: no call is made)."""
    import ctypes
    A.attn_timing_enable(True)
    a, b = ctypes.c_float(), ctypes.c_float()
    assert L.attn_timing_read(ctypes.byref(a), ctypes.byref(b)) == 1
    assert L.attn_timing_read(None, None) == 1
    A.attn_timing_enable(False)


def _bwd(L, shape, n_null=None, misalign=None, ws=16, ws_bytes=1 << 30, scale=0.125, causal=1,
         dtype=0):
    s = shape.c() if shape is not None else None
    ptrs = [16] * 10      # q k v out dout lse cu dq dk dv (cu at index 6: NULL = dense)
    ptrs[6] = 0
    if n_null is not None:
        ptrs[n_null] = 0
    if misalign is not None:
        ptrs[misalign] = 24
    args = [ctypes.c_void_p(p) if p else None for p in ptrs]
    return L.attn_bwd(*args, causal, scale, dtype, None,
                      ctypes.byref(s) if s is not None else None,
                      ctypes.c_void_p(ws) if ws else None, ws_bytes)


def test_bwd_workspace_size(L):
    s = A.Shape(16384, 7, 32, 128, 4096)
    n = A.bwd_workspace_size(s)
    max_entries = 16384 // 128 + 7 + 1
    # lists, D (fp32 [H, T]) and the fp32 dQ accumulator
    assert n >= 256 + 2 * 16 * max_entries + 4 * 16384 * 32 + 4 * 16384 * 32 * 128
    # MXFP8: plus the dequantised q, k, v and dout
    assert A.bwd_workspace_size(s, A.ATTN_MXFP8) >= n + 4 * 2 * 16384 * 32 * 128
    assert A.bwd_workspace_size(s, 7) == 0
    assert A.bwd_workspace_size(A.Shape(16, 1, 1, 96, 16)) == 0
    assert A.bwd_workspace_size(A.Shape(-1, 1, 1, 64, 16)) == 0


def test_bwd_host_checks_return_before_launch(L):
    ok = A.Shape(256, 1, 2, 64, 256)
    assert _bwd(L, None) == 1
    assert _bwd(L, A.Shape(256, 1, 2, 96, 256)) == 2            # d unsupported
    assert _bwd(L, ok, dtype=7) == 2                            # unknown dtype
    n_bf16 = A.bwd_workspace_size(ok)
    assert _bwd(L, ok, dtype=1, ws_bytes=n_bf16) == 4           # MXFP8 needs more
    assert _bwd(L, ok, scale=-1.0) == 1
    assert _bwd(L, ok, causal=3) == 1
    assert _bwd(L, A.Shape(256, 2, 2, 64, 100)) == 1            # dense: T != B*N
    for i in (0, 3, 4, 5, 7, 9):
        assert _bwd(L, ok, n_null=i) == 1
    for i in (1, 4, 5, 8):
        assert _bwd(L, ok, misalign=i) == 3
    assert _bwd(L, ok, ws=0) == 4
    assert _bwd(L, ok, ws_bytes=64) == 4
    assert _bwd(L, A.Shape(0, 0, 2, 64, 0)) == 0                # T == 0: no-op


def test_rotated_quantiser_host_checks(L):
    vp = ctypes.c_void_p
    assert L.attn_quantize_mxfp8_rotated(None, None, None, None, 0, 128, None) == 0   # empty
    assert L.attn_quantize_mxfp8_rotated(None, None, None, None, 4, 96, None) == 2    # cols
    assert L.attn_quantize_mxfp8_rotated(None, None, None, None, -1, 128, None) == 1
    assert L.attn_quantize_mxfp8_rotated(vp(16), None, vp(16), vp(16), 4, 128, None) == 1
    assert L.attn_quantize_mxfp8_rotated(vp(16), vp(16), vp(24), vp(16), 4, 64, None) == 3
    assert L.attn_quantize_mxfp8_rotated(vp(16), vp(16), vp(16), vp(18), 4, 64, None) == 3


def test_incoherent_forward_host_checks(L):
    vp = ctypes.c_void_p
    ok = A.Shape(256, 1, 2, 64, 256).c()
    empty = A.Shape(0, 0, 2, 64, 0).c()
    p = vp(16)

    def call(shape, signs, ws_bytes=1 << 26):
        return L.attn_fwd_incoherent(p, p, p, None, p, p, 1, 0.125, signs, None,
                                     ctypes.byref(shape) if shape is not None else None, p,
                                     ws_bytes)
    assert call(ok, None) == 1                    # signs required
    assert call(ok, vp(18)) == 3                  # signs misaligned
    assert call(None, vp(16)) == 1                # no shape
    assert call(ok, vp(16), ws_bytes=64) == 4     # workspace too small (MXFP8 layout)
    assert call(empty, None) == 0                 # T == 0: no-op


def test_nvfp4_quantiser_host_checks(L):
    vp = ctypes.c_void_p
    assert L.attn_quantize_nvfp4(None, None, None, 0, 64, None) == 0         # empty
    assert L.attn_quantize_nvfp4(None, None, None, 4, 40, None) == 1         # cols % 16
    assert L.attn_quantize_nvfp4(vp(16), vp(16), None, 4, 64, None) == 1     # scales NULL
    assert L.attn_quantize_nvfp4(vp(24), vp(16), vp(16), 4, 64, None) == 3   # x misaligned
    assert L.attn_quantize_nvfp4(vp(16), vp(12), vp(16), 4, 64, None) == 3   # codes misaligned
