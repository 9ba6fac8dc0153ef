"""C ABI checks that need no GPU: the library loads, exports every declared symbol, validates its
arguments on the host and reports sizes. Error paths never launch anything, so they are safe to run
with host buffers standing in for device pointers (the canaries prove nothing was written)."""
import ctypes

import numpy as np
import pytest
import torch

import local_circular_window_b200 as L
from local_circular_window_b200 import _binding as Bd


def test_library_exports_every_declared_function():
    names = L.header_functions()
    assert len(names) >= 10
    missing = [n for n in names if not hasattr(L.lib(), n)]
    assert missing == []


def test_version_and_status_strings():
    assert L.version() >= 100
    for code, name in Bd.STATUS_NAMES.items():
        assert L.status_string(code) == name
    assert L.status_string(99) == "CLEAR_ERR_UNKNOWN"


@pytest.mark.parametrize("fields,expected", [
    (dict(r=0), 1), (dict(B=0), 1), (dict(heads=0), 1), (dict(H=0), 1), (dict(W=-3), 1), (dict(n_text=-1), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(window=3), 1), (dict(window=-1), 1), (dict(H=1 << 15, W=1 << 15), 1), (dict(n_text=1 << 25), 1),
])
def test_invalid_params_statuses(fields, expected):
    base = dict(B=1, heads=2, n_text=16, H=16, W=16, d=64, r=4)
    base.update(fields)
    p = L.make_params(**base)
    st = ctypes.c_int(0)
    assert L.lib().clear_attn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(st)) == 0
    assert st.value == expected
    assert L.lib().clear_attn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(st)) == 0
    assert st.value == expected


def _canary(n=4096):
    a = np.full(n, 0x5A, dtype=np.uint8)
    return a, ctypes.c_void_p(a.ctypes.data)


def test_forward_argument_errors_launch_nothing():
    p = L.make_params(1, 2, 16, 16, 16, 64, 4)
    bufs = [_canary() for _ in range(6)]
    q, k, v, o, lse, ws = (b[1] for b in bufs)
    wsz = L.fwd_workspace_size(p)
    f = L.lib().clear_attn_fwd
    # null pointers
    assert f(ctypes.byref(p), None, k, v, o, lse, ws, wsz, None) == 1
    assert f(ctypes.byref(p), q, k, v, None, lse, ws, wsz, None) == 1
    # misaligned pointer
    assert f(ctypes.byref(p), ctypes.c_void_p(q.value + 2), k, v, o, lse, ws, wsz, None) == 1
    # workspace too small / missing
    assert f(ctypes.byref(p), q, k, v, o, lse, ws, wsz - 1, None) == 3
    assert f(ctypes.byref(p), q, k, v, o, lse, None, wsz, None) == 3
    # bad params
    bad = L.make_params(1, 2, 16, 16, 16, 96, 4)
    assert f(ctypes.byref(bad), q, k, v, o, lse, ws, wsz, None) == 2
    for a, _ in bufs:
        assert (a == 0x5A).all()


def test_backward_argument_errors_launch_nothing():
    p = L.make_params(2, 3, 7, 9, 11, 128, 3)
    bufs = [_canary() for _ in range(10)]
    q, k, v, o, lse, dO, dq, dk, dv, ws = (b[1] for b in bufs)
    wsz = L.bwd_workspace_size(p)
    f = L.lib().clear_attn_bwd
    assert f(ctypes.byref(p), q, k, v, o, lse, None, dq, dk, dv, ws, wsz, None) == 1
    assert f(ctypes.byref(p), q, k, v, o, lse, dO, dq, ctypes.c_void_p(dk.value + 8), dv, ws, wsz, None) == 1
    assert f(ctypes.byref(p), q, k, v, o, lse, dO, dq, dk, dv, ws, wsz - 256, None) == 3
    zero_r = L.make_params(2, 3, 7, 9, 11, 128, 0)
    assert f(ctypes.byref(zero_r), q, k, v, o, lse, dO, dq, dk, dv, ws, wsz, None) == 1
    for a, _ in bufs:
        assert (a == 0x5A).all()


def test_host_forward_argument_errors_launch_nothing():
    # Every argument error is caught before any CUDA call (this runs without a GPU).
    p = L.make_params(2, 3, 16, 16, 16, 64, 4)
    bufs = [_canary() for _ in range(6)]
    q, k, v, o, lse, ws = (b[1] for b in bufs)
    wsz = L.fwd_host_workspace_size(p)
    f = L.lib().clear_attn_fwd_host
    assert f(ctypes.byref(p), None, k, v, o, lse, ws, wsz, None) == 1
    assert f(ctypes.byref(p), q, k, v, o, None, ws, wsz, None) == 1
    assert f(ctypes.byref(p), q, ctypes.c_void_p(k.value + 4), v, o, lse, ws, wsz, None) == 1
    assert f(ctypes.byref(p), q, k, v, o, lse, ws, wsz - 1, None) == 3
    assert f(ctypes.byref(p), q, k, v, o, lse, None, wsz, None) == 3
    bad = L.make_params(2, 3, 16, 16, 16, 96, 4)
    assert f(ctypes.byref(bad), q, k, v, o, lse, ws, wsz, None) == 2
    for a, _ in bufs:
        assert (a == 0x5A).all()


def _a256(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("B,heads,group", [(1, 24, 1), (2, 24, 2), (1, 5, 1), (3, 17, 3)])
def test_host_workspace_size(B, heads, group):
    # Device copies of q, k, v, o (bf16), one aligned lse block (fp32) per group, then the forward
    # workspace of one group of `group` slices (at most 24 groups of consecutive slices).
    T, d = 512 + 64 * 64, 128
    p = L.make_params(B, heads, 512, 64, 64, d, 8)
    tens = _a256(B * heads * T * d * 2)
    n_groups = -(-B * heads // group)
    fws = L.fwd_workspace_size(L.make_params(1, group, 512, 64, 64, d, 8))
    assert L.fwd_host_workspace_size(p) == 4 * tens + n_groups * _a256(group * T * 4) + fws
    st = ctypes.c_int(0)
    assert L.lib().clear_attn_fwd_host_workspace_size(ctypes.byref(L.make_params(1, 2, 16, 16, 16, 64, 0)),
                                                      ctypes.byref(st)) == 0
    assert L.status_string(st.value) == "CLEAR_ERR_INVALID_ARG"


@pytest.mark.parametrize("limit_ms", [0, -5, 5001])
def test_selftest_rejects_bad_limits_before_any_cuda_call(limit_ms):
    assert L.status_string(L.lib().clear_attn_selftest_expiry(limit_ms, None)) == "CLEAR_ERR_INVALID_ARG"


def test_shifted_window_limits():
    # Needs H, W >= 2r - 1 (never clamped) and has no backward.
    st = ctypes.c_int(0)
    bad = L.make_params(1, 2, 16, 16, 9, 64, 6, "shifted")   # 2r - 1 = 11 > W = 9
    assert L.lib().clear_attn_fwd_workspace_size(ctypes.byref(bad), ctypes.byref(st)) == 0
    assert L.status_string(st.value) == "CLEAR_ERR_INVALID_ARG"
    ok = L.make_params(1, 2, 16, 16, 11, 64, 6, "shifted")
    L.lib().clear_attn_fwd_workspace_size(ctypes.byref(ok), ctypes.byref(st))
    assert st.value == 0
    assert L.lib().clear_attn_bwd_workspace_size(ctypes.byref(ok), ctypes.byref(st)) == 0
    assert L.status_string(st.value) == "CLEAR_ERR_UNSUPPORTED"
    bufs = [_canary() for _ in range(10)]
    assert L.status_string(L.lib().clear_attn_bwd(ctypes.byref(ok), *(p_ for _, p_ in bufs), ctypes.c_size_t(1 << 20),
                                                  None)) == "CLEAR_ERR_UNSUPPORTED"
    assert all((a == 0x5A).all() for a, _ in bufs)


def test_workspace_sizes():
    # Forward scratch holds the split partials of the text rows: S * BH * n_text rows of d fp32 plus
    # (max, sum) pairs; none without text.
    p = L.make_params(1, 24, 512, 64, 64, 128, 8)
    nt, ni, S, cps = L.forward_shape(p)
    rows = S * 24 * 512
    need = rows * 128 * 4 + rows * 8
    got = L.fwd_workspace_size(p)
    assert need <= got <= need + 512
    assert L.fwd_workspace_size(L.make_params(1, 2, 0, 8, 8, 64, 2)) == 0
    # Backward scratch: D and LSE*log2(e) per row, and three sets of text-row split partials. The
    # backward splits the keys into 128-token chunks, up to 64 chunks per split: one split here.
    b = L.bwd_workspace_size(p)
    sb = -(-(-(-4608 // 128)) // 64)
    rows_b = sb * 24 * 512
    need_b = 2 * 24 * 4608 * 4 + 3 * rows_b * 128 * 4
    assert need_b <= b <= need_b + 4 * 512


def test_no_fallback_without_library(monkeypatch, tmp_path):
    # The binding refuses to import when the shared library is absent (no CPU fallback path).
    import importlib.util
    import os
    src = os.path.join(os.path.dirname(Bd.__file__), "_binding.py")
    code = open(src).read().replace('LIB_PATH = os.path.join(_PKG, "libclear_attn.so")',
                                    f'LIB_PATH = {str(tmp_path / "missing.so")!r}')
    mod_path = tmp_path / "binding_copy.py"
    mod_path.write_text(code)
    spec = importlib.util.spec_from_file_location("binding_copy", mod_path)
    with pytest.raises(ImportError):
        spec.loader.exec_module(importlib.util.module_from_spec(spec))


def test_host_forward_binding_checks_tensors():
    # The binding checks device, dtype, layout and shape before calling the library.
    B, heads, n_text, H, W, d = 1, 2, 16, 8, 8, 64
    T = n_text + H * W
    ok = torch.zeros((B, heads, T, d), dtype=torch.bfloat16)
    lse = torch.zeros((B, heads, T))
    bad_inputs = (torch.zeros((B, heads, T, d), dtype=torch.float32),                # dtype
                  torch.zeros((B, heads, d, T), dtype=torch.bfloat16).transpose(2, 3),  # layout
                  torch.zeros((B, heads, T + 1, d), dtype=torch.bfloat16))             # shape
    for bad in bad_inputs:
        with pytest.raises(ValueError):
            L.clear_attn_fwd_host(ok, bad, ok, n_text, H, W, 2, o=ok.clone(), lse=lse)
    with pytest.raises(ValueError):  # lse of the wrong dtype
        L.clear_attn_fwd_host(ok, ok, ok, n_text, H, W, 2, o=ok.clone(), lse=lse.double())


@pytest.mark.parametrize("items,expected", [
    ([], 1), ([(1, 0, 4)], 1), ([(-1, 4, 4)], 1), ([(3, 4, 4), (2, 5, 0)], 1), ([(0, 1 << 15, 1 << 15)], 1),
])
def test_varlen_workspace_query_rejects_bad_items(items, expected):
    with pytest.raises(L.ClearError) as e:
        if not items:
            p = L.make_params(1, 2, 0, 1, 1, 64, 3)
            st = ctypes.c_int(0)
            n = Bd._lib.clear_attn_fwd_varlen_workspace_size(ctypes.byref(p), 0, None, ctypes.byref(st))
            assert n == 0
            raise L.ClearError(st.value, "clear_attn_fwd_varlen_workspace_size")
        L.varlen_workspace_size(2, 64, 3, items)
    assert e.value.status == expected


def test_varlen_workspace_grows_with_text_rows():
    a = L.varlen_workspace_size(2, 128, 4, [(0, 16, 16), (0, 8, 8)])
    b = L.varlen_workspace_size(2, 128, 4, [(128, 16, 16), (0, 8, 8)])
    assert b > a > 0 and a % 256 == 0 and b % 256 == 0
    with pytest.raises(L.ClearError):
        L.varlen_workspace_size(2, 128, 4, [(1, 2, 2)] * 4097)


def test_rope_rotation_workspace_size():
    # The stand-alone rotation's workspace is its (cos, sin) table: max(H, W) positions x d/4 fp32
    # pairs, rounded up to 256 bytes; bad parameters report their status.
    for n_text, H, W, d in ((512, 64, 64, 128), (0, 13, 50, 64), (77, 24, 40, 128)):
        p = L.make_params(1, 2, n_text, H, W, d, 1)
        want = (max(H, W) * (d // 4) * 8 + 255) // 256 * 256
        assert L.rope_rotate_workspace_size(p) == want
    st = ctypes.c_int(0)
    bad = L.make_params(1, 2, 4, 8, 8, 96, 1)  # d = 96 is not supported
    assert L.lib().clear_attn_rope_workspace_size(ctypes.byref(bad), ctypes.byref(st)) == 0
    assert st.value != 0
