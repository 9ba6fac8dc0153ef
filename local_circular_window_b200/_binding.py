"""ctypes binding of libclear_attn.so (argument marshalling only: every step runs in the library).

The library must have been built (``python -m local_circular_window_b200.build`` or
``__graft_entry__.build()``); importing this module without it raises ImportError. There is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libclear_attn.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "clear_attn.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m local_circular_window_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

CLEAR_OK = 0
STATUS_NAMES = {0: "CLEAR_OK", 1: "CLEAR_ERR_INVALID_ARG", 2: "CLEAR_ERR_UNSUPPORTED", 3: "CLEAR_ERR_WORKSPACE",
                4: "CLEAR_ERR_CUDA", 5: "CLEAR_ERR_DEVICE_TIMEOUT"}


class ClearStrides(ctypes.Structure):
    """Mirror of clear_attn_strides_t: {batch, head, token} element strides of q, k, v and o."""
    _fields_ = [("q", ctypes.c_longlong * 3), ("k", ctypes.c_longlong * 3), ("v", ctypes.c_longlong * 3),
                ("o", ctypes.c_longlong * 3)]


class ClearStripe(ctypes.Structure):
    """Mirror of clear_attn_stripe_t."""
    _fields_ = [("q_row0", ctypes.c_int), ("q_row1", ctypes.c_int), ("key_row0", ctypes.c_int),
                ("key_row1", ctypes.c_int), ("text_keys", ctypes.c_int)]


class ClearParams(ctypes.Structure):
    """Mirror of clear_attn_params_t."""
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("n_text", ctypes.c_int), ("H", ctypes.c_int),
                ("W", ctypes.c_int), ("d", ctypes.c_int), ("r", ctypes.c_int), ("window", ctypes.c_int)]


WINDOWS = {"circle": 0, "square": 1, "shifted": 2}  # CLEAR_WINDOW_CIRCLE, _SQUARE, _SHIFTED


def _window_code(window) -> int:
    return WINDOWS[window] if isinstance(window, str) else int(window)


class ClearError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


_P = ctypes.POINTER(ClearParams)
_vp = ctypes.c_void_p
_ll = ctypes.c_longlong
_i = ctypes.c_int

_lib.clear_attn_version.restype = _i
_lib.clear_status_string.restype = ctypes.c_char_p
_lib.clear_status_string.argtypes = [_i]
_lib.clear_attn_fwd_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_fwd_workspace_size.argtypes = [_P, ctypes.POINTER(_i)]
_lib.clear_attn_bwd_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_bwd_workspace_size.argtypes = [_P, ctypes.POINTER(_i)]
_lib.clear_attn_fwd.restype = _i
_lib.clear_attn_fwd.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_fwd_strided.restype = _i
_lib.clear_attn_fwd_strided.argtypes = [_P, ctypes.POINTER(ClearStrides), _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t,
                                        _vp]
_S = ctypes.POINTER(ClearStripe)
_lib.clear_attn_fwd_stripe_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_fwd_stripe_workspace_size.argtypes = [_P, _S, ctypes.POINTER(_i)]
_lib.clear_attn_fwd_stripe.restype = _i
_lib.clear_attn_fwd_stripe.argtypes = [_P, _S, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
class ClearRope(ctypes.Structure):
    _fields_ = [("theta", ctypes.c_float), ("ntk", ctypes.c_float)]


_lib.clear_attn_fwd_rope_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_fwd_rope_workspace_size.argtypes = [_P, ctypes.POINTER(_i)]
_lib.clear_attn_fwd_rope.restype = _i
_lib.clear_attn_fwd_rope.argtypes = [_P, ctypes.POINTER(ClearRope), _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_rope_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_rope_workspace_size.argtypes = [_P, ctypes.POINTER(_i)]
_lib.clear_attn_bwd_rope_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_bwd_rope_workspace_size.argtypes = [_P, ctypes.POINTER(_i)]
_lib.clear_attn_bwd_rope.restype = _i
_lib.clear_attn_bwd_rope.argtypes = [_P, ctypes.POINTER(ClearRope), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     ctypes.c_size_t, _vp]
_lib.clear_attn_rope.restype = _i
_lib.clear_attn_rope.argtypes = [_P, ctypes.POINTER(ClearRope), _i, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_fwd_fp8.restype = _i
_lib.clear_attn_fwd_fp8.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_fwd_varlen_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_fwd_varlen_workspace_size.argtypes = [_P, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)]
_lib.clear_attn_fwd_varlen.restype = _i
_lib.clear_attn_fwd_varlen.argtypes = [_P, _i, ctypes.POINTER(_i), _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_text_merge.restype = _i
_lib.clear_attn_text_merge.argtypes = [_P, _i, _i, _vp, _vp, _vp, _vp, _vp]
_lib.clear_sched_stripe_forward_shape.restype = _i
_lib.clear_sched_stripe_forward_shape.argtypes = [_P, _S, ctypes.POINTER(_ll), ctypes.POINTER(_ll), ctypes.POINTER(_i),
                                                  ctypes.POINTER(_i)]
_lib.clear_sched_stripe_item_tiles.restype = _i
_lib.clear_sched_stripe_item_tiles.argtypes = [_P, _S, _ll, ctypes.POINTER(_i), ctypes.POINTER(_i), _i,
                                               ctypes.POINTER(_i)]
_lib.clear_attn_fwd_noalloc.restype = _i
_lib.clear_attn_fwd_noalloc.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.clear_attn_fwd_host_workspace_size.restype = ctypes.c_size_t
_lib.clear_attn_fwd_host_workspace_size.argtypes = [_P, ctypes.POINTER(_i)]
_lib.clear_attn_fwd_host.restype = _i
_lib.clear_attn_fwd_host.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_bwd.restype = _i
_lib.clear_attn_bwd.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.clear_attn_check.restype = _i
_lib.clear_attn_check.argtypes = [_vp]
_lib.clear_attn_selftest_expiry.restype = _i
_lib.clear_attn_selftest_expiry.argtypes = [_i, _vp]
_lib.clear_attn_device_diag.restype = None
_lib.clear_attn_device_diag.argtypes = [ctypes.POINTER(_i)]
_lib.clear_sched_forward_shape.restype = _i
_lib.clear_sched_forward_shape.argtypes = [_P, ctypes.POINTER(_ll), ctypes.POINTER(_ll), ctypes.POINTER(_i),
                                           ctypes.POINTER(_i)]
_lib.clear_sched_item_tiles.restype = _i
_lib.clear_sched_item_tiles.argtypes = [_P, _ll, ctypes.POINTER(_i), ctypes.POINTER(_i), _i, ctypes.POINTER(_i)]
_lib.clear_sched_pair_counts.restype = _i
_lib.clear_sched_pair_counts.argtypes = [_P, ctypes.POINTER(_ll), ctypes.POINTER(_ll)]


def lib() -> ctypes.CDLL:
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/clear_attn.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(clear_[a-z_]+)\s*\(", text)))


def make_params(B: int, heads: int, n_text: int, H: int, W: int, d: int, r: int, window="circle") -> ClearParams:
    return ClearParams(B, heads, n_text, H, W, d, r, _window_code(window))


def version() -> int:
    return _lib.clear_attn_version()


def status_string(status: int) -> str:
    return _lib.clear_status_string(status).decode()


def fwd_workspace_size(p: ClearParams) -> int:
    st = _i(0)
    n = _lib.clear_attn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_fwd_workspace_size")
    return n


def fwd_host_workspace_size(p: ClearParams) -> int:
    st = _i(0)
    n = _lib.clear_attn_fwd_host_workspace_size(ctypes.byref(p), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_fwd_host_workspace_size")
    return n


def bwd_workspace_size(p: ClearParams) -> int:
    st = _i(0)
    n = _lib.clear_attn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_bwd_workspace_size")
    return n


def make_stripe(q_row0: int, q_row1: int, key_row0: int, key_row1: int, text_keys: bool) -> ClearStripe:
    return ClearStripe(q_row0, q_row1, key_row0, key_row1, 1 if text_keys else 0)


def _stripe_ref(stripe):
    return None if stripe is None else ctypes.byref(stripe)


def forward_shape(p: ClearParams, stripe: ClearStripe = None):
    """(text pairs, image pairs, text splits, chunks per split) of the forward (of a stripe if given)."""
    nt, ni, s, c = _ll(0), _ll(0), _i(0), _i(0)
    st = _lib.clear_sched_stripe_forward_shape(ctypes.byref(p), _stripe_ref(stripe), ctypes.byref(nt),
                                               ctypes.byref(ni), ctypes.byref(s), ctypes.byref(c))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_sched_stripe_forward_shape")
    return nt.value, ni.value, s.value, c.value


def item_tiles(p: ClearParams, item: int, stripe: ClearStripe = None):
    """(q_info, tiles) of one forward work item (of a stripe if given); tiles: (kind, a, b, flags)."""
    q = (_i * 5)()
    n = _i(0)
    st = _lib.clear_sched_stripe_item_tiles(ctypes.byref(p), _stripe_ref(stripe), item, q, None, 0, ctypes.byref(n))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_sched_stripe_item_tiles")
    buf = (_i * (4 * max(1, n.value)))()
    st = _lib.clear_sched_stripe_item_tiles(ctypes.byref(p), _stripe_ref(stripe), item, q, buf, n.value,
                                            ctypes.byref(n))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_sched_stripe_item_tiles")
    tiles = [tuple(buf[4 * i:4 * i + 4]) for i in range(n.value)]
    return tuple(q), tiles


def pair_counts(p: ClearParams):
    u, e = _ll(0), _ll(0)
    st = _lib.clear_sched_pair_counts(ctypes.byref(p), ctypes.byref(u), ctypes.byref(e))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_sched_pair_counts")
    return u.value, e.value


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_qkv(name, t, shape):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(shape)}")


def clear_attn_fwd(q, k, v, n_text: int, H: int, W: int, r: int, o=None, lse=None, workspace=None, stream=None,
                   window="circle"):
    """CLEAR attention forward through the C ABI. Returns (o, lse); raises ClearError on failure.
    window: "circle" (CLEAR's mask), "square" (|dx| < r and |dy| < r) or "shifted" (that square with
    its centre clamped inside the grid; forward only)."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_qkv(name, t, q.shape)
    p = make_params(B, heads, n_text, H, W, d, r, window)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, heads, T), dtype=torch.float32, device=q.device)
    ws_bytes = fwd_workspace_size(p)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    st = _lib.clear_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace),
                             0 if workspace is None else workspace.numel() * workspace.element_size(),
                             _stream_ptr(stream))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_attn_fwd")
    return o, lse


def _bht_strides(t):
    return (t.stride(0), t.stride(1), t.stride(2))


def clear_attn_fwd_strided(q, k, v, n_text: int, H: int, W: int, r: int, o=None, lse=None, workspace=None,
                           stream=None, window="circle"):
    """CLEAR attention forward on strided [B, heads, T, d] views (each token row contiguous), e.g.
    q = qkv[:, :, 0].permute(0, 2, 1, 3) of a packed [B, T, 3, heads, d] buffer, through
    clear_attn_fwd_strided: nothing is copied. o may be any such view (allocated contiguous if None).
    Returns (o, lse)."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and tuple(t.shape) == tuple(q.shape) and t.stride(3) == 1):
            raise ValueError(f"{name} must be a CUDA bf16 view of shape {tuple(q.shape)} with contiguous rows")
    p = make_params(B, heads, n_text, H, W, d, r, window)
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if not (o.is_cuda and o.dtype == torch.bfloat16 and tuple(o.shape) == tuple(q.shape) and o.stride(3) == 1):
        raise ValueError(f"o must be a CUDA bf16 view of shape {tuple(q.shape)} with contiguous rows")
    if lse is None:
        lse = torch.empty((B, heads, T), dtype=torch.float32, device=q.device)
    st = ClearStrides((ctypes.c_longlong * 3)(*_bht_strides(q)), (ctypes.c_longlong * 3)(*_bht_strides(k)),
                      (ctypes.c_longlong * 3)(*_bht_strides(v)), (ctypes.c_longlong * 3)(*_bht_strides(o)))
    ws_bytes = fwd_workspace_size(p)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = _lib.clear_attn_fwd_strided(ctypes.byref(p), ctypes.byref(st), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                         _ptr(lse), _ptr(workspace),
                                         0 if workspace is None else workspace.numel() * workspace.element_size(),
                                         _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_fwd_strided")
    return o, lse


def clear_attn_fwd_stripe(q, k, v, n_text: int, H: int, W: int, r: int, stripe: ClearStripe, o=None, lse=None,
                          workspace=None, stream=None, window="circle"):
    """Forward of one stripe of a patch-parallel split through clear_attn_fwd_stripe: q, k, v are the
    stripe's contiguous [B, heads, n_text + H*W, d] tensors (halo rows included). Only the text rows
    and image rows [q_row0, q_row1) of o and lse are written. Returns (o, lse)."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_qkv(name, t, q.shape)
    p = make_params(B, heads, n_text, H, W, d, r, window)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, heads, T), dtype=torch.float32, device=q.device)
    st = _i(0)
    ws_bytes = _lib.clear_attn_fwd_stripe_workspace_size(ctypes.byref(p), ctypes.byref(stripe), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_fwd_stripe_workspace_size")
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = _lib.clear_attn_fwd_stripe(ctypes.byref(p), ctypes.byref(stripe), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                        _ptr(lse), _ptr(workspace),
                                        0 if workspace is None else workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_fwd_stripe")
    return o, lse


def clear_attn_fwd_fp8(q8, k8, v, qk_descale, n_text: int, H: int, W: int, r: int, o=None, lse=None, workspace=None,
                       stream=None, window="circle"):
    """Forward with E4M3 score products through clear_attn_fwd_fp8. q8, k8: contiguous CUDA uint8
    E4M3 codes [B, heads, T, d] (d = 128); v: bf16 like q8; qk_descale: CUDA float32 [B, heads]
    (s_q * s_k per head). Returns (o, lse)."""
    B, heads, T, d = q8.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q8", q8), ("k8", k8)):
        if not (t.is_cuda and t.dtype == torch.uint8 and t.is_contiguous() and tuple(t.shape) == (B, heads, T, d)):
            raise ValueError(f"{name} must be a contiguous CUDA uint8 tensor of shape {(B, heads, T, d)}")
    _check_qkv("v", v, q8.shape)
    if not (qk_descale.is_cuda and qk_descale.dtype == torch.float32 and qk_descale.is_contiguous()
            and qk_descale.numel() == B * heads):
        raise ValueError("qk_descale must be a contiguous CUDA float32 tensor of B * heads values")
    p = make_params(B, heads, n_text, H, W, d, r, window)
    if o is None:
        o = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, heads, T), dtype=torch.float32, device=q8.device)
    if workspace is None:
        n = fwd_workspace_size(p)
        workspace = torch.empty(max(16, n), dtype=torch.uint8, device=q8.device)
    status = _lib.clear_attn_fwd_fp8(ctypes.byref(p), _ptr(q8), _ptr(k8), _ptr(v), _ptr(qk_descale), _ptr(o), _ptr(lse),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_fwd_fp8")
    return o, lse


def rope_workspace_size(p: ClearParams) -> int:
    st = _i(0)
    n = _lib.clear_attn_fwd_rope_workspace_size(ctypes.byref(p), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_fwd_rope_workspace_size")
    return n


def clear_attn_fwd_rope(q, k, v, n_text: int, H: int, W: int, r: int, theta: float = 10000.0, ntk: float = 1.0,
                        o=None, lse=None, workspace=None, stream=None, window="circle"):
    """Forward on rotary-embedded q and k through clear_attn_fwd_rope: one streaming pass rotates q
    and k (axial 2D RoPE with the NTK-aware base) into the workspace, then the forward runs on the
    rotated copies; the inputs are not modified. Tensors as clear_attn_fwd. Returns (o, lse)."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_qkv(name, t, q.shape)
    p = make_params(B, heads, n_text, H, W, d, r, window)
    rope = ClearRope(theta, ntk)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, heads, T), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(rope_workspace_size(p), dtype=torch.uint8, device=q.device)
    status = _lib.clear_attn_fwd_rope(ctypes.byref(p), ctypes.byref(rope), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_fwd_rope")
    return o, lse


def _item_array(items):
    flat = [int(x) for it in items for x in it]
    if not items or any(len(it) != 3 for it in items):
        raise ValueError("items must be a non-empty sequence of (n_text, H, W)")
    return (_i * len(flat))(*flat)


def varlen_tokens(items):
    """Token count of a packed mixed-resolution batch and each item's first token."""
    starts, t = [], 0
    for n_text, H, W in items:
        starts.append(t)
        t += n_text + H * W
    return t, starts


def varlen_workspace_size(heads: int, d: int, r: int, items, window="circle") -> int:
    p = make_params(1, heads, 0, 1, 1, d, r, window)
    st = _i(0)
    n = _lib.clear_attn_fwd_varlen_workspace_size(ctypes.byref(p), len(items), _item_array(items), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_fwd_varlen_workspace_size")
    return n


def clear_attn_fwd_varlen(q, k, v, items, r: int, o=None, lse=None, workspace=None, stream=None, window="circle"):
    """Mixed-resolution batch forward through clear_attn_fwd_varlen: one launch over items of their
    own (n_text, H, W). q, k, v: contiguous bf16 CUDA [heads, T_total, d], the items packed along the
    token axis in order (varlen_tokens gives each item's first token). Returns (o, lse) with o like q
    and lse fp32 [heads, T_total]."""
    heads, T, d = q.shape
    total, _ = varlen_tokens(items)
    if T != total:
        raise ValueError("q's token axis must hold every item's n_text + H * W tokens")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_qkv(name, t, q.shape)
    p = make_params(1, heads, 0, 1, 1, d, r, window)
    shapes = _item_array(items)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((heads, T), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(varlen_workspace_size(heads, d, r, items, window), dtype=torch.uint8, device=q.device)
    status = _lib.clear_attn_fwd_varlen(ctypes.byref(p), len(items), shapes, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                        _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_fwd_varlen")
    return o, lse


TEXT_MERGE_MODES = {"exact": 0, "eq7": 1}


def clear_attn_text_merge(o_parts, lse_parts, mode="exact", o=None, lse=None, stream=None):
    """Merges the text rows of P stripes through clear_attn_text_merge. o_parts: bf16
    [P, B, heads, n_text, d]; lse_parts: fp32 [P, B, heads, n_text] (contiguous CUDA tensors).
    mode "exact" (disjoint key shares, log-sum-exp weights) or "eq7" (the paper's patch-wise
    average). Returns (o [B, heads, n_text, d], lse [B, heads, n_text])."""
    P, B, heads, n_text, d = o_parts.shape
    if not (o_parts.is_cuda and o_parts.dtype == torch.bfloat16 and o_parts.is_contiguous()):
        raise ValueError("o_parts must be a contiguous CUDA bf16 tensor")
    if not (lse_parts.is_cuda and lse_parts.dtype == torch.float32 and lse_parts.is_contiguous()
            and tuple(lse_parts.shape) == (P, B, heads, n_text)):
        raise ValueError("lse_parts must be a contiguous CUDA fp32 tensor [P, B, heads, n_text]")
    p = make_params(B, heads, n_text, 1, 1, d, 1)
    o = torch.empty((B, heads, n_text, d), dtype=torch.bfloat16, device=o_parts.device) if o is None else o
    lse = torch.empty((B, heads, n_text), dtype=torch.float32, device=o_parts.device) if lse is None else lse
    status = _lib.clear_attn_text_merge(ctypes.byref(p), P, TEXT_MERGE_MODES[mode], _ptr(o_parts), _ptr(lse_parts),
                                        _ptr(o), _ptr(lse), _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_text_merge")
    return o, lse


def clear_attn_fwd_host(q, k, v, n_text: int, H: int, W: int, r: int, o=None, lse=None, workspace=None,
                        stream=None, window="circle"):
    """CLEAR attention forward from pinned host tensors to pinned host tensors through the C ABI
    (clear_attn_fwd_host: the library copies slice groups in and out on its own streams, overlapped
    with the forward). q, k, v: contiguous bf16 CPU tensors in pinned memory; o, lse: pinned CPU
    outputs (allocated pinned if None); workspace: a CUDA uint8 tensor on the current device
    (allocated if None). The call is asynchronous: synchronise `stream` before reading o and lse.
    Returns (o, lse); raises ClearError on failure."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_host(name, t, q.shape, torch.bfloat16)
    p = make_params(B, heads, n_text, H, W, d, r, window)
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, heads, T), dtype=torch.float32, pin_memory=True)
    _check_host("o", o, q.shape, torch.bfloat16)
    _check_host("lse", lse, (B, heads, T), torch.float32)
    ws_bytes = fwd_host_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    st = _lib.clear_attn_fwd_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_attn_fwd_host")
    return o, lse


def clear_attn_bwd(q, k, v, o, lse, dO, n_text: int, H: int, W: int, r: int, dq=None, dk=None, dv=None,
                   workspace=None, stream=None, window="circle"):
    """CLEAR attention backward through the C ABI. Returns (dq, dk, dv). window as for the forward."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO)):
        _check_qkv(name, t, q.shape)
    p = make_params(B, heads, n_text, H, W, d, r, window)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws_bytes = bwd_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    st = _lib.clear_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream_ptr(stream))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_attn_bwd")
    return dq, dk, dv


def clear_attn_check(stream=None) -> int:
    """Synchronise the stream and return the device status (CLEAR_OK or an error code)."""
    return _lib.clear_attn_check(_stream_ptr(stream))


def device_diag() -> list:
    """Context of the wait behind the last device timeout reported to this thread (diagnosis)."""
    out = (_i * 8)()
    _lib.clear_attn_device_diag(out)
    return list(out)


def selftest_expiry(limit_ms: int, stream=None) -> int:
    """Launches the failure-detection self-test (a wait that expires after limit_ms); returns the
    launch status. clear_attn_check() then reports CLEAR_ERR_DEVICE_TIMEOUT."""
    return _lib.clear_attn_selftest_expiry(int(limit_ms), _stream_ptr(stream))


def _check_host(name, t, shape, dtype):
    # Page-locking is checked by the library (CLEAR_ERR_INVALID_ARG if missing).
    if not (t.device.type == "cpu" and t.dtype == dtype and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name} must be a contiguous CPU {dtype} tensor of shape {tuple(shape)}")


def rope_rotate_workspace_size(p: ClearParams) -> int:
    st = _i(0)
    n = _lib.clear_attn_rope_workspace_size(ctypes.byref(p), ctypes.byref(st))
    if st.value != CLEAR_OK:
        raise ClearError(st.value, "clear_attn_rope_workspace_size")
    return n


def clear_attn_rope(q, k, n_text: int, H: int, W: int, theta: float = 10000.0, ntk: float = 1.0, inverse: bool = False,
                    q_out=None, k_out=None, workspace=None, stream=None):
    """The rotary embedding alone through clear_attn_rope: q and k (bf16 [B, heads, T, d]) rotated by
    axial 2D RoPE with the NTK-aware base (inverse=True: by the negated angles, the transpose) into
    q_out and k_out (new tensors by default; q_out=q, k_out=k rotates in place). Returns
    (q_out, k_out)."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k)):
        _check_qkv(name, t, q.shape)
    p = make_params(B, heads, n_text, H, W, d, 1)
    rope = ClearRope(theta, ntk)
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    for name, t in (("q_out", q_out), ("k_out", k_out)):
        _check_qkv(name, t, q.shape)
    if workspace is None:
        workspace = torch.empty(rope_rotate_workspace_size(p), dtype=torch.uint8, device=q.device)
    status = _lib.clear_attn_rope(ctypes.byref(p), ctypes.byref(rope), 1 if inverse else 0, _ptr(q), _ptr(k), _ptr(q_out),
                                  _ptr(k_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream_ptr(stream))
    if status != CLEAR_OK:
        raise ClearError(status, "clear_attn_rope")
    return q_out, k_out


def clear_attn_bwd_rope(q, k, v, o, lse, dO, n_text: int, H: int, W: int, r: int, theta: float = 10000.0,
                        ntk: float = 1.0, dq=None, dk=None, dv=None, workspace=None, stream=None, window="circle"):
    """Backward of clear_attn_fwd_rope through clear_attn_bwd_rope: gradients with respect to the
    unrotated q, k and v (o and lse as clear_attn_fwd_rope returned them). Returns (dq, dk, dv)."""
    B, heads, T, d = q.shape
    if T != n_text + H * W:
        raise ValueError("T must equal n_text + H * W")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dO", dO)):
        _check_qkv(name, t, q.shape)
    p = make_params(B, heads, n_text, H, W, d, r, window)
    rope = ClearRope(theta, ntk)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        st = _i(0)
        n = _lib.clear_attn_bwd_rope_workspace_size(ctypes.byref(p), ctypes.byref(st))
        if st.value != CLEAR_OK:
            raise ClearError(st.value, "clear_attn_bwd_rope_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    st = _lib.clear_attn_bwd_rope(ctypes.byref(p), ctypes.byref(rope), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                  _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    if st != CLEAR_OK:
        raise ClearError(st, "clear_attn_bwd_rope")
    return dq, dk, dv
