"""The strided forward (clear_attn_fwd_strided) reads q, k, v in place from a packed qkv buffer, as a
FLUX-style attention layer produces them ([B, T, 3, heads, d]: one projection, then split), and
writes o as [B, T, heads, d]. Only the addressing differs from clear_attn_fwd, so the results must
be bit-identical to the contiguous call on copies of the same tensors."""
import ctypes

import numpy as np
import pytest
import torch

import local_circular_window_b200 as L
from clear_inputs import Workload, make_random


def _packed(wl, seed):
    buf = make_random((wl.B, wl.T, 3, wl.heads, wl.d), seed=seed, device="cuda")
    q, k, v = (buf[:, :, i].permute(0, 2, 1, 3) for i in range(3))  # [B, heads, T, d] views
    return buf, q, k, v


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [Workload("packed_ragged", 2, 3, 77, 24, 40, 128, 5),
                                Workload("packed_d64", 2, 2, 20, 16, 24, 64, 4),
                                Workload("packed_flux1024", 1, 24, 512, 64, 64, 128, 16)], ids=lambda w: w.name)
def test_packed_qkv_matches_contiguous_bit_for_bit(wl):
    buf, q, k, v = _packed(wl, seed=31)
    assert not q.is_contiguous() and q.stride() == (wl.T * 3 * wl.heads * wl.d, wl.d, 3 * wl.heads * wl.d, 1)
    o_btd = torch.full((wl.B, wl.T, wl.heads, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    o_view = o_btd.permute(0, 2, 1, 3)
    o, lse = L.clear_attn_fwd_strided(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o_view)
    assert L.clear_attn_check() == 0
    ref_o, ref_lse = L.clear_attn_fwd(q.contiguous(), k.contiguous(), v.contiguous(), wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    assert torch.equal(o, ref_o) and torch.equal(o_btd, ref_o.permute(0, 2, 1, 3))
    assert torch.equal(lse, ref_lse)


@pytest.mark.gpu
def test_strided_square_window_and_contiguous_strides():
    # The strided call on plain contiguous tensors is the ordinary forward; the window option passes
    # through unchanged.
    wl = Workload("sq", 1, 2, 16, 19, 21, 128, 3)
    buf, q, k, v = _packed(wl, seed=32)
    qc, kc, vc = q.contiguous(), k.contiguous(), v.contiguous()
    o1, l1 = L.clear_attn_fwd_strided(qc, kc, vc, wl.n_text, wl.H, wl.W, wl.r, window="square")
    o2, l2 = L.clear_attn_fwd_strided(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window="square")
    o3, l3 = L.clear_attn_fwd(qc, kc, vc, wl.n_text, wl.H, wl.W, wl.r, window="square")
    assert L.clear_attn_check() == 0
    assert torch.equal(o1, o3) and torch.equal(o2, o3) and torch.equal(l1, l3) and torch.equal(l2, l3)


def _call_raw(p, st):
    bufs = [np.full(4096, 0x5A, dtype=np.uint8) for _ in range(6)]
    ptrs = [ctypes.c_void_p(((b.ctypes.data + 15) // 16) * 16) for b in bufs]
    status = L.lib().clear_attn_fwd_strided(ctypes.byref(p), st, ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[4],
                                            ptrs[5], 4096, None)
    assert all((b[32:-32] == 0x5A).all() for b in bufs)  # nothing launched, host canaries untouched
    return L.status_string(status)


def test_strided_rejects_unaligned_or_missing_strides():
    p = L.make_params(1, 2, 16, 8, 8, 128, 2)
    T = 16 + 64
    good = (T * 2 * 128, T * 128, 128)
    mk = lambda s4: ctypes.byref(L.ClearStrides(*[(ctypes.c_longlong * 3)(*t) for t in s4]))
    assert _call_raw(p, None) == "CLEAR_ERR_INVALID_ARG"
    for bad in [(T * 2 * 128, T * 128, 132), (T * 2 * 128 + 4, T * 128, 128), (T * 2 * 128, 0, 128),
                (T * 2 * 128, -T * 128, 128)]:
        for which in range(4):
            s4 = [good] * 4
            s4[which] = bad
            assert _call_raw(p, mk(s4)) == "CLEAR_ERR_UNSUPPORTED", (which, bad)
