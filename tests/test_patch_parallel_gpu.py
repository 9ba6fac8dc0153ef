"""Patch-parallel kernels on one GPU: the stripe forward (clear_attn_fwd_stripe) and the text-row
merge (clear_attn_text_merge) against the oracle, and a whole split computed stripe after stripe
(patch_parallel.forward_by_stripes), which runs every rank's kernels in turn:
* exact mode equals the full-problem oracle forward on every row;
* eq7 mode gives the oracle's patch-wise text average (Eq. 7) on the text rows."""
import numpy as np
import pytest
import torch

import local_circular_window_b200 as L
import oracle
from local_circular_window_b200 import patch_parallel as pp
from clear_inputs import Workload, make_inputs
from gpu_util import LSE_ABS, assert_close, gpu_inputs


def _np(t):
    return t.float().cpu().numpy()


STRIPES = [
    # (n_text, H, W, d, r, window, q_row0, q_row1, key_row0, key_row1, text_keys)
    (77, 40, 24, 128, 5, "circle", 4, 36, 4, 36, 1),      # interior stripe, 4-row halos
    (77, 40, 24, 128, 5, "circle", 4, 36, 4, 36, 0),      # exact mode, rank > 0: no text keys
    (30, 37, 19, 128, 4, "square", 0, 34, 0, 34, 1),      # top stripe: no top halo, ragged rows
    (30, 37, 19, 64, 4, "circle", 3, 37, 3, 37, 0),       # bottom stripe, d = 64
    (16, 21, 33, 128, 2, "circle", 1, 20, 0, 0, 1),       # text rows see the text keys only
    (0, 29, 17, 128, 3, "circle", 2, 27, 2, 27, 0),       # no text tokens
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", STRIPES, ids=lambda c: "-".join(map(str, c)))
def test_stripe_forward_matches_oracle(case):
    n_text, H, W, d, r, window, q0, q1, k0, k1, tk = case
    wl = Workload("stripe", 2, 3, n_text, H, W, d, r)
    q, k, v = gpu_inputs(wl, seed=41)
    st = L.make_stripe(q0, q1, k0, k1, bool(tk))
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    L.clear_attn_fwd_stripe(q, k, v, n_text, H, W, r, st, o=o, lse=lse, window=window)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    Ot, Lt, Oi, Li = oracle.clear_attention_stripe(q, k, v, n_text, H, W, r, q0, q1, k0, k1, bool(tk), window=window)
    a, b = n_text + q0 * W, n_text + q1 * W
    assert_close(_np(o[:, :, a:b]), Oi, "image rows")
    assert np.abs(_np(lse[:, :, a:b]) - Li).max() <= LSE_ABS
    if n_text:
        assert_close(_np(o[:, :, :n_text]), Ot, "text rows")
        assert np.abs(_np(lse[:, :, :n_text]) - Lt).max() <= LSE_ABS
    # Halo rows are not written.
    assert torch.isnan(o[:, :, n_text:a].float()).all() and torch.isnan(o[:, :, b:].float()).all()
    assert torch.isnan(lse[:, :, n_text:a]).all() and torch.isnan(lse[:, :, b:]).all()


@pytest.mark.gpu
def test_stripe_forward_rejects_bad_stripes():
    wl = Workload("bad", 1, 2, 8, 12, 10, 128, 3)
    q, k, v = gpu_inputs(wl, seed=42)
    with pytest.raises(L.ClearError) as e:
        L.clear_attn_fwd_stripe(q, k, v, 8, 12, 10, 3, L.make_stripe(2, 10, 2, 10, True), window="shifted")
    assert e.value.status == 2  # unsupported
    for st in (L.make_stripe(5, 5, 0, 12, True), L.make_stripe(0, 13, 0, 12, True), L.make_stripe(0, 12, 3, 2, True),
               L.make_stripe(0, 12, 0, 0, False)):
        with pytest.raises(L.ClearError) as e:
            L.clear_attn_fwd_stripe(q, k, v, 8, 12, 10, 3, st)
        assert e.value.status == 1  # invalid argument
    assert L.clear_attn_check() == 0


def _merge_f64(o_parts, lse_parts, mode):
    o_parts, lse_parts = o_parts.astype(np.float64), lse_parts.astype(np.float64)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m)
    lse = m + np.log(w.sum(axis=0))
    if mode == "exact":
        return (w[..., None] * o_parts).sum(axis=0) / w.sum(axis=0)[..., None], lse
    return o_parts.mean(axis=0), lse


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["exact", "eq7"])
@pytest.mark.parametrize("parts,d", [(1, 128), (3, 128), (8, 64)])
def test_text_merge_matches_definition(mode, parts, d):
    g = torch.Generator().manual_seed(7 + parts)
    o_parts = torch.randn((parts, 2, 3, 45, d), generator=g).to(torch.bfloat16)
    lse_parts = (torch.randn((parts, 2, 3, 45), generator=g) * 4.0).float()
    if parts > 1:
        lse_parts[1, 0, 0, :7] = float("-inf")  # a part without keys for some rows: weight 0
    o, lse = L.clear_attn_text_merge(o_parts.cuda(), lse_parts.cuda(), mode)
    torch.cuda.synchronize()
    ref_o, ref_l = _merge_f64(o_parts.float().numpy(), lse_parts.numpy(), mode)
    assert np.abs(_np(o) - ref_o).max() <= 8e-3  # one bf16 rounding of |o| < 8
    assert np.abs(_np(lse) - ref_l).max() <= 1e-5 * max(1.0, np.abs(ref_l).max())


@pytest.mark.gpu
@pytest.mark.parametrize("stripes,wl", [
    (2, Workload("pp2", 1, 4, 77, 40, 24, 128, 5)),
    (3, Workload("pp3_square", 2, 2, 30, 37, 19, 128, 4)),
    (4, Workload("pp4_d64", 1, 3, 64, 64, 32, 64, 8)),
], ids=lambda x: x if isinstance(x, int) else x.name)
@pytest.mark.parametrize("window", ["circle", "square"])
def test_forward_by_stripes_exact_is_the_full_forward(stripes, wl, window):
    q, k, v = gpu_inputs(wl, seed=43)
    o, lse = pp.forward_by_stripes(q, k, v, wl.n_text, wl.H, wl.W, wl.r, stripes, mode="exact", window=window)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    O, Lse = oracle.clear_attention_forward(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window=window)
    assert_close(_np(o), O, "all rows")
    assert np.abs(_np(lse) - Lse).max() <= LSE_ABS


@pytest.mark.gpu
def test_forward_by_stripes_eq7_text_rows():
    wl = Workload("pp_eq7", 1, 3, 40, 36, 20, 128, 4)
    q, k, v = gpu_inputs(wl, seed=44)
    o, lse = pp.forward_by_stripes(q, k, v, wl.n_text, wl.H, wl.W, wl.r, 3, mode="eq7")
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    edges = [lo for lo, _ in pp.stripe_bounds(wl.H, 3)] + [wl.H]
    ref = oracle.clear_text_rows_patch_average(q, k, v, wl.n_text, wl.H, wl.W, edges)
    assert_close(_np(o[:, :, :wl.n_text]), ref, "eq7 text rows")
    O, _ = oracle.clear_attention_forward(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert_close(_np(o[:, :, wl.n_text:]), O[:, :, wl.n_text:], "image rows")


@pytest.mark.gpu
def test_forward_by_stripes_flux1024_sampled():
    # The FLUX 1024^2 call (64 x 64 grid, 512 text tokens, 24 heads, r = 16) over 4 stripes, checked
    # on every text row and a sample of image rows near the stripe boundaries.
    wl = Workload("flux1024_r16", 1, 24, 512, 64, 64, 128, 16)
    q, k, v = gpu_inputs(wl, seed=45)
    o, lse = pp.forward_by_stripes(q, k, v, wl.n_text, wl.H, wl.W, wl.r, 4, mode="exact")
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    rows = list(range(0, 512, 7)) + [512 + y * 64 + x for y in (0, 15, 16, 31, 32, 47, 48, 63) for x in (0, 17, 63)]
    for h in (0, 11, 23):
        Or, Lr = oracle.clear_attention_rows(q, k, v, wl.n_text, wl.H, wl.W, wl.r, 0, h, rows)
        assert_close(_np(o[0, h, rows]), Or, f"head {h}")
        assert np.abs(_np(lse[0, h, rows]) - Lr).max() <= LSE_ABS
