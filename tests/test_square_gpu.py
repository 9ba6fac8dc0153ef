"""GPU parity of the square-window variant (window="square": image pairs kept iff |dx| < r and
|dy| < r), forward and backward, against the float64 oracle with the same window. The kernels see
the window only through its half-width per vertical distance, so these runs exercise the same
scheduler, masks and pipelines as the circle with a different table."""
import numpy as np
import pytest
import torch

import oracle
from clear_inputs import WORKLOADS, Workload, make_inputs
from gpu_util import LSE_ABS, assert_close, gpu_inputs, sample_rows

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import local_circular_window_b200 as L

SQ = "square"

SMALL = [
    Workload("ragged_d128", 2, 3, 77, 24, 40, 128, 5),
    Workload("no_text", 1, 2, 0, 19, 21, 128, 3),
    Workload("wide_text_d64", 1, 2, 200, 13, 50, 64, 7),
    Workload("r1", 1, 2, 5, 9, 17, 128, 1),
    Workload("full_radius", 1, 2, 16, 16, 12, 64, 16),  # r = max(H, W): every pair kept
    Workload("text300_r16", 1, 2, 300, 32, 32, 128, 16),
]


def _fwd(wl, q, k, v):
    o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window=SQ)
    assert L.clear_attn_check() == 0
    return o, lse


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_square_forward_small_full_oracle(wl):
    q, k, v = gpu_inputs(wl, seed=0)
    o, lse = _fwd(wl, q, k, v)
    O, LSE = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r, window=SQ)
    assert_close(o.float().cpu().numpy(), O, f"square {wl.name} O")
    assert_close(lse.cpu().numpy(), LSE, f"square {wl.name} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS / 10)


@pytest.mark.parametrize("name", ["flux1024_r8", "flux1024_r16"])
def test_square_flux1024_heads_full_oracle(name):
    wl = WORKLOADS[name]
    q, k, v = gpu_inputs(wl, seed=0)
    o, lse = _fwd(wl, q, k, v)
    for h in (0, 11, 23):
        O, LSE = oracle.clear_attention_forward(q[:, h:h + 1].cpu(), k[:, h:h + 1].cpu(), v[:, h:h + 1].cpu(),
                                                wl.n_text, wl.H, wl.W, wl.r, window=SQ)
        assert_close(o[:, h:h + 1].float().cpu().numpy(), O, f"square {name} h{h} O")
        assert_close(lse[:, h:h + 1].cpu().numpy(), LSE, f"square {name} h{h} LSE", max_abs=LSE_ABS,
                     mean_abs=LSE_ABS / 10)


def test_square_8k_sampled_rows():
    wl = WORKLOADS["8k_r8"]
    q, k, v = make_inputs(wl, seed=0, device="cuda")
    o, lse = _fwd(wl, q, k, v)
    rows = sample_rows(wl, np.random.default_rng(1), n_interior=64, n_border=32, n_text=16)
    for h in (0, 23):
        Or, Lr = oracle.clear_attention_rows(q, k, v, wl.n_text, wl.H, wl.W, wl.r, 0, h, rows, window=SQ)
        assert_close(o[0, h, rows].float().cpu().numpy(), Or, f"square 8k h{h} O")
        assert_close(lse[0, h, rows].cpu().numpy(), Lr, f"square 8k h{h} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS)
    del q, k, v, o, lse
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wl", [SMALL[0], SMALL[2], SMALL[4],
                                Workload("bwd_square_r16", 2, 3, 512, 64, 64, 128, 16)], ids=lambda w: w.name)
def test_square_backward_full_oracle(wl):
    q, k, v, dO = gpu_inputs(wl, seed=0, grad=True)
    o, lse = _fwd(wl, q, k, v)
    dq, dk, dv = L.clear_attn_bwd(q, k, v, o, lse, dO, wl.n_text, wl.H, wl.W, wl.r, window=SQ)
    assert L.clear_attn_check() == 0
    rq, rk, rv = oracle.clear_attention_backward(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), wl.n_text, wl.H, wl.W, wl.r,
                                                 window=SQ)
    assert_close(dq.float().cpu().numpy(), rq, f"square {wl.name} dQ")
    assert_close(dk.float().cpu().numpy(), rk, f"square {wl.name} dK")
    assert_close(dv.float().cpu().numpy(), rv, f"square {wl.name} dV")


# ------------------------------------------------------------------------------------------------
# Border-shifted square window (window="shifted"): forward only.
# ------------------------------------------------------------------------------------------------

SHIFTED = [
    Workload("sh_ragged_d128", 2, 3, 77, 24, 40, 128, 5),
    Workload("sh_no_text", 1, 2, 0, 19, 21, 128, 3),
    Workload("sh_wide_text_d64", 1, 2, 200, 13, 50, 64, 7),
    Workload("sh_window_is_grid", 1, 2, 16, 15, 15, 64, 8),  # 2r - 1 = 15: every window is the grid
    Workload("sh_text300_r16", 1, 2, 300, 32, 32, 128, 16),
]


@pytest.mark.parametrize("wl", SHIFTED, ids=lambda w: w.name)
def test_shifted_forward_small_full_oracle(wl):
    q, k, v = gpu_inputs(wl, seed=0)
    o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window="shifted")
    assert L.clear_attn_check() == 0
    O, LSE = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r,
                                            window="shifted")
    assert_close(o.float().cpu().numpy(), O, f"shifted {wl.name} O")
    assert_close(lse.cpu().numpy(), LSE, f"shifted {wl.name} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS / 10)


def test_shifted_flux1024_and_8k_sampled():
    for name in ("flux1024_r8", "8k_r8"):
        wl = WORKLOADS[name]
        q, k, v = make_inputs(wl, seed=0, device="cuda")
        o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window="shifted")
        assert L.clear_attn_check() == 0
        rows = sample_rows(wl, np.random.default_rng(2), n_interior=64, n_border=48, n_text=16)
        for h in (0, 23):
            Or, Lr = oracle.clear_attention_rows(q, k, v, wl.n_text, wl.H, wl.W, wl.r, 0, h, rows, window="shifted")
            assert_close(o[0, h, rows].float().cpu().numpy(), Or, f"shifted {name} h{h} O")
            assert_close(lse[0, h, rows].cpu().numpy(), Lr, f"shifted {name} h{h} LSE", max_abs=LSE_ABS,
                         mean_abs=LSE_ABS)
        del q, k, v, o, lse
        torch.cuda.empty_cache()


def test_shifted_backward_is_unsupported():
    wl = SHIFTED[1]
    q, k, v, dO = gpu_inputs(wl, seed=0, grad=True)
    o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window="shifted")
    with pytest.raises(L.ClearError) as e:
        L.clear_attn_bwd(q, k, v, o, lse, dO, wl.n_text, wl.H, wl.W, wl.r, window="shifted")
    assert "CLEAR_ERR_UNSUPPORTED" in str(e.value)
    assert L.clear_attn_check() == 0
