"""GPU parity of the FP8-score forward (clear_attn_fwd_fp8: E4M3 q and k, bf16 v) against the
oracle's FP8 forward, which decodes the same codes exactly. Everything after the scores matches the
bf16 forward, so the bf16 tolerance applies."""
import numpy as np
import pytest
import torch

import oracle
from clear_inputs import Workload, make_inputs, quantize_e4m3
from gpu_util import LSE_ABS, assert_close, sample_rows

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import local_circular_window_b200 as L


def _fp8_inputs(wl, seed, device="cpu"):
    q, k, v = make_inputs(wl, seed=seed, dtype=torch.float32, device=device)
    q8, sq = quantize_e4m3(q)
    k8, sk = quantize_e4m3(k)
    return q8, k8, v.to(torch.bfloat16), sq, sk


def _run(wl, q8, k8, v, sq, sk, window="circle"):
    desc = (sq * sk).float().contiguous().cuda()
    o, lse = L.clear_attn_fwd_fp8(q8.cuda(), k8.cuda(), v.cuda(), desc, wl.n_text, wl.H, wl.W, wl.r, window=window)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    return o, lse


SMALL = [
    Workload("f8_ragged", 2, 3, 77, 24, 40, 128, 5),
    Workload("f8_no_text", 1, 2, 0, 19, 21, 128, 3),
    Workload("f8_text300_r16", 1, 2, 300, 32, 32, 128, 16),
    Workload("f8_full_radius", 1, 2, 16, 16, 16, 128, 22),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_fp8_forward_small_full_oracle(wl):
    q8, k8, v, sq, sk = _fp8_inputs(wl, seed=61)
    o, lse = _run(wl, q8, k8, v, sq, sk)
    O, LSE = oracle.clear_attention_forward_fp8(q8, k8, v, sq, sk, wl.n_text, wl.H, wl.W, wl.r)
    assert_close(o.float().cpu().numpy(), O, f"{wl.name} O")
    assert np.abs(lse.cpu().numpy() - LSE).max() <= LSE_ABS


def test_fp8_forward_square_window_and_text_splits():
    # Square window; T > 8192 so the text rows are split over several key ranges and merged.
    wl = Workload("f8_split", 1, 2, 200, 96, 96, 128, 6)
    q8, k8, v, sq, sk = _fp8_inputs(wl, seed=62)
    o, lse = _run(wl, q8, k8, v, sq, sk, window="square")
    rows = sample_rows(wl, np.random.default_rng(3), n_text=64)
    for h in range(2):
        qd = oracle.e4m3_decode(q8[0, h].numpy()) * float(sq[0, h])
        kd = oracle.e4m3_decode(k8[0, h].numpy()) * float(sk[0, h])
        Or, Lr = oracle.clear_attention_rows(qd[None, None], kd[None, None], v[0:1, h:h + 1].double().numpy(),
                                             wl.n_text, wl.H, wl.W, wl.r, 0, 0, rows, window="square")
        assert_close(o[0, h, rows].float().cpu().numpy(), Or, f"head {h}")
        assert np.abs(lse[0, h, rows].cpu().numpy() - Lr).max() <= LSE_ABS


def test_fp8_forward_flux1024_r16():
    wl = Workload("flux1024_r16", 1, 24, 512, 64, 64, 128, 16)
    q8, k8, v, sq, sk = _fp8_inputs(wl, seed=63)
    o, lse = _run(wl, q8, k8, v, sq, sk)
    for h in (0, 11, 23):
        O, LSE = oracle.clear_attention_forward_fp8(q8[:, h:h + 1], k8[:, h:h + 1], v[:, h:h + 1], sq[:, h:h + 1],
                                                    sk[:, h:h + 1], wl.n_text, wl.H, wl.W, wl.r)
        assert_close(o[:, h:h + 1].float().cpu().numpy(), O, f"head {h}")
        assert np.abs(lse[:, h:h + 1].cpu().numpy() - LSE).max() <= LSE_ABS


def test_fp8_rejects_d64_and_bad_descale():
    wl = Workload("f8_d64", 1, 1, 4, 8, 8, 64, 2)
    q8 = torch.zeros((1, 1, wl.T, 64), dtype=torch.uint8, device="cuda")
    v = torch.zeros((1, 1, wl.T, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.ClearError) as e:
        L.clear_attn_fwd_fp8(q8, q8, v, torch.ones(1, device="cuda"), 4, 8, 8, 2)
    assert e.value.status == 2
    assert L.clear_attn_check() == 0
