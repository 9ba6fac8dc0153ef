"""GPU parity of the backward (clear_attn_bwd through the C ABI) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from clear_inputs import WORKLOADS, Workload
from gpu_util import assert_close, gpu_inputs

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import local_circular_window_b200 as L


def _fwd_bwd(wl, q, k, v, dO):
    o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    dq, dk, dv = L.clear_attn_bwd(q, k, v, o, lse, dO, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    return dq, dk, dv


SMALL = [
    Workload("tiny", 1, 2, 16, 16, 16, 64, 4),
    Workload("ragged_d128", 1, 2, 77, 24, 40, 128, 5),
    Workload("no_text", 1, 2, 0, 19, 21, 128, 3),
    Workload("text300_r16", 1, 1, 300, 32, 32, 128, 16),
    Workload("full_radius_d64", 1, 2, 16, 16, 16, 64, 22),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_backward_small_full_oracle(wl):
    q, k, v, dO = gpu_inputs(wl, seed=0, grad=True)
    dq, dk, dv = _fwd_bwd(wl, q, k, v, dO)
    rq, rk, rv = oracle.clear_attention_backward(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    assert_close(dq.float().cpu().numpy(), rq, f"{wl.name} dQ")
    assert_close(dk.float().cpu().numpy(), rk, f"{wl.name} dK")
    assert_close(dv.float().cpu().numpy(), rv, f"{wl.name} dV")


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_backward_distillation_config(seed):
    wl = WORKLOADS["bwd_flux1024_r32"]
    q, k, v, dO = gpu_inputs(wl, seed=seed, grad=True)
    dq, dk, dv = _fwd_bwd(wl, q, k, v, dO)
    for b, h in ((0, 0), (1, 11), (0, 23)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = oracle.clear_attention_backward(q[sl].cpu(), k[sl].cpu(), v[sl].cpu(), dO[sl].cpu(),
                                                     wl.n_text, wl.H, wl.W, wl.r)
        assert_close(dq[sl].float().cpu().numpy(), rq, f"bwd s{seed} b{b}h{h} dQ")
        assert_close(dk[sl].float().cpu().numpy(), rk, f"bwd s{seed} b{b}h{h} dK")
        assert_close(dv[sl].float().cpu().numpy(), rv, f"bwd s{seed} b{b}h{h} dV")


def test_backward_text_splits():
    wl = Workload("split2", 1, 1, 130, 96, 96, 128, 6)
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    assert L.forward_shape(p)[2] >= 2
    q, k, v, dO = gpu_inputs(wl, seed=4, grad=True)
    dq, dk, dv = _fwd_bwd(wl, q, k, v, dO)
    # T = 9346: the full oracle backward is one 9346^2 head in float64 (about 0.7 GB per matrix).
    rq, rk, rv = oracle.clear_attention_backward(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    assert_close(dq.float().cpu().numpy(), rq, "split2 dQ")
    assert_close(dk.float().cpu().numpy(), rk, "split2 dK")
    assert_close(dv.float().cpu().numpy(), rv, "split2 dV")
