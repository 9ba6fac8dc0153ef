"""Failure detection on the GPU without a fault.

Every wait in the kernels is bounded: on expiry it records the site in a device error word and the
kernel returns, so a stuck pipeline surfaces as CLEAR_ERR_DEVICE_TIMEOUT from clear_attn_check()
instead of a hung GPU. clear_attn_selftest_expiry makes one such wait run out on purpose (it waits
on a barrier nothing arrives on, for a caller-chosen 100 ms) and these tests check that the host
sees it, that the report is cleared after reading, and that the context still runs attention.
"""
import pytest
import torch

import local_circular_window_b200 as L
from clear_inputs import Workload, make_inputs


@pytest.mark.gpu
def test_expired_wait_is_reported_and_context_survives():
    wl = Workload("small", 1, 2, 40, 16, 24, 128, 4)
    q, k, v = make_inputs(wl, seed=3, device="cuda")
    o_ref, lse_ref = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0

    assert L.selftest_expiry(100) == 0
    assert L.status_string(L.clear_attn_check()) == "CLEAR_ERR_DEVICE_TIMEOUT"
    diag = L.device_diag()
    assert diag[0] == 5 and diag[1] == 31 and diag[5] == 100  # code, wait site, limit in ms
    assert L.clear_attn_check() == 0  # reading the report cleared it

    o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)  # the forward is deterministic
