"""The forward from host buffers (clear_attn_fwd_host).

The library copies groups of (batch, head) slices from page-locked host memory to the device, runs
the forward on each group and copies o and lse back, on its own copy streams. Each group is an
ordinary forward call over independent slices, so the image rows must come out bit-identical to
one clear_attn_fwd call over all slices; the text rows (split partials merged by a second kernel)
are held to the usual bf16 tolerance. The oracle checks the small case directly.
"""
import pytest
import torch

import local_circular_window_b200 as L
import oracle
from clear_inputs import WORKLOADS, Workload, make_inputs
from gpu_util import LSE_ABS, assert_close


def _pinned_nan(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, pin_memory=True)


def _run_host(wl, hq, hk, hv, stream, ws=None, reps=1):
    ho = _pinned_nan(hq.shape, torch.bfloat16)
    hl = _pinned_nan((wl.B, wl.heads, wl.T), torch.float32)
    for _ in range(reps):  # later calls reuse the workspace while earlier copies may still run
        L.clear_attn_fwd_host(hq, hk, hv, wl.n_text, wl.H, wl.W, wl.r, o=ho, lse=hl, workspace=ws, stream=stream)
    stream.synchronize()
    assert L.clear_attn_check(stream) == 0
    return ho, hl


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [Workload("ragged_b2", 2, 3, 77, 24, 40, 128, 5),
                                Workload("b2_h13_d64", 2, 13, 40, 20, 20, 64, 6),  # 26 slices: groups of 2
                                WORKLOADS["flux1024_r16"], WORKLOADS["flux2048_r16"]], ids=lambda w: w.name)
def test_host_forward_matches_device_forward(wl):
    q, k, v = make_inputs(wl, seed=11, device="cuda")
    ref_o, ref_lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    ref_o, ref_lse = ref_o.cpu(), ref_lse.cpu()
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    del q, k, v
    stream = torch.cuda.Stream()
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    ws = torch.empty(L.fwd_host_workspace_size(p), dtype=torch.uint8, device="cuda")
    ho, hl = _run_host(wl, hq, hk, hv, stream, ws=ws, reps=2)
    n = wl.n_text
    assert torch.equal(ho[:, :, n:], ref_o[:, :, n:]), f"{wl.name}: image rows of O differ"
    assert torch.equal(hl[:, :, n:], ref_lse[:, :, n:]), f"{wl.name}: image rows of LSE differ"
    assert_close(ho[:, :, :n].float().numpy(), ref_o[:, :, :n].float().numpy(), f"{wl.name} text O")
    assert_close(hl[:, :, :n].numpy(), ref_lse[:, :, :n].numpy(), f"{wl.name} text LSE", max_abs=LSE_ABS,
                 mean_abs=LSE_ABS)
    del ws
    torch.cuda.empty_cache()


@pytest.mark.gpu
def test_host_forward_matches_oracle():
    wl = Workload("small_b2", 2, 2, 16, 16, 16, 128, 4)
    hq, hk, hv = (t.pin_memory() for t in make_inputs(wl, seed=5, device="cpu"))
    ho, hl = _run_host(wl, hq, hk, hv, torch.cuda.Stream())
    ref_o, ref_lse = oracle.clear_attention_forward(hq, hk, hv, wl.n_text, wl.H, wl.W, wl.r)
    assert_close(ho.float().numpy(), ref_o, "host fwd O")
    assert_close(hl.numpy(), ref_lse, "host fwd LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS)


@pytest.mark.gpu
def test_host_forward_rejects_pageable_buffers():
    # Pageable host memory cannot overlap with anything: rejected before any copy, outputs untouched.
    wl = Workload("small", 1, 2, 16, 16, 16, 128, 4)
    q, k, v = make_inputs(wl, seed=3, device="cpu")
    o = torch.full(q.shape, 7.0, dtype=torch.bfloat16)
    lse = torch.full((wl.B, wl.heads, wl.T), 7.0, dtype=torch.float32)
    with pytest.raises(L.ClearError) as e:
        L.clear_attn_fwd_host(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o, lse=lse)
    assert L.status_string(e.value.status) == "CLEAR_ERR_INVALID_ARG"
    po, pl = o.pin_memory(), lse.pin_memory()
    with pytest.raises(L.ClearError) as e:  # pinned outputs, pageable inputs
        L.clear_attn_fwd_host(q, k, v.pin_memory(), wl.n_text, wl.H, wl.W, wl.r, o=po, lse=pl)
    assert L.status_string(e.value.status) == "CLEAR_ERR_INVALID_ARG"
    with pytest.raises(L.ClearError) as e:  # pinned inputs, pageable lse
        L.clear_attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), wl.n_text, wl.H, wl.W, wl.r, o=po,
                              lse=lse)
    assert L.status_string(e.value.status) == "CLEAR_ERR_INVALID_ARG"
    torch.cuda.synchronize()
    for t in (o, lse, po, pl):
        assert (t == 7.0).all()
    assert L.clear_attn_check() == 0
