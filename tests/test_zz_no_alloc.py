"""The allocation-free forward (clear_attn_fwd_noalloc).

It serves callers that cannot call cudaMalloc or pass a workspace, for example a plugin running
inside another framework's execution step, or a serving loop that reserved all device memory up
front. It takes its scratch from a fixed array compiled into the library, so its results must
match clear_attn_fwd's (within the usual bf16 tolerance: only the text rows' split count, hence
their summation order, may differ), call after call, since every call reuses that array.

This file is collected last on purpose, so a stop-at-first-failure run has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import local_circular_window_b200 as L
import oracle
from clear_inputs import WORKLOADS, Workload, make_inputs
from gpu_util import LSE_ABS, assert_close, gpu_inputs


def _noalloc(wl, q, k, v):
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((wl.B, wl.heads, wl.T), float("nan"), dtype=torch.float32, device=q.device)
    st = L.lib().clear_attn_fwd_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.status_string(st)
    assert L.clear_attn_check() == 0
    return o, lse


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [Workload("ragged", 1, 3, 77, 24, 40, 128, 5), WORKLOADS["flux1024_r16"],
                                WORKLOADS["8k_r8"]], ids=lambda w: w.name)
def test_noalloc_matches_fwd_on_consecutive_calls(wl):
    q, k, v = make_inputs(wl, seed=7, device="cuda")
    ref_o, ref_lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        o, lse = _noalloc(wl, q, k, v)
        assert_close(o.float().cpu().numpy(), ref_o.float().cpu().numpy(), f"{wl.name} O")
        assert_close(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"{wl.name} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS)
    del q, k, v
    torch.cuda.empty_cache()


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [Workload("no_text", 1, 2, 0, 16, 24, 128, 4), Workload("d64", 1, 2, 20, 16, 24, 64, 4)],
                         ids=lambda w: w.name)
def test_noalloc_no_text_and_d64(wl):
    # Without text tokens the call needs no scratch at all; with d = 64 it runs the other kernel
    # instantiation. Both must equal clear_attn_fwd on two calls in a row, and the oracle.
    q, k, v = gpu_inputs(wl, seed=11)
    ref_o, ref_lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    O, LSE = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    for _ in range(2):
        o, lse = _noalloc(wl, q, k, v)
        assert_close(o.float().cpu().numpy(), ref_o.float().cpu().numpy(), f"{wl.name} O vs fwd")
        assert_close(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"{wl.name} LSE vs fwd", max_abs=LSE_ABS,
                     mean_abs=LSE_ABS)
        assert_close(o.float().cpu().numpy(), O, f"{wl.name} O vs oracle")
        assert_close(lse.cpu().numpy(), LSE, f"{wl.name} LSE vs oracle", max_abs=LSE_ABS, mean_abs=LSE_ABS / 10)


@pytest.mark.gpu
@pytest.mark.parametrize("window", ["square", "shifted"])
def test_noalloc_window_variants_match_fwd(window):
    wl = Workload("ragged", 1, 3, 77, 24, 40, 128, 5)
    q, k, v = make_inputs(wl, seed=8, device="cuda")
    ref_o, ref_lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, window=window)
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r, window)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((wl.B, wl.heads, wl.T), float("nan"), dtype=torch.float32, device=q.device)
    st = L.lib().clear_attn_fwd_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.status_string(st)
    assert L.clear_attn_check() == 0
    assert_close(o.float().cpu().numpy(), ref_o.float().cpu().numpy(), f"noalloc {window} O")
    assert_close(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"noalloc {window} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # One split of 1024 heads x 4096 text rows needs 1024 * 4096 * (4 * 128 + 8) bytes > 32 MiB:
    # rejected on the host before anything is launched (host canaries stay untouched).
    p = L.make_params(1, 1024, 4096, 8, 8, 128, 2)
    bufs = [np.full(4096, 0x5A, dtype=np.uint8) for _ in range(5)]
    ptrs = [ctypes.c_void_p(b.ctypes.data) for b in bufs]
    st = L.lib().clear_attn_fwd_noalloc(ctypes.byref(p), *ptrs, None)
    assert L.status_string(st) == "CLEAR_ERR_WORKSPACE"
    assert all((b == 0x5A).all() for b in bufs)
