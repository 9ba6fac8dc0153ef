"""Pins of the oracle's FP8 (E4M3) functions: the format decoder against torch's float8_e4m3fn
conversion for all 256 codes and against hand-worked values of the format definition, and the FP8
forward against the plain forward on the decoded inputs, with a scale invariance and a mutant."""
import numpy as np
import pytest
import torch

import oracle
from clear_inputs import Workload, make_inputs, quantize_e4m3


def test_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all() and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x80, -0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x3C, 1.5), (0xC0, -2.0), (0x7E, 448.0), (0xFE, -448.0), (0x77, 240.0),
])
def test_decode_worked_values(code, value):
    # sign | exponent (bias 7) | mantissa: 0x38 = 0|0111|000 = 1.0; 0x7E = 0|1111|110 = 2^8 * 1.75 = 448;
    # 0x01 = smallest subnormal 2^-6 * 1/8; 0x77 = 0|1110|111 = 2^7 * 1.875 = 240.
    got = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
    assert got == value and np.signbit(got) == np.signbit(value)


def _fp8_inputs(wl, seed):
    q, k, v = make_inputs(wl, seed=seed, dtype=torch.float32)
    q8, sq = quantize_e4m3(q)
    k8, sk = quantize_e4m3(k)
    return q8, k8, v.to(torch.bfloat16), sq, sk


def test_fp8_forward_is_the_plain_forward_of_decoded_inputs():
    wl = Workload("f8", 2, 2, 5, 6, 7, 16, 3)
    q8, k8, v, sq, sk = _fp8_inputs(wl, 3)
    O, L = oracle.clear_attention_forward_fp8(q8, k8, v, sq, sk, 5, 6, 7, 3)
    qd = torch.from_numpy(q8.numpy()).view(torch.float8_e4m3fn).double() * sq.double()[:, :, None, None]
    kd = torch.from_numpy(k8.numpy()).view(torch.float8_e4m3fn).double() * sk.double()[:, :, None, None]
    O2, L2 = oracle.clear_attention_forward(qd, kd, v, 5, 6, 7, 3)
    assert np.abs(O - O2).max() < 1e-12 and np.abs(L - L2).max() < 1e-12


def test_fp8_forward_scale_invariance_and_mutant():
    # Only the product s_q * s_k enters the scores: moving a factor between them changes nothing,
    # while dropping s_k (a plausible mistake) does.
    wl = Workload("f8", 1, 2, 4, 5, 5, 16, 2)
    q8, k8, v, sq, sk = _fp8_inputs(wl, 4)
    O, _ = oracle.clear_attention_forward_fp8(q8, k8, v, sq, sk, 4, 5, 5, 2)
    O2, _ = oracle.clear_attention_forward_fp8(q8, k8, v, sq * 4.0, sk / 4.0, 4, 5, 5, 2)
    O3, _ = oracle.clear_attention_forward_fp8(q8, k8, v, sq, torch.ones_like(sk), 4, 5, 5, 2)
    assert np.abs(O - O2).max() < 1e-12
    assert np.abs(O - O3).max() > 1e-3


def test_quantization_error_is_within_half_an_e4m3_step():
    # The input encoding: decode(code) * scale is within 2^-4 relative (half a mantissa step) of the
    # value for normal codes, so the FP8 path computes scores of inputs this close to the bf16 ones.
    wl = Workload("f8", 1, 3, 8, 6, 6, 64, 3)
    q, _, _ = make_inputs(wl, seed=5, dtype=torch.float32)
    q8, sq = quantize_e4m3(q)
    dec = oracle.e4m3_decode(q8.numpy()) * sq.double().numpy()[:, :, None, None]
    qn = q.double().numpy()
    normal = np.abs(dec) >= 2.0 ** -6 * sq.double().numpy()[:, :, None, None]
    rel = np.abs(dec - qn)[normal] / np.abs(qn)[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-12
