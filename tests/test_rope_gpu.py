"""GPU parity of the forward on rotary-embedded q and k (clear_attn_fwd_rope) against the oracle's
RoPE forward (q and k rotated in float64, then the plain forward).

The rotation pass works in fp32 and stores the rotated q and k as bf16 for the score products, so
they are rounded to bf16 once more. Two checks follow from that:
  * at operand precision: the oracle's float64 rotation rounded to bf16 on the CPU, then the plain
    oracle forward, held to the standard bf16 bar;
  * against the float64 rotation: the extra rounding (unit roundoff u = 2^-8, error at most u|x|
    and spread evenly, standard deviation <= u|x|/sqrt(3)) moves a scaled score q.k/sqrt(d) of
    unit-normal q, k by sigma_s = u*sqrt(2/3), whatever d; the LSE moves by a softmax-weighted mean
    of those moves, never more than the largest, so it is held to LSE_ABS + 6 sigma_s."""
import math

import numpy as np
import pytest
import torch

import oracle
from clear_inputs import WORKLOADS, Workload
from gpu_util import LSE_ABS, MAX_ABS, MEAN_ABS, assert_close, gpu_inputs, sample_rows

pytestmark = pytest.mark.gpu

ROPE_LSE_ABS = LSE_ABS + 6 * 2.0 ** -8 * math.sqrt(2.0 / 3.0)


def rotated_bf16(x, n_text, H, W, theta, ntk):
    """The oracle's float64 rotation, rounded to bf16 on the CPU (the score products' operand type)."""
    return torch.from_numpy(oracle.rope_2d(x, n_text, H, W, theta, ntk)).to(torch.bfloat16)

if torch.cuda.is_available():
    import local_circular_window_b200 as L

SMALL = [
    (Workload("rope_ragged", 2, 3, 77, 24, 40, 128, 5), 10000.0, 10.0, "circle"),
    (Workload("rope_no_text", 1, 2, 0, 19, 21, 128, 3), 10000.0, 1.0, "circle"),
    (Workload("rope_d64", 1, 2, 200, 13, 50, 64, 7), 10000.0, 10.0, "square"),
    (Workload("rope_text300", 1, 2, 300, 32, 32, 128, 16), 500.0, 2.0, "circle"),
    (Workload("rope_shifted", 1, 2, 16, 20, 20, 128, 4), 10000.0, 10.0, "shifted"),
]


@pytest.mark.parametrize("wl,theta,ntk,window", SMALL, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_rope_forward_small_full_oracle(wl, theta, ntk, window):
    q, k, v = gpu_inputs(wl, seed=71)
    q0, k0 = q.clone(), k.clone()
    o, lse = L.clear_attn_fwd_rope(q, k, v, wl.n_text, wl.H, wl.W, wl.r, theta=theta, ntk=ntk, window=window)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    assert torch.equal(q, q0) and torch.equal(k, k0)  # the inputs are not modified
    got_o, got_lse = o.float().cpu().numpy(), lse.cpu().numpy()
    qb = rotated_bf16(q.cpu(), wl.n_text, wl.H, wl.W, theta, ntk)
    kb = rotated_bf16(k.cpu(), wl.n_text, wl.H, wl.W, theta, ntk)
    O, LSE = oracle.clear_attention_forward(qb, kb, v.cpu(), wl.n_text, wl.H, wl.W, wl.r, window=window)
    assert_close(got_o, O, f"{wl.name} O (bf16 operands)")
    assert np.abs(got_lse - LSE).max() <= LSE_ABS
    O64, LSE64 = oracle.clear_attention_forward_rope(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r,
                                                     theta=theta, ntk=ntk, window=window)
    assert_close(got_o, O64, f"{wl.name} O (float64 rotation)", max_abs=MAX_ABS, mean_abs=MEAN_ABS)
    assert np.abs(got_lse - LSE64).max() <= ROPE_LSE_ABS


def test_rope_forward_flux2048_sampled_rows():
    # FLUX 2048^2 call (128 x 128 grid, 512 text tokens, r=16) with the review's NTK factor 10:
    # every text split merged, rows sampled across the grid and its borders.
    wl = WORKLOADS["flux2048_r16"]
    q, k, v = gpu_inputs(wl, seed=72)
    o, lse = L.clear_attn_fwd_rope(q, k, v, wl.n_text, wl.H, wl.W, wl.r, ntk=10.0)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    rows = sample_rows(wl, np.random.default_rng(4), n_text=24)
    for h in (0, 13):
        qh, kh, vh = q[0:1, h:h + 1].cpu(), k[0:1, h:h + 1].cpu(), v[0:1, h:h + 1].cpu()
        got_o, got_lse = o[0, h, rows].float().cpu().numpy(), lse[0, h, rows].cpu().numpy()
        qb = rotated_bf16(qh, wl.n_text, wl.H, wl.W, 10000.0, 10.0)
        kb = rotated_bf16(kh, wl.n_text, wl.H, wl.W, 10000.0, 10.0)
        Ob, Lb = oracle.clear_attention_rows(qb, kb, vh, wl.n_text, wl.H, wl.W, wl.r, 0, 0, rows)
        assert_close(got_o, Ob, f"head {h} (bf16 operands)")
        assert np.abs(got_lse - Lb).max() <= LSE_ABS
        qr = oracle.rope_2d(qh, wl.n_text, wl.H, wl.W, ntk=10.0)
        kr = oracle.rope_2d(kh, wl.n_text, wl.H, wl.W, ntk=10.0)
        Or, Lr = oracle.clear_attention_rows(qr, kr, vh.double().numpy(), wl.n_text, wl.H, wl.W, wl.r, 0, 0, rows)
        assert_close(got_o, Or, f"head {h} (float64 rotation)")
        assert np.abs(got_lse - Lr).max() <= ROPE_LSE_ABS


def test_rope_rejects_bad_parameters():
    wl = Workload("rope_bad", 1, 1, 4, 8, 8, 128, 2)
    q, k, v = gpu_inputs(wl, seed=73)
    for theta, ntk in ((1.0, 1.0), (10000.0, 0.0), (float("nan"), 1.0)):
        with pytest.raises(L.ClearError) as e:
            L.clear_attn_fwd_rope(q, k, v, 4, 8, 8, 2, theta=theta, ntk=ntk)
        assert e.value.status == 1
    assert L.clear_attn_check() == 0


# The rotation alone (clear_attn_rope): the exact rotation rounded to bf16. bf16 keeps 8 significant
# bits, so rounding moves a value v by at most 2^-8 |v|; the fp32 arithmetic and table add at most
# ~2^-20 of the operands (inputs are unit normal: an absolute 1e-5 covers it).
def _assert_rotated(got, ref, what):
    got = got.double().cpu().numpy()
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5
    assert (err <= bound).all(), f"{what}: worst excess {(err - bound).max():.3e}"


ROT = [
    (Workload("rot_ragged", 2, 3, 77, 24, 40, 128, 1), 10000.0, 10.0),
    (Workload("rot_d64", 1, 2, 200, 13, 50, 64, 1), 500.0, 1.0),
    (Workload("rot_no_text", 1, 2, 0, 19, 21, 128, 1), 10000.0, 2.0),
]


@pytest.mark.parametrize("wl,theta,ntk", ROT, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_rope_rotation_alone(wl, theta, ntk):
    q, k, _ = gpu_inputs(wl, seed=73)
    for inverse in (False, True):
        qr, kr = L.clear_attn_rope(q, k, wl.n_text, wl.H, wl.W, theta=theta, ntk=ntk, inverse=inverse)
        torch.cuda.synchronize()
        for name, x, xr in (("q", q, qr), ("k", k, kr)):
            ref = oracle.rope_2d(x.cpu(), wl.n_text, wl.H, wl.W, theta, ntk, inverse=inverse)
            _assert_rotated(xr, ref, f"{wl.name} {name} inverse={inverse}")
            assert torch.equal(xr[:, :, :wl.n_text], x[:, :, :wl.n_text])  # text tokens are copied
    # in place equals out of place, and the inverse undoes the rotation up to two bf16 roundings
    q2, k2 = q.clone(), k.clone()
    L.clear_attn_rope(q2, k2, wl.n_text, wl.H, wl.W, theta=theta, ntk=ntk, q_out=q2, k_out=k2)
    qr, kr = L.clear_attn_rope(q, k, wl.n_text, wl.H, wl.W, theta=theta, ntk=ntk)
    torch.cuda.synchronize()
    assert torch.equal(q2, qr) and torch.equal(k2, kr)
    qb, _ = L.clear_attn_rope(qr, kr, wl.n_text, wl.H, wl.W, theta=theta, ntk=ntk, inverse=True)
    torch.cuda.synchronize()
    back = qb.double().cpu().numpy()
    x0 = q.double().cpu().numpy()
    # each rounding moves a pair by at most 2^-8 of its norm, and the rotations keep norms
    pair_norm = np.repeat(np.sqrt(x0[..., 0::2] ** 2 + x0[..., 1::2] ** 2), 2, axis=-1)
    assert (np.abs(back - x0) <= 2.0 ** -7 * pair_norm * 1.01 + 1e-5).all()
    assert L.clear_attn_check() == 0


def test_rope_rotation_flux2048_heads():
    wl = WORKLOADS["flux2048_r16"]
    q, k, _ = gpu_inputs(wl, seed=74)
    qr, kr = L.clear_attn_rope(q, k, wl.n_text, wl.H, wl.W, ntk=10.0)
    torch.cuda.synchronize()
    for h in (0, 23):
        ref = oracle.rope_2d(q[0:1, h:h + 1].cpu(), wl.n_text, wl.H, wl.W, ntk=10.0)
        _assert_rotated(qr[0:1, h:h + 1], ref, f"head {h}")


def test_rope_rotation_rejects_bad_inverse():
    import ctypes
    wl = Workload("rot_bad", 1, 1, 4, 8, 8, 128, 1)
    q, k, _ = gpu_inputs(wl, seed=75)
    p = L.make_params(1, 1, 4, 8, 8, 128, 1)
    rope = L.ClearRope(10000.0, 1.0)
    ws = torch.empty(L.rope_rotate_workspace_size(p), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    st = L.lib().clear_attn_rope(ctypes.byref(p), ctypes.byref(rope), 2, vp(q), vp(k), vp(out), vp(out), vp(ws),
                                 ctypes.c_size_t(ws.numel()), None)
    assert L.status_string(st) == "CLEAR_ERR_INVALID_ARG"


# The backward through the rotary embedding (clear_attn_bwd_rope): against the oracle's backward on
# the rotated q and k as bf16 (the operands the kernels multiply), with dQ and dK turned back by the
# oracle's inverse rotation in float64. The kernel rounds dQ and dK once more after turning them
# back, inside the standard bf16 bar.
BWD = [
    (Workload("rbwd_ragged", 1, 2, 77, 24, 40, 128, 5), 10000.0, 10.0, "circle"),
    (Workload("rbwd_d64_square", 1, 2, 30, 16, 20, 64, 4), 500.0, 2.0, "square"),
]


@pytest.mark.parametrize("wl,theta,ntk,window", BWD, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_rope_backward(wl, theta, ntk, window):
    q, k, v, dO = gpu_inputs(wl, seed=76, grad=True)
    o, lse = L.clear_attn_fwd_rope(q, k, v, wl.n_text, wl.H, wl.W, wl.r, theta=theta, ntk=ntk, window=window)
    dq, dk, dv = L.clear_attn_bwd_rope(q, k, v, o, lse, dO, wl.n_text, wl.H, wl.W, wl.r, theta=theta, ntk=ntk,
                                       window=window)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    qb = rotated_bf16(q.cpu(), wl.n_text, wl.H, wl.W, theta, ntk)
    kb = rotated_bf16(k.cpu(), wl.n_text, wl.H, wl.W, theta, ntk)
    rq, rk, rv = oracle.clear_attention_backward(qb, kb, v.cpu(), dO.cpu(), wl.n_text, wl.H, wl.W, wl.r, window=window)
    rq = oracle.rope_2d(rq, wl.n_text, wl.H, wl.W, theta, ntk, inverse=True)
    rk = oracle.rope_2d(rk, wl.n_text, wl.H, wl.W, theta, ntk, inverse=True)
    assert_close(dq.float().cpu().numpy(), rq, f"{wl.name} dQ")
    assert_close(dk.float().cpu().numpy(), rk, f"{wl.name} dK")
    assert_close(dv.float().cpu().numpy(), rv, f"{wl.name} dV")
