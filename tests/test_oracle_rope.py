"""Pins of the oracle's rotary embedding (rope_2d) and the RoPE forward: the 1D case against an
independent library implementation of interleaved rotary embedding (transformers' GPT-J routine),
norm preservation, the relative-position property on the grid, untouched text tokens, and the
NTK-aware base."""
import numpy as np
import pytest
import torch

import oracle
from clear_inputs import Workload, make_inputs


def _gptj_rotate(x, positions):
    """Interleaved rotary embedding of x [T, dim] at integer positions by the GPT-J routine (base
    10000): a library implementation independent of the oracle."""
    from transformers.models.gptj.modeling_gptj import apply_rotary_pos_emb, create_sinusoidal_positions
    dim = x.shape[-1]
    table = create_sinusoidal_positions(int(max(positions)) + 1, dim).double()  # [P, dim]: sin | cos
    sincos = table[torch.as_tensor(positions)]
    sin, cos = sincos[:, : dim // 2], sincos[:, dim // 2:]
    out = apply_rotary_pos_emb(torch.as_tensor(x)[None, :, None, :], sin[None], cos[None])
    return out[0, :, 0, :].numpy()


@pytest.mark.parametrize("axis", ["x", "y"])
def test_one_axis_matches_library_rope(axis):
    # A one-row grid (positions along x) or one-column grid (along y): that axis' half of the head
    # dims is plain 1D rotary embedding, the other half is rotated by position 0 (unchanged).
    d, n = 32, 23
    H, W = (1, n) if axis == "x" else (n, 1)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((n, d))
    got = oracle.rope_2d(x, 0, H, W)
    half = slice(d // 2, d) if axis == "x" else slice(0, d // 2)
    other = slice(0, d // 2) if axis == "x" else slice(d // 2, d)
    ref = _gptj_rotate(x[:, half], list(range(n)))
    assert np.abs(got[:, half] - ref).max() < 1e-5
    assert np.array_equal(got[:, other], x[:, other])


def test_rotation_preserves_every_pair_norm_and_text_rows():
    wl = Workload("rp", 1, 2, 5, 6, 7, 16, 3)
    q, _, _ = make_inputs(wl, seed=1, dtype=torch.float32)
    qr = oracle.rope_2d(q, 5, 6, 7, ntk=10.0)
    qd = q.double().numpy()
    n0 = qd[..., 0::2] ** 2 + qd[..., 1::2] ** 2
    n1 = qr[..., 0::2] ** 2 + qr[..., 1::2] ** 2
    assert np.abs(n0 - n1).max() < 1e-12
    assert np.array_equal(qr[:, :, :5], qd[:, :, :5])  # text tokens are not rotated
    assert np.abs(qr[:, :, 5:] - qd[:, :, 5:]).max() > 0.1


def test_scores_depend_only_on_the_grid_offset():
    # (R_a q) . (R_b k) depends on a - b only: shifting both tokens by the same grid offset leaves
    # the dot product unchanged, while a different offset changes it.
    d, H, W = 16, 9, 11
    rng = np.random.default_rng(2)
    qv, kv = rng.standard_normal(d), rng.standard_normal(d)
    x = np.zeros((H * W, d))

    def dot(pq, pk):
        a = x.copy(); b = x.copy()
        a[pq[0] * W + pq[1]] = qv
        b[pk[0] * W + pk[1]] = kv
        ra = oracle.rope_2d(a, 0, H, W, ntk=10.0)
        rb = oracle.rope_2d(b, 0, H, W, ntk=10.0)
        return float(ra[pq[0] * W + pq[1]] @ rb[pk[0] * W + pk[1]])

    base = dot((2, 3), (4, 1))
    assert abs(dot((5, 8), (7, 6)) - base) < 1e-12
    assert abs(dot((0, 2), (2, 0)) - base) < 1e-12
    assert abs(dot((2, 3), (4, 2)) - base) > 1e-3


def test_ntk_base():
    # The NTK-aware base theta * alpha^(d/(d-2)): alpha = 1 is plain RoPE; alpha > 1 slows every pair
    # but the first, whose rate base^0 = 1 is fixed; the slowest pair's rate is divided by about alpha.
    f1 = oracle.rope_inv_freq(64, 10000.0, 1.0)
    f10 = oracle.rope_inv_freq(64, 10000.0, 10.0)
    assert np.allclose(f1, 10000.0 ** (-np.arange(0, 64, 2) / 64.0))
    assert f10[0] == 1.0 and (f10[1:] < f1[1:]).all()
    assert abs(f1[-1] / f10[-1] - 10.0) < 1e-9


def test_rope_forward_is_the_plain_forward_of_rotated_inputs():
    wl = Workload("rf", 1, 2, 4, 5, 6, 16, 3)
    q, k, v = make_inputs(wl, seed=3, dtype=torch.float32)
    O, L = oracle.clear_attention_forward_rope(q, k, v, 4, 5, 6, 3, ntk=10.0)
    O2, L2 = oracle.clear_attention_forward(oracle.rope_2d(q, 4, 5, 6, ntk=10.0), oracle.rope_2d(k, 4, 5, 6, ntk=10.0),
                                            v, 4, 5, 6, 3)
    assert np.abs(O - O2).max() < 1e-12 and np.abs(L - L2).max() < 1e-12
    O3, _ = oracle.clear_attention_forward(q, k, v, 4, 5, 6, 3)
    assert np.abs(O - O3).max() > 1e-3


def test_inverse_rotation_is_the_transpose():
    # The inverse turns every pair back: it undoes the rotation both ways, and it is the transpose,
    # <R x, y> = <x, R^T y> over every token.
    wl = Workload("ri", 1, 2, 3, 5, 7, 16, 3)
    x, y, _ = make_inputs(wl, seed=4, dtype=torch.float32)
    xd, yd = x.double().numpy(), y.double().numpy()
    rx = oracle.rope_2d(x, 3, 5, 7, ntk=10.0)
    assert np.abs(oracle.rope_2d(rx, 3, 5, 7, ntk=10.0, inverse=True) - xd).max() < 1e-12
    assert np.abs(oracle.rope_2d(oracle.rope_2d(x, 3, 5, 7, ntk=10.0, inverse=True), 3, 5, 7, ntk=10.0) - xd).max() < 1e-12
    ry_t = oracle.rope_2d(y, 3, 5, 7, ntk=10.0, inverse=True)
    assert np.abs((rx * yd).sum(-1) - (xd * ry_t).sum(-1)).max() < 1e-12
    # and it is not the identity: an image token moves
    assert np.abs(ry_t[:, :, 3:] - yd[:, :, 3:]).max() > 0.1
