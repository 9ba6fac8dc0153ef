"""Mixed-resolution batches (clear_attn_fwd_varlen): items of their own (n_text, H, W) packed along
the token axis run in one forward launch. Each item's image rows must equal clear_attn_fwd on that
item alone bit for bit (the same tiles and arithmetic). Its text rows are split-KV partials merged
in a fixed order, and the batch may split them differently from the single call (a single call
chooses its split count for its own load balance, the batch by the plain rule), so they are held to
the single call within the bf16 bar. Small items are checked against the oracle as well."""
import numpy as np
import pytest
import torch

import local_circular_window_b200 as L
import oracle
from clear_inputs import make_random
from gpu_util import LSE_ABS, assert_close


def _same_item(o, lse, oi, li, n_text, what):
    """Image rows bit for bit; text rows within the bf16 bar (their split merge may differ)."""
    assert torch.equal(o[..., n_text:, :], oi[..., n_text:, :]), what
    assert torch.equal(lse[..., n_text:], li[..., n_text:]), what
    if n_text:
        assert_close(o[..., :n_text, :].float().cpu().numpy(), oi[..., :n_text, :].float().cpu().numpy(), f"{what} text")
        assert (lse[..., :n_text] - li[..., :n_text]).abs().max().item() <= LSE_ABS, what


def _packed(items, heads, d, seed):
    total, starts = L.varlen_tokens(items)
    q, k, v = (make_random((heads, total, d), seed=seed + i, device="cuda") for i in range(3))
    return q, k, v, starts


def _item(t, start, n_text, H, W):
    return t[:, start:start + n_text + H * W].unsqueeze(0).contiguous()


CASES = [
    # FLUX-shaped 64^2 and 128^2 grids with 512 text tokens, a 40 x 24 grid without text, a wide one
    ([(512, 64, 64), (512, 128, 128), (0, 40, 24), (16, 24, 40)], 4, 128, 8, "circle"),
    ([(77, 24, 40), (0, 19, 21), (130, 13, 50), (5, 64, 64)], 3, 64, 5, "circle"),
    ([(33, 40, 24), (0, 24, 40), (200, 16, 16)], 2, 128, 4, "square"),
    ([(10, 20, 20), (64, 12, 30)], 2, 128, 4, "shifted"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("items,heads,d,r,window", CASES, ids=lambda c: str(c) if not isinstance(c, list) else "x".join(f"{a}-{b}-{c_}" for a, b, c_ in c))
def test_mixed_batch_equals_items_alone(items, heads, d, r, window):
    q, k, v, starts = _packed(items, heads, d, seed=51)
    o, lse = L.clear_attn_fwd_varlen(q, k, v, items, r, window=window)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    for (n_text, H, W), s in zip(items, starts):
        T = n_text + H * W
        qi, ki, vi = (_item(t, s, n_text, H, W) for t in (q, k, v))
        oi, li = L.clear_attn_fwd(qi, ki, vi, n_text, H, W, r, window=window)
        torch.cuda.synchronize()
        _same_item(o[:, s:s + T], lse[:, s:s + T], oi[0], li[0], n_text, (n_text, H, W))
        if T <= 2000:
            O, Lse = oracle.clear_attention_forward(qi, ki, vi, n_text, H, W, r, window=window)
            assert_close(o[:, s:s + T].float().cpu().numpy(), O[0], f"item {(n_text, H, W)}")
            assert np.abs(lse[:, s:s + T].cpu().numpy() - Lse[0]).max() <= LSE_ABS


@pytest.mark.gpu
def test_single_item_batch_is_the_plain_call():
    items = [(300, 33, 47)]
    q, k, v, starts = _packed(items, 3, 128, seed=52)
    o, lse = L.clear_attn_fwd_varlen(q, k, v, items, 6)
    oi, li = L.clear_attn_fwd(q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0), 300, 33, 47, 6)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    _same_item(o, lse, oi[0], li[0], 300, "single item")


@pytest.mark.gpu
def test_many_small_items():
    # 40 items of assorted small shapes (some without text): every item against its own call.
    rng = np.random.default_rng(7)
    items = [(int(rng.choice([0, 3, 130])), int(rng.integers(1, 30)), int(rng.integers(1, 40))) for _ in range(40)]
    q, k, v, starts = _packed(items, 2, 64, seed=53)
    o, lse = L.clear_attn_fwd_varlen(q, k, v, items, 3)
    torch.cuda.synchronize()
    assert L.clear_attn_check() == 0
    for (n_text, H, W), s in zip(items, starts):
        T = n_text + H * W
        oi, li = L.clear_attn_fwd(*(_item(t, s, n_text, H, W) for t in (q, k, v)), n_text, H, W, 3)
        torch.cuda.synchronize()
        _same_item(o[:, s:s + T], lse[:, s:s + T], oi[0], li[0], n_text, (n_text, H, W))
