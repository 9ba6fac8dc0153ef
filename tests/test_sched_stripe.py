"""The forward's tile scheduler in stripe mode (patch-parallel inference): image pairs cover exactly
the kept pairs of the stripe's own query rows, and text pairs visit exactly the key set the stripe
names (each token once across the splits). Truth: the oracle's explicit mask of the stripe grid."""
import numpy as np
import pytest

import local_circular_window_b200 as L
import oracle

KQH, KQW, KKH, KKW, TILE, KCHUNK = 8, 16, 4, 16, 128, 64


def _keys_of_tile(tile, n_text, H, W):
    kind, a, b, flags = tile
    if kind == 0:
        return list(range(a, a + b))
    return [n_text + y * W + x for y in range(a, a + KKH) for x in range(b, b + KKW) if 0 <= y < H and 0 <= x < W]


def _queries_of_half(q_info, half, n_text, W, q_row1):
    is_text, bh, q0, x0, valid_b = q_info
    if half == 1 and not valid_b:
        return []
    if is_text:
        return [t for t in range(q0 + half * TILE, q0 + (half + 1) * TILE) if t < n_text]
    y0 = q0 + half * KQH
    return [n_text + y * W + x for y in range(y0, y0 + KQH) for x in range(x0, x0 + KQW) if y < q_row1 and x < W]


# (n_text, H, W, r, q_row0, q_row1, key_row0, key_row1, text_keys)
CASES = [(16, 20, 18, 4, 3, 17, 3, 17, True), (16, 20, 18, 4, 3, 17, 3, 17, False), (5, 9, 40, 3, 0, 7, 0, 7, True),
         (0, 12, 12, 5, 4, 12, 4, 12, False), (70, 26, 30, 6, 5, 21, 5, 21, False), (70, 26, 30, 6, 0, 26, 0, 26, True),
         (9, 10, 33, 2, 1, 9, 0, 0, True)]


@pytest.mark.parametrize("window", ["circle", "square"])
@pytest.mark.parametrize("case", CASES)
def test_stripe_tiles_cover_mask_exactly(case, window):
    n_text, H, W, r, qa, qb, ka, kb, tk = case
    p = L.make_params(1, 1, n_text, H, W, 64, r, window)
    s = L.make_stripe(qa, qb, ka, kb, tk)
    T = n_text + H * W
    n_txt, n_img, S, cps = L.forward_shape(p, s)
    M = oracle.clear_mask(n_text, H, W, r, window=window)
    want_text = set(range(n_text)) if tk else set()
    want_text |= set(range(n_text + ka * W, n_text + kb * W))
    text_cover = {}
    covered_queries = set()
    for item in range(n_txt + n_img):
        q_info, tiles = L.item_tiles(p, item, s)
        keys = [key for t in tiles for key in _keys_of_tile(t, n_text, H, W)]
        assert len(keys) == len(set(keys)), "a key is visited twice by one pair"
        if q_info[0]:
            text_cover.setdefault(q_info[2], []).extend(keys)
            continue
        for half in (0, 1):
            queries = _queries_of_half(q_info, half, n_text, W, qb)
            covered_queries |= set(queries)
            if not queries:
                continue
            need = set(np.nonzero(M[queries].any(axis=0))[0].tolist())
            got = set(k for t in tiles if t[3] & (1 << half) for k in _keys_of_tile(t, n_text, H, W))
            assert need <= got, "a kept pair of this half is not covered"
    assert covered_queries == set(range(n_text + qa * W, n_text + qb * W))
    for q0, keys in text_cover.items():
        assert sorted(keys) == sorted(want_text), "text rows must visit exactly the stripe's key set"
    assert len(text_cover) == (n_text + 2 * TILE - 1) // (2 * TILE)


def test_stripe_argument_errors():
    p = L.make_params(1, 1, 8, 10, 10, 64, 3)
    for bad in [(0, 0, 0, 10, True), (3, 2, 0, 10, True), (0, 11, 0, 10, True), (0, 10, 5, 4, True),
                (0, 10, 0, 11, True), (0, 10, 4, 4, False)]:
        with pytest.raises(L.ClearError) as e:
            L.forward_shape(p, L.make_stripe(*bad))
        assert e.value.status == 1, bad
    ps = L.make_params(1, 1, 8, 10, 10, 64, 3, "shifted")
    with pytest.raises(L.ClearError) as e:
        L.forward_shape(ps, L.make_stripe(0, 10, 0, 10, True))
    assert e.value.status == 2
