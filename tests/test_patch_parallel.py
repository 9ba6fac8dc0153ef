"""Patch-parallel inference on CPU: gloo ranks split the grid into row stripes, exchange r - 1 halo
rows with their neighbours and merge the text rows. The stripe forward and the text merge are
injected (oracle stripe rows, float64 merge), so these tests check the partitioning, the halo
exchange and the merge rule against the oracle's single-process results:
* "exact": every image row and every text row equals the full-problem oracle forward;
* "eq7": image rows as above, text rows equal the oracle's patch-wise average (Eq. 7)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from clear_inputs import Workload, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_stripe_forward(record):
    def fwd(q, k, v, n_text, H, W, r, stripe, window):
        record["stripe_k"] = k.clone()
        Ot, Lt, Oi, Li = oracle.clear_attention_stripe(q, k, v, n_text, H, W, r, stripe.q_row0, stripe.q_row1,
                                                       stripe.key_row0, stripe.key_row1, bool(stripe.text_keys),
                                                       window=window)
        o = torch.full(q.shape, float("nan"), dtype=torch.float64)
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float64)
        a, b = n_text + stripe.q_row0 * W, n_text + stripe.q_row1 * W
        o[:, :, :n_text], lse[:, :, :n_text] = torch.from_numpy(Ot), torch.from_numpy(Lt)
        o[:, :, a:b], lse[:, :, a:b] = torch.from_numpy(Oi), torch.from_numpy(Li)
        return o, lse
    return fwd


def _f64_merge(o_parts, lse_parts, mode):
    m = lse_parts.max(dim=0).values
    w = torch.exp(lse_parts - m)
    lse = m + torch.log(w.sum(dim=0))
    if mode == "exact":
        o = (w[..., None] * o_parts).sum(dim=0) / w.sum(dim=0)[..., None]
    else:
        o = o_parts.mean(dim=0)
    return o, lse


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from local_circular_window_b200 import patch_parallel as pp
        n_text, H, W, r, mode, window = case
        wl = Workload("pp", 2, 2, n_text, H, W, 16, r)
        q, k, v = (t.double() for t in make_inputs(wl, seed=11, dtype=torch.float32))
        plan = pp.make_plan(n_text, H, W, r, world, rank)
        own = slice(n_text + plan.lo * W, n_text + plan.hi * W)
        record = {}
        got = pp.patch_parallel_forward(q[:, :, :n_text], k[:, :, :n_text], v[:, :, :n_text],
                                        q[:, :, own], k[:, :, own], v[:, :, own], n_text, H, W, r, mode=mode,
                                        window=window, local_forward=_oracle_stripe_forward(record),
                                        text_merge=_f64_merge)
        halo = slice(n_text + (plan.lo - plan.top) * W, n_text + (plan.hi + plan.bot) * W)
        halo_ok = torch.equal(record["stripe_k"][:, :, n_text:], k[:, :, halo])
        out[rank] = (plan.lo, plan.hi, plan.top, plan.bot, halo_ok) + tuple(t.numpy() for t in got)
    finally:
        dist.destroy_process_group()


CASES = [
    (5, 9, 6, 3, "exact", "circle", 2),
    (5, 9, 6, 3, "eq7", "circle", 2),
    (3, 10, 5, 3, "exact", "square", 3),
    (4, 11, 4, 2, "eq7", "circle", 3),
    (0, 8, 5, 3, "exact", "circle", 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_gloo_ranks_match_the_oracle(case):
    *problem, world = case
    n_text, H, W, r, mode, window = problem
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), tuple(problem), out), nprocs=world, join=True)
    wl = Workload("pp", 2, 2, n_text, H, W, 16, r)
    q, k, v = make_inputs(wl, seed=11, dtype=torch.float32)
    O, L = oracle.clear_attention_forward(q, k, v, n_text, H, W, r, window=window)
    rows = []
    for rank in range(world):
        lo, hi, top, bot, halo_ok, o_text, l_text, o_own, l_own = out[rank]
        assert halo_ok, f"rank {rank}: halo rows differ from the neighbours' rows"
        assert top == min(r - 1, lo) and bot == min(r - 1, H - hi)
        rows.append((lo, hi))
        a, b = n_text + lo * W, n_text + hi * W
        assert np.abs(o_own - O[:, :, a:b]).max() < 1e-12 and np.abs(l_own - L[:, :, a:b]).max() < 1e-12
        if n_text == 0:
            continue
        if mode == "exact":
            assert np.abs(o_text - O[:, :, :n_text]).max() < 1e-12
            assert np.abs(l_text - L[:, :, :n_text]).max() < 1e-12
        else:
            edges = [lo_ for lo_, _ in _bounds(H, world)] + [H]
            ref = oracle.clear_text_rows_patch_average(q, k, v, n_text, H, W, edges)
            assert np.abs(o_text - ref).max() < 1e-12
            assert np.abs(o_text - O[:, :, :n_text]).max() > 1e-4  # the approximation is not the exact rows
    assert rows == _bounds(H, world) and rows[0][0] == 0 and rows[-1][1] == H


def _bounds(H, world):
    base, extra = divmod(H, world)
    out, lo = [], 0
    for p in range(world):
        hi = lo + base + (p < extra)
        out.append((lo, hi))
        lo = hi
    return out


def test_plan_rejects_stripes_thinner_than_the_halo():
    from local_circular_window_b200 import patch_parallel as pp
    with pytest.raises(ValueError):
        pp.make_plan(4, 8, 8, 5, 4, 0)  # 2-row stripes, 4-row halo
    plan = pp.make_plan(4, 8, 8, 3, 4, 1)
    assert (plan.lo, plan.hi, plan.top, plan.bot) == (2, 4, 2, 2)
    with pytest.raises(ValueError):
        pp.make_plan(4, 8, 8, 3, 4, 4)


def test_stripe_bounds_balanced_and_contiguous():
    from local_circular_window_b200 import patch_parallel as pp
    for H in (1, 7, 64, 129):
        for world in (1, 2, 3, 8):
            if world > H:
                continue
            b = pp.stripe_bounds(H, world)
            assert b == _bounds(H, world)
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1 and sum(sizes) == H


def _head_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from local_circular_window_b200 import patch_parallel as pp
        n_text, H, W, r, heads = 4, 7, 6, 3, 5
        wl = Workload("hp", 1, heads, n_text, H, W, 16, r)
        q, k, v = (t.double() for t in make_inputs(wl, seed=12, dtype=torch.float32))
        lo, hi = pp.head_bounds(heads, world)[rank]

        def fwd(q_, k_, v_):
            O, Lse = oracle.clear_attention_forward(q_, k_, v_, n_text, H, W, r)
            return torch.from_numpy(O), torch.from_numpy(Lse)

        o, lse = pp.head_parallel_forward(q[:, lo:hi], k[:, lo:hi], v[:, lo:hi], n_text, H, W, r, local_forward=fwd)
        out[rank] = (o.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_ranks_gather_the_full_result(world):
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_head_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    wl = Workload("hp", 1, 5, 4, 7, 6, 16, 3)
    q, k, v = make_inputs(wl, seed=12, dtype=torch.float32)
    O, Lse = oracle.clear_attention_forward(q, k, v, 4, 7, 6, 3)
    for rank in range(world):
        o, lse = out[rank]
        assert o.shape == O.shape and np.abs(o - O).max() < 1e-12 and np.abs(lse - Lse).max() < 1e-12
