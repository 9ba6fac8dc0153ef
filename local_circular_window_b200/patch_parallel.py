"""Patch-parallel CLEAR inference: heads split over ranks, or the image grid split into row stripes,
one per rank (GPU).

Head sharding needs no exchange at all: heads are independent problems, so each rank runs the
forward on its own heads (head_parallel_forward gathers the outputs if asked).

CLEAR's window has radius r, so an image query reaches r - 1 grid rows up and down: a rank that owns
rows [lo, hi) needs, besides the text tokens every rank holds, only r - 1 rows of keys from each
neighbour (pith.science review of the CLEAR paper, "If this is right": boundary communication of
size O(r x W) between adjacent patches). Text queries attend to every key; each rank computes them
over a share of the keys, and the shares are merged:

* mode "exact": the shares are disjoint (rank 0 takes the text keys and its rows, every other rank
  its own rows) and the text rows are merged with log-sum-exp weights, which is exactly the
  single-GPU result;
* mode "eq7": every rank takes the text keys and its own rows, and the text rows are averaged over
  ranks, the patch-wise approximation of Eq. 7 in the paper (pith review, "What carries the
  argument").

Communication is torch.distributed (NCCL between GPUs, gloo on CPU): a batched send/recv of the halo
rows with the two neighbours, and an all-gather of the text rows. All arithmetic runs in the CUDA
library (clear_attn_fwd_stripe, clear_attn_text_merge). ``local_forward`` and ``text_merge`` can be
replaced, which the CPU tests use to check the partitioning and the exchange with a reference.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as B


def head_bounds(heads: int, world: int):
    """Heads [lo, hi) of each rank: a balanced split of the heads over `world` ranks."""
    base, extra = divmod(heads, world)
    out, lo = [], 0
    for p in range(world):
        hi = lo + base + (1 if p < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def head_parallel_forward(q, k, v, n_text: int, H: int, W: int, r: int, group=None, window: str = "circle",
                          gather: bool = True, local_forward=None):
    """Forward of this rank's heads. q, k, v: [B, heads_r, T, d], the heads head_bounds assigns to this
    rank. Returns (o, lse) of those heads, or, with gather, of all heads on every rank (an all-gather
    of the outputs; the forward itself exchanges nothing)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    fwd = local_forward or (lambda q_, k_, v_: B.clear_attn_fwd(q_, k_, v_, n_text, H, W, r, window=window))
    o, lse = fwd(q, k, v)
    if not gather:
        return o, lse
    counts = [torch.zeros(1, dtype=torch.int64, device=o.device) for _ in range(world)]
    dist.all_gather(counts, torch.tensor([o.shape[1]], dtype=torch.int64, device=o.device), group)
    counts = [int(c.item()) for c in counts]
    m = max(counts)
    pad_o = o.new_zeros((o.shape[0], m) + tuple(o.shape[2:]))
    pad_l = lse.new_zeros((lse.shape[0], m) + tuple(lse.shape[2:]))
    pad_o[:, :o.shape[1]] = o
    pad_l[:, :lse.shape[1]] = lse
    os_ = [torch.empty_like(pad_o) for _ in range(world)]
    ls_ = [torch.empty_like(pad_l) for _ in range(world)]
    dist.all_gather(os_, pad_o, group)
    dist.all_gather(ls_, pad_l, group)
    return (torch.cat([t[:, :c] for t, c in zip(os_, counts)], dim=1),
            torch.cat([t[:, :c] for t, c in zip(ls_, counts)], dim=1))


def stripe_bounds(H: int, world: int):
    """Rows [lo, hi) of each rank: a balanced split of H rows into `world` contiguous stripes."""
    base, extra = divmod(H, world)
    bounds, lo = [], 0
    for p in range(world):
        hi = lo + base + (1 if p < extra else 0)
        bounds.append((lo, hi))
        lo = hi
    return bounds


@dataclass(frozen=True)
class StripePlan:
    """One rank's stripe: own rows [lo, hi), `top` halo rows above and `bot` below."""
    rank: int
    world: int
    n_text: int
    H: int
    W: int
    r: int
    lo: int
    hi: int
    top: int
    bot: int

    @property
    def own_rows(self) -> int:
        return self.hi - self.lo

    @property
    def stripe_rows(self) -> int:
        return self.top + self.own_rows + self.bot

    def stripe(self, mode: str) -> B.ClearStripe:
        """Query rows: the own rows. Text rows see the own rows, and the text keys in mode "eq7" or
        on rank 0 (the exact mode's disjoint shares)."""
        text_keys = mode == "eq7" or self.rank == 0
        return B.make_stripe(self.top, self.top + self.own_rows, self.top, self.top + self.own_rows, text_keys)


def make_plan(n_text: int, H: int, W: int, r: int, world: int, rank: int) -> StripePlan:
    """The stripe of `rank`. Halos come from the immediate neighbours only, so every stripe must be
    at least r - 1 rows tall (with many ranks and a large radius, a small grid cannot be split)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    bounds = stripe_bounds(H, world)
    halo = r - 1
    if world > 1 and min(hi - lo for lo, hi in bounds) < max(1, halo):
        raise ValueError(f"stripes of {H} rows over {world} ranks are thinner than the halo of {halo} rows (r = {r})")
    lo, hi = bounds[rank]
    top = min(halo, lo)
    bot = min(halo, H - hi)
    return StripePlan(rank, world, n_text, H, W, r, lo, hi, top, bot)


def exchange_halos(own, plan: StripePlan, group=None):
    """Sends this rank's first / last r - 1 rows to the rank above / below and receives its halos.

    own: [B, heads, own_rows * W, d] image tokens of this rank (k or v). Returns (top, bot) with
    [B, heads, plan.top * W, d] and [B, heads, plan.bot * W, d] (empty at the grid's edges)."""
    import torch.distributed as dist

    Bsz, heads, _, d = own.shape
    W = plan.W
    top = own.new_empty((Bsz, heads, plan.top * W, d))
    bot = own.new_empty((Bsz, heads, plan.bot * W, d))
    ops = []
    if plan.top:  # rank above: its bottom rows are my top halo, my top rows are its bottom halo
        ops.append(dist.P2POp(dist.irecv, top, plan.rank - 1, group))
        ops.append(dist.P2POp(dist.isend, own[:, :, :plan.top * W].contiguous(), plan.rank - 1, group))
    if plan.bot:
        ops.append(dist.P2POp(dist.irecv, bot, plan.rank + 1, group))
        ops.append(dist.P2POp(dist.isend, own[:, :, own.shape[2] - plan.bot * W:].contiguous(), plan.rank + 1, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    return top, bot


def _cuda_stripe_forward(q, k, v, n_text, H, W, r, stripe, window):
    return B.clear_attn_fwd_stripe(q, k, v, n_text, H, W, r, stripe, window=window)


def _cuda_text_merge(o_parts, lse_parts, mode):
    return B.clear_attn_text_merge(o_parts, lse_parts, mode)


def _stripe_tensors(text, top, own, bot, zero_halo: bool):
    if zero_halo:  # query tensor: halo rows are not computed, any values do
        top, bot = torch.zeros_like(top), torch.zeros_like(bot)
    return torch.cat([text, top, own, bot], dim=2).contiguous()


def _check_mode(mode):
    if mode not in ("exact", "eq7"):
        raise ValueError("mode must be 'exact' or 'eq7'")


def patch_parallel_forward(q_text, k_text, v_text, q_own, k_own, v_own, n_text: int, H: int, W: int, r: int,
                           mode: str = "exact", group=None, window: str = "circle", local_forward=None,
                           text_merge=None):
    """Forward of this rank's stripe, inside a torch.distributed group of `world` ranks.

    q_text, k_text, v_text: [B, heads, n_text, d], the same on every rank. q_own, k_own, v_own:
    [B, heads, own_rows * W, d], this rank's rows of the grid (stripe_bounds). Returns
    (o_text [B, heads, n_text, d], lse_text [B, heads, n_text], the same on every rank;
     o_own [B, heads, own_rows * W, d], lse_own [B, heads, own_rows * W]).
    """
    import torch.distributed as dist

    _check_mode(mode)
    if window not in ("circle", "square"):
        raise ValueError("patch-parallel inference offers the circle and square windows")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    plan = make_plan(n_text, H, W, r, world, rank)
    if q_own.shape[2] != plan.own_rows * W:
        raise ValueError(f"rank {rank} owns rows [{plan.lo}, {plan.hi}): expected {plan.own_rows * W} image tokens")
    k_top, k_bot = exchange_halos(k_own, plan, group)
    v_top, v_bot = exchange_halos(v_own, plan, group)
    q_top = q_own.new_empty((q_own.shape[0], q_own.shape[1], plan.top * W, q_own.shape[3]))
    q_bot = q_own.new_empty((q_own.shape[0], q_own.shape[1], plan.bot * W, q_own.shape[3]))
    qs = _stripe_tensors(q_text, q_top, q_own, q_bot, zero_halo=True)
    ks = _stripe_tensors(k_text, k_top, k_own, k_bot, zero_halo=False)
    vs = _stripe_tensors(v_text, v_top, v_own, v_bot, zero_halo=False)
    fwd = local_forward or _cuda_stripe_forward
    o_s, lse_s = fwd(qs, ks, vs, n_text, plan.stripe_rows, W, r, plan.stripe(mode), window)
    a, b = n_text + plan.top * W, n_text + (plan.top + plan.own_rows) * W
    o_own, lse_own = o_s[:, :, a:b], lse_s[:, :, a:b]
    if n_text == 0:
        return o_s[:, :, :0], lse_s[:, :, :0], o_own, lse_own
    o_tp, l_tp = o_s[:, :, :n_text].contiguous(), lse_s[:, :, :n_text].contiguous()
    o_parts = [torch.empty_like(o_tp) for _ in range(world)]
    l_parts = [torch.empty_like(l_tp) for _ in range(world)]
    dist.all_gather(o_parts, o_tp, group)
    dist.all_gather(l_parts, l_tp, group)
    merge = text_merge or _cuda_text_merge
    o_text, lse_text = merge(torch.stack(o_parts).contiguous(), torch.stack(l_parts).contiguous(), mode)
    return o_text, lse_text, o_own, lse_own


def forward_by_stripes(q, k, v, n_text: int, H: int, W: int, r: int, stripes: int, mode: str = "exact",
                       window: str = "circle"):
    """The same split run in one process, stripe after stripe (no communication): one GPU computes a
    grid stripe by stripe, e.g. to bound the memory of intermediate tensors, with the same results
    as `stripes` ranks. q, k, v: contiguous [B, heads, n_text + H*W, d] on the GPU. Returns (o, lse)
    of the whole problem."""
    _check_mode(mode)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    o_parts, l_parts = [], []
    for rank in range(stripes):
        plan = make_plan(n_text, H, W, r, stripes, rank)
        rows = slice(n_text + (plan.lo - plan.top) * W, n_text + (plan.hi + plan.bot) * W)
        qs, ks, vs = (torch.cat([t[:, :, :n_text], t[:, :, rows]], dim=2).contiguous() for t in (q, k, v))
        o_s, lse_s = B.clear_attn_fwd_stripe(qs, ks, vs, n_text, plan.stripe_rows, W, r, plan.stripe(mode),
                                             window=window)
        a, b = n_text + plan.top * W, n_text + (plan.top + plan.own_rows) * W
        o[:, :, n_text + plan.lo * W:n_text + plan.hi * W] = o_s[:, :, a:b]
        lse[:, :, n_text + plan.lo * W:n_text + plan.hi * W] = lse_s[:, :, a:b]
        if n_text:
            o_parts.append(o_s[:, :, :n_text])
            l_parts.append(lse_s[:, :, :n_text])
    if n_text:
        ot, lt = B.clear_attn_text_merge(torch.stack(o_parts).contiguous(), torch.stack(l_parts).contiguous(), mode)
        o[:, :, :n_text], lse[:, :, :n_text] = ot, lt
    return o, lse
