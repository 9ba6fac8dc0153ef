"""GPU parity of the forward (clear_attn_fwd through the C ABI) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from clear_inputs import WORKLOADS, Workload, make_inputs
from gpu_util import LSE_ABS, assert_close, gpu_inputs, oracle_rows, sample_rows

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import local_circular_window_b200 as L


def _run(wl, q, k, v):
    o, lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    assert L.clear_attn_check() == 0
    return o, lse


# Small shapes: several query tiles, ragged text count and ragged grid edges, both head dims.
SMALL = [
    Workload("tiny", 1, 2, 16, 16, 16, 64, 4),
    Workload("ragged_d128", 2, 3, 77, 24, 40, 128, 5),
    Workload("no_text", 1, 2, 0, 19, 21, 128, 3),
    Workload("wide_text_d64", 1, 2, 200, 13, 50, 64, 7),
    Workload("r1", 1, 2, 5, 9, 17, 128, 1),
    Workload("full_radius", 1, 2, 16, 16, 16, 64, 22),
    Workload("text300_r16", 1, 2, 300, 32, 32, 128, 16),
    Workload("tall", 1, 1, 9, 70, 18, 128, 12),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_forward_small_full_oracle(wl):
    q, k, v = gpu_inputs(wl, seed=0)
    o, lse = _run(wl, q, k, v)
    O, LSE = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    assert_close(o.float().cpu().numpy(), O, f"{wl.name} O")
    assert_close(lse.cpu().numpy(), LSE, f"{wl.name} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS / 10)


def test_tiny_config_fp32_inputs_rounded_to_bf16():
    # The tiny workload is specified with float32 inputs; the kernel takes bf16, so the same rounded
    # values feed the oracle. The fp32-input oracle is reported for information.
    wl = WORKLOADS["tiny"]
    q32, k32, v32 = make_inputs(wl, seed=0, dtype=torch.float32)
    q, k, v = (t.to(torch.bfloat16).cuda() for t in (q32, k32, v32))
    o, lse = _run(wl, q, k, v)
    O, LSE = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    assert_close(o.float().cpu().numpy(), O, "tiny O")
    O32, _ = oracle.clear_attention_forward(q32, k32, v32, wl.n_text, wl.H, wl.W, wl.r)
    assert np.abs(o.float().cpu().numpy() - O32).max() < 0.1


def test_text_splits_exercised():
    # T > 64 chunks of 128 keys forces at least two splits of each text query tile.
    wl = Workload("split2", 1, 2, 130, 96, 96, 128, 6)
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    assert L.forward_shape(p)[2] >= 2
    q, k, v = gpu_inputs(wl, seed=3)
    o, lse = _run(wl, q, k, v)
    rows = sample_rows(wl, np.random.default_rng(0), n_text=130)
    for h in range(wl.heads):
        Or, Lr = oracle_rows(q, k, v, wl, 0, h, rows)
        assert_close(o[0, h, rows].float().cpu().numpy(), Or, f"split2 h{h} O")
        assert_close(lse[0, h, rows].cpu().numpy(), Lr, f"split2 h{h} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS)


@pytest.mark.parametrize("name", ["flux1024_r8", "flux1024_r16", "flux1024_r32"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_flux1024_heads_full_oracle(name, seed):
    wl = WORKLOADS[name]
    q, k, v = gpu_inputs(wl, seed=seed)
    o, lse = _run(wl, q, k, v)
    assert torch.isfinite(o.float()).all()
    for h in (0, 11, 23):
        O, LSE = oracle.clear_attention_forward(q[:, h:h + 1].cpu(), k[:, h:h + 1].cpu(), v[:, h:h + 1].cpu(),
                                                wl.n_text, wl.H, wl.W, wl.r)
        assert_close(o[:, h:h + 1].float().cpu().numpy(), O, f"{name} s{seed} h{h} O")
        assert_close(lse[:, h:h + 1].cpu().numpy(), LSE, f"{name} h{h} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS / 10)


@pytest.mark.parametrize("name", ["flux2048_r16", "8k_r8", "8k_r32"])
def test_large_configs_sampled_rows(name):
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl, seed=0, device="cuda")
    o, lse = _run(wl, q, k, v)
    rng = np.random.default_rng(0)
    rows = sample_rows(wl, rng, n_interior=64, n_border=32, n_text=16)
    for h in (0, 11, 23):
        Or, Lr = oracle_rows(q, k, v, wl, 0, h, rows)
        assert_close(o[0, h, rows].float().cpu().numpy(), Or, f"{name} h{h} O")
        assert_close(lse[0, h, rows].cpu().numpy(), Lr, f"{name} h{h} LSE", max_abs=LSE_ABS, mean_abs=LSE_ABS)
    del q, k, v, o, lse
    torch.cuda.empty_cache()


def test_repeated_calls_are_deterministic():
    wl = SMALL[1]
    q, k, v = gpu_inputs(wl, seed=5)
    o1, l1 = _run(wl, q, k, v)
    o2, l2 = _run(wl, q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_nonzero_stream_and_outputs_in_place():
    wl = SMALL[0]
    q, k, v = gpu_inputs(wl, seed=1)
    s = torch.cuda.Stream()
    o = torch.full_like(q, float("nan"))
    lse = torch.full((wl.B, wl.heads, wl.T), float("nan"), device="cuda")
    with torch.cuda.stream(s):
        L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o, lse=lse, stream=s)
    assert L.clear_attn_check(s) == 0
    O, _ = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    assert_close(o.float().cpu().numpy(), O, "stream O")


@pytest.mark.parametrize("d", [128, 64])
def test_outputs_only_16_byte_aligned(d):
    # The ABI promises 16-byte alignment only; the epilogue's 32-byte stores are used only when o
    # (and the workspace holding the text partials) are 32-byte aligned. Offsetting both by 16 bytes
    # takes the narrow-store path, which must give the same bits.
    wl = Workload("ragged_d", 1, 3, 77, 24, 40, d, 5)
    q, k, v = gpu_inputs(wl, seed=9)
    p = L.make_params(wl.B, wl.heads, wl.n_text, wl.H, wl.W, wl.d, wl.r)
    wsz = L.fwd_workspace_size(p)
    ref_o, ref_lse = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r)
    o_buf = torch.full((q.numel() + 8,), float("nan"), dtype=torch.bfloat16, device="cuda")
    o = o_buf[8:].view(q.shape)
    ws = torch.empty(wsz + 16, dtype=torch.uint8, device="cuda")[16:]
    assert o.data_ptr() % 32 == 16 and ws.data_ptr() % 32 == 16
    o2, lse2 = L.clear_attn_fwd(q, k, v, wl.n_text, wl.H, wl.W, wl.r, o=o, workspace=ws)
    assert L.clear_attn_check() == 0
    assert torch.equal(o2, ref_o) and torch.equal(lse2, ref_lse)


@pytest.mark.parametrize("boost", [3.0, 8.0])
def test_forward_scores_far_above_the_first_tiles(boost):
    # A row's exponent base is its running max; a later tile whose scores lie far above it must
    # raise the base and rescale the stored sum and O without losing exactness. Keys in the bottom
    # image rows are scaled up and aligned with every query, so for many rows the last tiles carry
    # scores about 30 (boost 3) or 90 (boost 8) log2 units above the text and upper-window keys
    # visited first. (Much larger scores, in the thousands, also perturb the tensor core's fp32
    # accumulation of S at the bf16 tolerance's scale; that is not what this checks.)
    wl = Workload("late_peak", 1, 2, 40, 24, 32, 128, 6)
    q, k, v = (t.float() for t in make_inputs(wl, seed=21, dtype=torch.float32))
    q = q.abs() * 0.5 + 0.2
    img0 = wl.n_text + 16 * wl.W
    k[:, :, img0:] = k[:, :, img0:].abs() * boost
    q, k, v = (t.to(torch.bfloat16).cuda() for t in (q, k, v))
    o, lse = _run(wl, q, k, v)
    O, LSE = oracle.clear_attention_forward(q.cpu(), k.cpu(), v.cpu(), wl.n_text, wl.H, wl.W, wl.r)
    assert_close(o.float().cpu().numpy(), O, f"boost {boost} O")
    rel = np.abs(lse.cpu().numpy() - LSE) / np.maximum(1.0, np.abs(LSE))
    assert rel.max() <= LSE_ABS, f"boost {boost} LSE rel {rel.max():.3e}"
