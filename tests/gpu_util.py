"""Helpers shared by the GPU parity tests: seeded inputs, sampled rows, tolerance checks."""
import math

import numpy as np
import torch

import oracle
from clear_inputs import Workload, make_inputs

# Tolerance for bf16 inputs with fp32 accumulation (same bar for O and for dQ, dK, dV).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def err_stats(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    e = np.abs(got - ref)
    return float(e.max()), float(e.mean()), float(e.max() / max(1e-30, np.abs(ref).max()))


def assert_close(got, ref, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    mx, mn, rel = err_stats(got, ref)
    assert np.isfinite(np.asarray(got, dtype=np.float64)).all(), f"{what}: non-finite output"
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max abs {mx:.3e}, mean abs {mn:.3e}, rel {rel:.3e}"
    return mx, mn


def gpu_inputs(wl: Workload, seed: int, grad=False):
    """Inputs drawn on the CPU (tiny/medium shapes) so the oracle sees the exact same bf16 values."""
    t = make_inputs(wl, seed=seed, dtype=torch.bfloat16, device="cpu", with_grad_out=grad)
    return tuple(x.cuda() for x in t)


def sample_rows(wl: Workload, rng: np.random.Generator, n_interior=48, n_border=24, n_text=8):
    """Query rows for sampled parity at full size: the 4 corners, border rows, random interior
    rows and text rows."""
    H, W, nt = wl.H, wl.W, wl.n_text
    rows = [nt + 0, nt + W - 1, nt + (H - 1) * W, nt + (H - 1) * W + W - 1]
    for _ in range(n_border):
        side = int(rng.integers(4))
        if side == 0:
            y, x = 0, int(rng.integers(W))
        elif side == 1:
            y, x = H - 1, int(rng.integers(W))
        elif side == 2:
            y, x = int(rng.integers(H)), 0
        else:
            y, x = int(rng.integers(H)), W - 1
        rows.append(nt + y * W + x)
    for _ in range(n_interior):
        rows.append(nt + int(rng.integers(H)) * W + int(rng.integers(W)))
    if nt:
        rows += sorted(rng.choice(nt, size=min(n_text, nt), replace=False).tolist())
    return sorted(set(rows))


def oracle_rows(q, k, v, wl: Workload, b: int, h: int, rows):
    """Oracle O and LSE for selected rows of one (b, h); only that head is copied to the host."""
    return oracle.clear_attention_rows(q, k, v, wl.n_text, wl.H, wl.W, wl.r, b, h, rows)
