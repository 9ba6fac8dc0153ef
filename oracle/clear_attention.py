"""Plain, slow CPU float64 oracle for CLEAR attention. TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the bench's CPU-baseline / reference legs may import this
module. The product path (the CUDA library and its Python binding) never calls it, and this module
imports nothing from the product package.

What it computes (sources are the pages about arXiv 2412.16112, "CLEAR: Conv-Like Linearization
Revs Pre-Trained Diffusion Transformers Up"):

* "pith review" = the pith.science machine review of the paper;
* "atlas summary" = the atlas.scime.ai AI summary of the paper.

1. Mask  [pith review, "Core claim"]: with text tokens first, M_ij = 1 iff i is a text token, or
   j is a text token, or the Euclidean grid distance of image tokens i and j is below r:
   dx^2 + dy^2 < r^2.  The review writes the condition 1-based (i <= n_text); here indices are
   0-based, so "text" means index < n_text.
2. One softmax over the union of text keys and window keys  [atlas summary, "Approach";
   pith review, "What carries the argument" (formulation consistency with softmax attention,
   Eq. 1 in "Assumptions")].
3. Scale 1/sqrt(c), c = head dim  [pith review, "What carries the argument", the Eq. 7 text].
4. Backward (dQ, dK, dV): the pages print none; they say only the attention layers are fine-tuned
   by gradient descent [pith review, "The reading"], so the gradient is the analytic gradient of
   the forward above (standard softmax-attention calculus, written out in `clear_attention_backward`).

5. Square-window variant (a comparison mask, not CLEAR's): the pages set the circular window
   against the usual square local window [nav.superapi.store page, "Technical Principles of
   CLEAR"] and give the circle's cost as about pi/4 of a square window's [pith review, "What
   carries the argument"]. Read as the same rule with the Chebyshev distance: image tokens i and j
   are kept iff |dx| < r and |dy| < r (the square circumscribing the disc, same strictness).
   Every function below takes window="circle" (CLEAR, the default) or window="square".
6. Border-shifted square window (the other comparison mask): the pages name Neighborhood
   Attention as the prior art CLEAR builds on [codewithpapers page, "Builds on"; pith review,
   desk verdict, which reads CLEAR as neighborhood attention with a disc-shaped window].
   Neighborhood attention keeps a fixed square of (2r-1) x (2r-1) keys per query and, at the
   grid border, shifts the window inward instead of clipping it, so every query sees the same
   number of keys. Read here as:
   image pair (i, j) kept iff |y_j - cy(y_i)| < r and |x_j - cx(x_i)| < r with the centre clamped,
   cy(y) = min(max(y, r-1), H-r) (likewise cx); it needs H, W >= 2r-1. window="shifted".

7. Patch-parallel inference [pith review, "If this is right" (adjacent patches exchange only
   O(r x W) boundary tokens) and "What carries the argument" (Eq. 7)]: `clear_attention_stripe`
   gives one stripe's rows (image rows of its own grid rows, text rows over the keys it is given),
   and `clear_text_rows_patch_average` the patch-wise average of Eq. 7 for the text rows.

8. FP8 score products (not on the pages; a variant for inference): q and k arrive as 8-bit
   floating-point codes in the OCP FP8 E4M3 format with a dequantization scale per (batch, head),
   v stays bf16. `e4m3_decode` writes the format out (sign bit, 4 exponent bits with bias 7,
   3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; the all-ones exponent and mantissa
   is NaN, the format has no infinities) and `clear_attention_forward_fp8` runs the plain forward
   above on q = decode(q8) * s_q and k = decode(k8) * s_k: the scores are those of the dequantized
   inputs, the rest is unchanged.

9. Rotary position embedding applied to q and k before the scores (an optional first step): the
   review lists an NTK-aware RoPE scale factor of 10 among the free parameters ["Assumptions &
   free parameters"] and the paper cites RoFormer (rotary embedding: each pair of adjacent head
   dims (2i, 2i+1) rotated by position * base^(-2i/d)) and NTK-aware scaled RoPE (the base raised
   to theta * alpha^(d/(d-2)) for a scale factor alpha). Read for the token grid as axial 2D RoPE:
   the first half of the head dims rotated by the grid row y, the second half by the column x,
   each half with its own d/2 dims in the formulas above; text tokens are not rotated.
   `rope_2d`, `clear_attention_forward_rope`.

Readings where the pages leave a step open (each listed with its reason in the design notes):
strict "<" in the radius test; image tokens in row-major order t = n_text + y*W + x; windows are
clipped at the grid border (border queries see fewer keys); text queries attend to every token
exactly (no patch-wise approximation); LSE is the natural-log log-sum-exp of the scaled, masked
scores; r is an integer >= 1.

Everything here is float64 and builds the explicit mask, with no blocking or fusion.
"""
from __future__ import annotations

import math

import numpy as np


# ----------------------------------------------------------------------------------------------
# Geometry and mask
# ----------------------------------------------------------------------------------------------

def token_coords(n_text: int, H: int, W: int):
    """Grid coordinates (y, x) of every token; text tokens get (-1, -1) and is_text=True.

    Image token (y, x) sits at index n_text + y*W + x (row-major reading of the grid order).
    """
    T = n_text + H * W
    y = np.full(T, -1, dtype=np.int64)
    x = np.full(T, -1, dtype=np.int64)
    img = np.arange(H * W, dtype=np.int64)
    y[n_text:] = img // W
    x[n_text:] = img % W
    is_text = np.zeros(T, dtype=bool)
    is_text[:n_text] = True
    return y, x, is_text


WINDOWS = ("circle", "square", "shifted")


def clear_mask(n_text: int, H: int, W: int, r: int, rows=None, window: str = "circle") -> np.ndarray:
    """Boolean CLEAR mask M [len(rows), T] (all T rows if rows is None).

    [pith review, "Core claim"]: M_ij = 1 if i <= n_text or j <= n_text or
    (d^x_ij)^2 + (d^y_ij)^2 < r^2 (1-based there; 0-based "< n_text" here). With window="square"
    the last test is |dx| < r and |dy| < r.
    """
    assert window in WINDOWS
    y, x, is_text = token_coords(n_text, H, W)
    T = y.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    dy = y[rows][:, None] - y[None, :]
    dx = x[rows][:, None] - x[None, :]
    if window == "circle":
        near = dx * dx + dy * dy < r * r
    elif window == "square":
        near = (np.abs(dx) < r) & (np.abs(dy) < r)
    else:  # border-shifted square: distances from the clamped window centre of the query
        assert H >= 2 * r - 1 and W >= 2 * r - 1, "the shifted window needs H, W >= 2r - 1"
        cy = np.clip(y[rows], r - 1, H - r)[:, None]
        cx = np.clip(x[rows], r - 1, W - r)[:, None]
        near = (np.abs(y[None, :] - cy) < r) & (np.abs(x[None, :] - cx) < r)
    return is_text[rows][:, None] | is_text[None, :] | near


# ----------------------------------------------------------------------------------------------
# Forward / backward (explicit mask, float64)
# ----------------------------------------------------------------------------------------------

def _as_f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor: exact upcast (bf16 and fp32 are exact in fp64)
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def _masked_softmax_rows(S: np.ndarray, M: np.ndarray):
    """Row softmax of S restricted to M; returns (P, LSE). Masked entries get probability 0."""
    S = np.where(M, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=1, keepdims=True)
    P = E / l
    lse = (m + np.log(l))[:, 0]
    return P, lse


def clear_attention_forward(q, k, v, n_text: int, H: int, W: int, r: int, scale=None, window: str = "circle"):
    """O = softmax_M(Q K^T * scale) V and LSE for every (batch, head).

    q, k, v: [B, heads, T, d] (numpy or torch; upcast exactly to float64).
    Returns O [B, heads, T, d] float64 and LSE [B, heads, T] float64 (natural log).
    Scale defaults to 1/sqrt(d) [pith review, "What carries the argument", Eq. 7 text].
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hh, T, d = q.shape
    assert T == n_text + H * W, "T must equal n_text + H*W"
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    M = clear_mask(n_text, H, W, r, window=window)
    O = np.empty_like(q)
    LSE = np.empty((B, Hh, T))
    for b in range(B):
        for h in range(Hh):
            S = (q[b, h] @ k[b, h].T) * scale
            P, lse = _masked_softmax_rows(S, M)
            O[b, h] = P @ v[b, h]
            LSE[b, h] = lse
    return O, LSE


def clear_attention_rows(q, k, v, n_text: int, H: int, W: int, r: int, b: int, h: int, rows,
                         scale=None, window: str = "circle"):
    """Forward outputs for selected query rows of one (b, h) only; mask rows built explicitly.

    Used where the full T x T mask does not fit (e.g. a 512 x 512 grid, T = 262,656).
    Returns O_rows [len(rows), d] and LSE_rows [len(rows)] in float64.
    """
    qb = _as_f64(q[b, h][rows] if hasattr(q, "detach") else np.asarray(q)[b, h][rows])
    kb, vb = _as_f64(k[b, h]), _as_f64(v[b, h])
    d = qb.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    M = clear_mask(n_text, H, W, r, rows=rows, window=window)
    S = (qb @ kb.T) * scale
    P, lse = _masked_softmax_rows(S, M)
    return P @ vb, lse


def clear_attention_backward(q, k, v, dO, n_text: int, H: int, W: int, r: int, scale=None,
                             window: str = "circle"):
    """Analytic gradient of the forward above with respect to q, k and v, given dO.

    With S = scale * Q K^T, P = softmax_M(S) row-wise and O = P V:
        dV = P^T dO
        dP = dO V^T
        D_i = sum_j P_ij dP_ij  (= rowsum(dO o O))
        dS = P o (dP - D)
        dQ = scale * dS K
        dK = scale * dS^T Q
    Masked entries have P = 0, so they carry no gradient.
    """
    q, k, v, dO = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dO)
    B, Hh, T, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    M = clear_mask(n_text, H, W, r, window=window)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    for b in range(B):
        for h in range(Hh):
            S = (q[b, h] @ k[b, h].T) * scale
            P, _ = _masked_softmax_rows(S, M)
            O = P @ v[b, h]
            dv[b, h] = P.T @ dO[b, h]
            dP = dO[b, h] @ v[b, h].T
            D = (dO[b, h] * O).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, h] = scale * (dS @ k[b, h])
            dk[b, h] = scale * (dS.T @ q[b, h])
    return dq, dk, dv


# ----------------------------------------------------------------------------------------------
# Counting: window size, kept pairs, useful FLOPs
# ----------------------------------------------------------------------------------------------

def window_half_width(r: int, ady: int, window: str = "circle") -> int:
    """Largest dx >= 0 kept at vertical distance ady >= 0 (from the window centre), or -1 if none."""
    if window in ("square", "shifted"):
        return r - 1 if ady < r else -1
    rem = r * r - ady * ady
    return math.isqrt(rem - 1) if rem > 0 else -1  # largest dx with dx^2 < rem


def window_lattice_count(r: int, window: str = "circle") -> int:  # noqa: C901
    """Keys in an interior query's window: #{(dx, dy) in Z^2 : dx^2 + dy^2 < r^2}.

    [pith review, "What carries the argument"]: the window's key count is constant in the
    resolution and is about pi/4 of the square window's. window="square" counts |dx|, |dy| < r.
    """
    if window in ("square", "shifted"):
        return (2 * r - 1) ** 2
    n = 0
    for dy in range(-r, r + 1):
        rem = r * r - dy * dy
        if rem <= 0:
            continue
        w = math.isqrt(rem - 1)  # largest dx with dx^2 < rem
        n += 2 * w + 1
    return n


def window_pairs(H: int, W: int, r: int, window: str = "circle") -> int:
    """Kept image-image pairs P(r) with border clipping: sum over offsets of the overlap area.
    The shifted window keeps exactly (2r-1)^2 image keys for every image query."""
    if window == "shifted":
        return H * W * (2 * r - 1) ** 2
    total = 0
    for dy in range(-(r - 1), r):
        w = window_half_width(r, abs(dy), window)
        for dx in range(-w, w + 1):
            total += max(0, H - abs(dy)) * max(0, W - abs(dx))
    return total


def kept_pairs(n_text: int, H: int, W: int, r: int, window: str = "circle") -> int:
    """Number of ones in M: text rows (all T keys) + image rows x text keys + window pairs."""
    N = H * W
    T = n_text + N
    return n_text * T + N * n_text + window_pairs(H, W, r, window)


def useful_flops_fwd(B: int, heads: int, n_text: int, H: int, W: int, r: int, d: int,
                     window: str = "circle") -> int:
    """Forward FLOPs on kept pairs only: 2*d for q.k plus 2*d for p*v, per kept (q, k) pair."""
    return 4 * d * B * heads * kept_pairs(n_text, H, W, r, window)


# ----------------------------------------------------------------------------------------------
# Patch-parallel inference: stripes of the grid and the patch-wise text approximation
# ----------------------------------------------------------------------------------------------

def clear_attention_stripe(q, k, v, n_text: int, H: int, W: int, r: int, q_row0: int, q_row1: int,
                           key_row0: int, key_row1: int, text_keys: bool, scale=None, window: str = "circle"):
    """Forward of one stripe of a patch-parallel split [pith review, "If this is right": adjacent
    patches exchange only O(r x W) boundary tokens].

    The problem (q, k, v, n_text, H, W) is the stripe itself: text tokens, then its H grid rows
    (halo rows included). Image query rows [q_row0, q_row1) get the ordinary CLEAR rows of this
    problem (mask of the stripe grid). Text query rows get one softmax over the keys the stripe
    names: the text tokens if text_keys, and the image tokens of rows [key_row0, key_row1).
    Returns (O_text [B, heads, n_text, d], LSE_text [B, heads, n_text],
             O_img [B, heads, (q_row1 - q_row0) * W, d], LSE_img [B, heads, (q_row1 - q_row0) * W]).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hh, T, d = q.shape
    assert T == n_text + H * W
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    img_rows = list(range(n_text + q_row0 * W, n_text + q_row1 * W))
    M_img = clear_mask(n_text, H, W, r, rows=img_rows, window=window)
    keep_txt = np.zeros(T, dtype=bool)
    if text_keys:
        keep_txt[:n_text] = True
    keep_txt[n_text + key_row0 * W:n_text + key_row1 * W] = True
    Ot = np.empty((B, Hh, n_text, d))
    Lt = np.empty((B, Hh, n_text))
    Oi = np.empty((B, Hh, len(img_rows), d))
    Li = np.empty((B, Hh, len(img_rows)))
    for b in range(B):
        for h in range(Hh):
            if n_text:
                S = (q[b, h, :n_text] @ k[b, h].T) * scale
                P, lse = _masked_softmax_rows(S, np.broadcast_to(keep_txt, S.shape))
                Ot[b, h], Lt[b, h] = P @ v[b, h], lse
            S = (q[b, h, img_rows] @ k[b, h].T) * scale
            P, lse = _masked_softmax_rows(S, M_img)
            Oi[b, h], Li[b, h] = P @ v[b, h], lse
    return Ot, Lt, Oi, Li


def clear_text_rows_patch_average(q, k, v, n_text: int, H: int, W: int, row_bounds, scale=None):
    """The patch-wise text approximation of Eq. 7 [pith review, "What carries the argument"]: text
    query rows averaged over N patches, O_text = (1/N) sum_p softmax(Q_text K_p^T * scale) V_p.

    Patch p holds grid rows [row_bounds[p], row_bounds[p+1]). The pages leave open whether K_p, V_p
    hold the text tokens too (the review's referee comment on Eq. 7); read here as yes: each GPU of
    a patch-parallel run holds the text tokens and its own image rows, so K_p, V_p are the text
    tokens followed by patch p's image tokens. Returns O_text [B, heads, n_text, d] in float64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hh, T, d = q.shape
    assert T == n_text + H * W and row_bounds[0] == 0 and row_bounds[-1] == H
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    n = len(row_bounds) - 1
    O = np.zeros((B, Hh, n_text, d))
    for p in range(n):
        cols = list(range(n_text)) + list(range(n_text + row_bounds[p] * W, n_text + row_bounds[p + 1] * W))
        for b in range(B):
            for h in range(Hh):
                S = (q[b, h, :n_text] @ k[b, h, cols].T) * scale
                P, _ = _masked_softmax_rows(S, np.ones_like(S, dtype=bool))
                O[b, h] += P @ v[b, h, cols]
    return O / n


# ----------------------------------------------------------------------------------------------
# FP8 (E4M3) score products
# ----------------------------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Value of each OCP FP8 E4M3 code (uint8 array) as float64: (-1)^s * 2^(e-7) * (1 + m/8) for
    exponent field e in 1..15, (-1)^s * 2^-6 * (m/8) for e = 0 (subnormals, including +-0), and
    NaN for the codes with e = 15 and m = 7 (0x7F, 0xFF)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, v)


def clear_attention_forward_fp8(q8, k8, v, s_q, s_k, n_text: int, H: int, W: int, r: int, scale=None,
                                window: str = "circle"):
    """CLEAR forward with E4M3 query and key codes. q8, k8: uint8 codes [B, heads, T, d]; v: values
    [B, heads, T, d]; s_q, s_k: dequantization scales [B, heads]. Returns (O, LSE) in float64 of
    the plain forward on q = decode(q8) * s_q, k = decode(k8) * s_k."""
    q8 = q8.detach().cpu().numpy() if hasattr(q8, "detach") else np.asarray(q8)
    k8 = k8.detach().cpu().numpy() if hasattr(k8, "detach") else np.asarray(k8)
    sq = _as_f64(s_q)[:, :, None, None]
    sk = _as_f64(s_k)[:, :, None, None]
    return clear_attention_forward(e4m3_decode(q8) * sq, e4m3_decode(k8) * sk, v, n_text, H, W, r, scale=scale,
                                   window=window)


# ----------------------------------------------------------------------------------------------
# Rotary position embedding (axial 2D, interleaved pairs, NTK-aware base)
# ----------------------------------------------------------------------------------------------

def rope_inv_freq(d_axis: int, theta: float = 10000.0, ntk: float = 1.0) -> np.ndarray:
    """Rotation rate of each dim pair of one axis: base^(-2i/d_axis), i = 0 .. d_axis/2 - 1, with
    the NTK-aware base theta * ntk^(d_axis / (d_axis - 2))."""
    base = theta * ntk ** (d_axis / (d_axis - 2.0))
    return base ** (-np.arange(0, d_axis, 2, dtype=np.float64) / d_axis)


def rope_2d(x, n_text: int, H: int, W: int, theta: float = 10000.0, ntk: float = 1.0,
            inverse: bool = False) -> np.ndarray:
    """Axial 2D rotary embedding of x [..., T, d] (float64 copy): image token (y, x) has dims
    [0, d/2) rotated by y and dims [d/2, d) by x, pair (2i, 2i+1) of an axis by angle
    position * rope_inv_freq(d/2)[i]: (a, b) -> (a cos - b sin, a sin + b cos). Text tokens are
    unchanged. inverse=True turns every pair by the negated angle: each 2x2 rotation is orthogonal,
    so that is its transpose and its inverse (what carries a gradient back through the embedding)."""
    x = _as_f64(x).copy()
    d = x.shape[-1]
    assert d % 4 == 0
    da = d // 2
    inv = rope_inv_freq(da, theta, ntk)
    y_pos, x_pos, is_text = token_coords(n_text, H, W)
    img = ~is_text
    for axis, pos in ((0, y_pos), (1, x_pos)):
        ang = pos[img][:, None] * inv[None, :]          # [N, da/2]
        if inverse:
            ang = -ang
        c, s_ = np.cos(ang), np.sin(ang)
        a = x[..., img, axis * da + 0:axis * da + da:2].copy()
        b = x[..., img, axis * da + 1:axis * da + da:2].copy()
        x[..., img, axis * da + 0:axis * da + da:2] = a * c - b * s_
        x[..., img, axis * da + 1:axis * da + da:2] = a * s_ + b * c
    return x


def clear_attention_forward_rope(q, k, v, n_text: int, H: int, W: int, r: int, theta: float = 10000.0,
                                 ntk: float = 1.0, scale=None, window: str = "circle"):
    """The plain forward on rope_2d(q) and rope_2d(k) (v unchanged). Returns (O, LSE) in float64."""
    return clear_attention_forward(rope_2d(q, n_text, H, W, theta, ntk), rope_2d(k, n_text, H, W, theta, ntk), v,
                                   n_text, H, W, r, scale=scale, window=window)
