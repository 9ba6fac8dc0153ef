/*
 * clear_attn.h — C ABI of the B200 (sm_100a) CLEAR attention library (libclear_attn.so).
 *
 * CLEAR ("CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion Transformers Up",
 * arXiv 2412.16112) replaces full attention in a diffusion transformer by a mask that keeps a
 * (query i, key j) pair iff i is a text token, or j is a text token, or image tokens i and j lie at
 * squared Euclidean grid distance dx^2 + dy^2 < r^2 (pith.science review, "Core claim"; atlas.scime.ai
 * summary, "Approach"). Each query row takes one softmax over its kept keys, with scores scaled by
 * 1/sqrt(d) (pith.science review, "What carries the argument", Eq. 7 text).
 *
 * Conventions shared by every call
 * --------------------------------
 * Tensors are dense, row-major, on the current CUDA device, with shape [B, heads, T, d] where
 * T = n_text + H*W: the n_text text tokens come first, then the image tokens of an H x W grid in
 * row-major order (token n_text + y*W + x is grid position (y, x)). Element type is bf16 for
 * q, k, v, o, dO, dq, dk, dv; lse is fp32 [B, heads, T], natural log of the softmax denominator
 * of the scaled, masked scores. Every pointer must be 16-byte aligned.
 *
 * Windows are clipped at the grid border (border queries see fewer keys). Text query rows attend
 * to all T keys exactly. r is an integer >= 1; any r whose square exceeds the grid diagonal's
 * square keeps every pair (full attention). Supported head dims: d = 64 and d = 128.
 *
 * Ownership: the caller owns every buffer and the stream. The library allocates no device memory
 * in these calls; scratch space comes from the caller's workspace (size from the *_workspace_size
 * queries). Outputs are written in full; inputs are never written.
 *
 * Asynchrony and errors: calls enqueue kernels on `stream` (a cudaStream_t passed as void*;
 * NULL = legacy default stream) and return without synchronising. Argument errors are detected on
 * the host before anything is launched: the call returns the error status and leaves every output
 * untouched. A kernel whose internal bounded wait expired records a device error word instead of
 * hanging; clear_attn_check() synchronises the stream and reports it as CLEAR_ERR_DEVICE_TIMEOUT.
 * Calls are thread-safe: the only mutable global state is the device error word, the
 * allocation-free forward's scratch array and the host-buffer forward's per-device copy streams
 * (created once, under a lock).
 */
#ifndef CLEAR_ATTN_H_
#define CLEAR_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(CLEAR_BUILD_SO) && defined(__GNUC__)
#define CLEAR_API __attribute__((visibility("default")))
#else
#define CLEAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CLEAR_OK = 0,
  CLEAR_ERR_INVALID_ARG = 1,      /* null/misaligned pointer, non-positive size, r < 1, overflow */
  CLEAR_ERR_UNSUPPORTED = 2,      /* d not in {64, 128}, or no sm_100 device */
  CLEAR_ERR_WORKSPACE = 3,        /* workspace missing or smaller than the queried size */
  CLEAR_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed (launch, tensor map) */
  CLEAR_ERR_DEVICE_TIMEOUT = 5    /* a kernel's bounded wait expired (reported by clear_attn_check) */
} clear_status_t;

/* Problem description. All fields are plain element counts. */
typedef struct {
  int B;        /* batch size, >= 1 */
  int heads;    /* attention heads, >= 1 */
  int n_text;   /* text tokens placed before the image tokens, >= 0 */
  int H, W;     /* image token grid, >= 1 each */
  int d;        /* head dim: 64 or 128 */
  int r;        /* window radius in grid units (strict: dx^2 + dy^2 < r^2), >= 1 */
  int window;   /* CLEAR_WINDOW_CIRCLE (0, CLEAR's mask); CLEAR_WINDOW_SQUARE (1): keep image pairs
                   with |dx| < r and |dy| < r instead, the square sliding window the pages compare
                   the circle with; CLEAR_WINDOW_SHIFTED (2): the same square around a centre
                   clamped to [r-1, H-r] x [r-1, W-r] (neighborhood-attention style: every image
                   query keeps (2r-1)^2 image keys), which needs H, W >= 2r-1 (else
                   CLEAR_ERR_INVALID_ARG) and has no backward (CLEAR_ERR_UNSUPPORTED from
                   clear_attn_bwd and its workspace query). Any other value is
                   CLEAR_ERR_INVALID_ARG. */
} clear_attn_params_t;

enum { CLEAR_WINDOW_CIRCLE = 0, CLEAR_WINDOW_SQUARE = 1, CLEAR_WINDOW_SHIFTED = 2 };

/* Library version (major * 10000 + minor * 100 + patch). */
CLEAR_API int clear_attn_version(void);

/* Human-readable name of a status code (static storage). */
CLEAR_API const char* clear_status_string(clear_status_t status);

/* Bytes of caller-provided device workspace clear_attn_fwd needs (0 when n_text == 0).
 * Returns 0 and sets *status (if non-NULL) on invalid params. */
CLEAR_API size_t clear_attn_fwd_workspace_size(const clear_attn_params_t* params, clear_status_t* status);

/* Bytes of caller-provided device workspace clear_attn_bwd needs. */
CLEAR_API size_t clear_attn_bwd_workspace_size(const clear_attn_params_t* params, clear_status_t* status);

/*
 * Forward: o = softmax_M(q k^T / sqrt(d)) v, lse = log sum_j exp(q_i.k_j / sqrt(d)) over kept j.
 *   q, k, v   in : bf16 [B, heads, T, d]
 *   o         out: bf16 [B, heads, T, d]
 *   lse       out: fp32 [B, heads, T]
 *   workspace in/out scratch: device memory of at least clear_attn_fwd_workspace_size() bytes
 *             (may be NULL when that size is 0); contents are undefined on return.
 *   stream    cudaStream_t (as void*).
 */
CLEAR_API clear_status_t clear_attn_fwd(const clear_attn_params_t* params, const void* q, const void* k,
                              const void* v, void* o, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Element strides of q, k, v and o for clear_attn_fwd_strided: {batch, head, token} for each
 * tensor, in elements (not bytes). The d elements of one token row are contiguous. */
typedef struct {
  long long q[3], k[3], v[3], o[3];
} clear_attn_strides_t;

/*
 * Forward on strided tensors: the same operation and results as clear_attn_fwd (bit for bit: the
 * arithmetic and its order are the same), but element (b, h, t, i) of q is read at
 *   q + b * strides->q[0] + h * strides->q[1] + t * strides->q[2] + i
 * (likewise k, v), and row (b, h, t) of o is written at the same place of o with strides->o. This
 * reads, e.g., a packed [B, T, 3, heads, d] qkv buffer (q = buf, k = buf + heads*d,
 * v = buf + 2*heads*d, strides {T*3*heads*d, d, 3*heads*d}) and writes o as [B, T, heads, d], with
 * no copy. The paper has no counterpart (its model feeds attention from such a packed projection).
 *   strides  every stride a positive multiple of 8 elements (16 bytes, as TMA requires) and below
 *            2^39, else CLEAR_ERR_UNSUPPORTED; NULL is CLEAR_ERR_INVALID_ARG. Overlapping o rows
 *            are the caller's error (results undefined).
 *   lse      fp32 [B, heads, T], contiguous, as in clear_attn_fwd.
 *   Pointers 16-byte aligned; workspace as for clear_attn_fwd (same size query).
 */
CLEAR_API clear_status_t clear_attn_fwd_strided(const clear_attn_params_t* params, const clear_attn_strides_t* strides,
                                                const void* q, const void* k, const void* v, void* o, float* lse,
                                                void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Patch-parallel inference (pith.science review of the CLEAR paper, "If this is right": adjacent
 * patches exchange only O(r x W) boundary tokens; "What carries the argument": Eq. 7). Each GPU
 * holds the text tokens and a stripe of image rows; a circular window of radius r reaches r - 1
 * rows, so a stripe extended by r - 1 halo rows on each side holds every key its own image
 * queries keep. Its text queries see a disjoint share of the keys, and the shares' text-row
 * outputs are merged exactly (log-sum-exp weights) or by the paper's patch-wise average.
 * --------------------------------------------------------------------------------------------- */

/* A stripe of the problem given in clear_attn_params_t (whose H x W grid is the stripe,
 * halo rows included). Rows are grid rows of the stripe. */
typedef struct {
  int q_row0, q_row1;     /* image query rows computed and written: [q_row0, q_row1), 0 <= q_row0 < q_row1 <= H */
  int key_row0, key_row1; /* image keys the text query rows see: rows [key_row0, key_row1) (may be empty) */
  int text_keys;          /* 1: text query rows also see the n_text text keys; 0: they do not */
} clear_attn_stripe_t;

/* Workspace bytes clear_attn_fwd_stripe needs (the text rows' split partials for this key set). */
CLEAR_API size_t clear_attn_fwd_stripe_workspace_size(const clear_attn_params_t* params,
                                                      const clear_attn_stripe_t* stripe, clear_status_t* status);

/*
 * Forward of one stripe. q, k, v, o: bf16 [B, heads, n_text + H*W, d] of the stripe (text tokens,
 * then the stripe's rows, halos included); lse fp32 [B, heads, n_text + H*W]. Image query rows
 * [q_row0, q_row1) attend, as in clear_attn_fwd, to all text keys and to the image keys of the
 * stripe within their window (windows are clipped at the stripe's edges, which halos of r - 1 rows
 * keep away from the computed rows). Text query rows attend to the keys the stripe names (see
 * clear_attn_stripe_t) and are normalised over them, with their lse. Only these rows of o and lse
 * are written; the halo rows are left untouched. The circle and square windows are offered; the
 * shifted window is CLEAR_ERR_UNSUPPORTED (its centre clamping needs the whole grid). Invalid row
 * ranges, or text rows left without any key, are CLEAR_ERR_INVALID_ARG. Otherwise as clear_attn_fwd.
 */
CLEAR_API clear_status_t clear_attn_fwd_stripe(const clear_attn_params_t* params, const clear_attn_stripe_t* stripe,
                                               const void* q, const void* k, const void* v, void* o, float* lse,
                                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Merges the text query rows of n_parts stripe forwards. params gives B, heads, n_text, d (H, W, r
 * are only checked). o_parts: bf16 [n_parts, B, heads, n_text, d] and lse_parts: fp32
 * [n_parts, B, heads, n_text], part p's text rows (normalised over its keys, and their lse); o: bf16
 * [B, heads, n_text, d], lse: fp32 [B, heads, n_text].
 *   mode 0: exact. lse = log sum_p exp(lse_p), o = sum_p exp(lse_p - lse) o_p: the softmax over the
 *           union of the parts' keys, which must be disjoint (text keys in exactly one part).
 *   mode 1: Eq. 7 of the paper, o = (1/n_parts) sum_p o_p, each part's keys being the text tokens
 *           and its own image rows; lse is written as in mode 0.
 * A part without keys (lse_p = -inf) has weight 0 in mode 0. CLEAR_ERR_INVALID_ARG for n_parts
 * outside [1, 4096], another mode, n_text = 0 or misaligned pointers.
 */
CLEAR_API clear_status_t clear_attn_text_merge(const clear_attn_params_t* params, int n_parts, int mode,
                                               const void* o_parts, const float* lse_parts, void* o, float* lse,
                                               void* stream);

/*
 * Forward with FP8 score products: q and k as OCP FP8 E4M3 codes (one byte per element), v in
 * bf16. The scores are the products of the decoded codes, scaled by qk_descale[b * heads + h]
 * (= s_q * s_k, the two inputs' dequantization scales) and by 1/sqrt(d); everything after the
 * scores (mask, softmax, P rounded to bf16, P V, O and LSE) is as in clear_attn_fwd (the CLEAR mask of
 * the pith.science review of "CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion
 * Transformers Up", "Core claim"; the paper has no FP8 path). The score products run as
 * tcgen05.mma kind::f8f6f4 at twice the bf16 rate on half the q and k bytes.
 *   q8, k8: uint8 [B, heads, T, d] contiguous, d = 128 (other d: CLEAR_ERR_UNSUPPORTED);
 *   v, o: bf16 [B, heads, T, d]; lse: fp32 [B, heads, T]; qk_descale: device fp32 [B * heads];
 *   workspace: clear_attn_fwd_workspace_size bytes (same as the bf16 forward).
 * Otherwise as clear_attn_fwd.
 */
CLEAR_API clear_status_t clear_attn_fwd_fp8(const clear_attn_params_t* params, const void* q8, const void* k8,
                                            const void* v, const float* qk_descale, void* o, float* lse,
                                            void* workspace, size_t workspace_bytes, void* stream);

/* Rotary position embedding applied by clear_attn_fwd_rope. */
typedef struct {
  float theta;  /* RoPE base, > 1 (10000 in RoFormer) */
  float ntk;    /* NTK-aware scale factor alpha > 0 (1: plain RoPE; the review lists 10 for CLEAR) */
} clear_attn_rope_t;

/* Workspace bytes of clear_attn_fwd_rope: the forward's, the (cos, sin) table, the rotated q and k
 * (2 * B * heads * T * d bf16 values). */
CLEAR_API size_t clear_attn_fwd_rope_workspace_size(const clear_attn_params_t* params, clear_status_t* status);

/*
 * The forward on rotary-embedded q and k: one streaming pass rotates q and k (HBM-bound, each
 * element read and written once, rounded to bf16 once) into the workspace, then the CLEAR forward
 * of clear_attn_fwd runs on the rotated copies; v is used as given. The rotary embedding is axial
 * 2D with interleaved pairs (RoFormer's rotary embedding and NTK-aware scaled RoPE, both cited by
 * the paper; the pith.science review of "CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion
 * Transformers Up" lists the NTK scale factor 10): image token (y, x) has head dims [0, d/2)
 * rotated by y and [d/2, d) by x, pair (2i, 2i+1) of an axis by the angle
 * position * base^(-2i/(d/2)), base = theta * ntk^((d/2)/(d/2 - 2)), (a, b) -> (a cos - b sin,
 * a sin + b cos); text tokens are not rotated. The (cos, sin) table is evaluated on the device in
 * double and rounded to fp32. Tensors as clear_attn_fwd (contiguous; d = 64 or 128); the inputs are
 * not modified. workspace: clear_attn_fwd_rope_workspace_size bytes, 256-byte aligned, written on
 * `stream` (calls that overlap on the GPU need their own workspaces); no host synchronisation, so
 * the call can be captured in a CUDA graph. CLEAR_ERR_INVALID_ARG for theta <= 1, ntk <= 0 or
 * non-finite values; otherwise as clear_attn_fwd.
 */
CLEAR_API clear_status_t clear_attn_fwd_rope(const clear_attn_params_t* params, const clear_attn_rope_t* rope,
                                             const void* q, const void* k, const void* v, void* o, float* lse,
                                             void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of clear_attn_rope: the (cos, sin) table, max(H, W) * d/4 fp32 pairs, rounded up to
 * 256 bytes. */
CLEAR_API size_t clear_attn_rope_workspace_size(const clear_attn_params_t* params, clear_status_t* status);

/*
 * The rotary embedding of clear_attn_fwd_rope on its own: q and k (bf16 [B, heads, T, d],
 * contiguous, d = 64 or 128) rotated into q_out and k_out, each element read and written once and
 * rounded to bf16 once; text tokens are copied unchanged. inverse = 1 turns every pair by the
 * negated angle, the transpose of the rotation (each 2x2 rotation is orthogonal): rotating the
 * gradients of the rotated q and k back with it gives the gradients of q and k, so a training step
 * can rotate once, run clear_attn_fwd and clear_attn_bwd on the rotated tensors, and rotate dQ, dK
 * back. q_out may be q and k_out may be k (in place). workspace: clear_attn_rope_workspace_size
 * bytes, 256-byte aligned, written on `stream`. CLEAR_ERR_INVALID_ARG for theta <= 1, ntk <= 0,
 * non-finite values, inverse other than 0 or 1, or misaligned pointers; CLEAR_ERR_WORKSPACE for a
 * small or misaligned workspace; otherwise as clear_attn_fwd.
 */
CLEAR_API clear_status_t clear_attn_rope(const clear_attn_params_t* params, const clear_attn_rope_t* rope, int inverse,
                                         const void* q, const void* k, void* q_out, void* k_out, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* Workspace bytes of clear_attn_bwd_rope: the backward's, the (cos, sin) table, the rotated q and k. */
CLEAR_API size_t clear_attn_bwd_rope_workspace_size(const clear_attn_params_t* params, clear_status_t* status);

/*
 * The backward of clear_attn_fwd_rope: the gradients with respect to the unrotated q, k and v.
 * q and k are rotated into the workspace as the forward saw them, clear_attn_bwd runs on the
 * rotated tensors (o and lse are the ones clear_attn_fwd_rope returned), and dq, dk are then turned
 * back by the inverse rotation, the transpose of the rotation (each 2x2 rotation is orthogonal),
 * in place; dv needs no turn. Tensors as clear_attn_bwd (contiguous; d = 64 or 128; the shifted
 * window is CLEAR_ERR_UNSUPPORTED as there). workspace: clear_attn_bwd_rope_workspace_size bytes,
 * 256-byte aligned, written on `stream`. CLEAR_ERR_INVALID_ARG for the rotary parameters as in
 * clear_attn_fwd_rope; otherwise as clear_attn_bwd.
 */
CLEAR_API clear_status_t clear_attn_bwd_rope(const clear_attn_params_t* params, const clear_attn_rope_t* rope,
                                             const void* q, const void* k, const void* v, const void* o,
                                             const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Mixed-resolution batch forward: n_items problems of their own (n_text, H, W) in ONE launch (their
 * pairs form one work list), e.g. a batch holding 1024^2 and 2048^2 images at once. Each item is the
 * CLEAR forward of clear_attn_fwd (pith.science review of "CLEAR: Conv-Like Linearization Revs
 * Pre-Trained Diffusion Transformers Up", "Core claim": text rows and text keys global, image keys
 * within radius r on the item's own grid); items never attend to each other.
 *   params: heads, d, r and window are shared by every item; B, n_text, H and W are not used.
 *   item_shapes: host int[3 * n_items], item i = (n_text_i, H_i, W_i), each checked as clear_attn_fwd
 *     checks its params (n_items in [1, 4096]).
 *   q, k, v, o: bf16 [heads, T_total, d] with T_total = sum_i (n_text_i + H_i * W_i); item i's tokens
 *     (text first, then its grid row-major) start at token sum_{j<i} T_j. lse: fp32 [heads, T_total].
 *   workspace: device memory of clear_attn_fwd_varlen_workspace_size bytes, 256-byte aligned; the
 *     call copies the items' geometry and tensor maps into it (an asynchronous copy on `stream`)
 *     before launching, so a workspace must not be shared by calls that overlap on the GPU.
 * The radius is clamped once, to the largest full-grid radius among the items (an item whose own
 * grid is smaller keeps all its pairs either way). Results equal clear_attn_fwd on each item alone.
 * CLEAR_ERR_INVALID_ARG for a bad item or count, misaligned pointers or T_total > 2^30;
 * CLEAR_ERR_WORKSPACE for a short or misaligned workspace.
 */
CLEAR_API size_t clear_attn_fwd_varlen_workspace_size(const clear_attn_params_t* params, int n_items,
                                                      const int* item_shapes, clear_status_t* status);
CLEAR_API clear_status_t clear_attn_fwd_varlen(const clear_attn_params_t* params, int n_items, const int* item_shapes,
                                               const void* q, const void* k, const void* v, void* o, float* lse,
                                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward for callers that cannot allocate device memory: same inputs, outputs and results as
 * clear_attn_fwd (up to the summation order of the text rows), but no workspace argument. The
 * paper has no counterpart; this entry point exists for integration. Some callers cannot call
 * cudaMalloc or hand out scratch buffers: a plugin invoked inside another framework's execution
 * step, where allocating would break that framework's memory plan, or a serving loop that reserved
 * all device memory up front. This call uses a scratch array of 32 MiB compiled into the library
 * instead (a static __device__ array: every GPU that loads the library holds it until exit), and
 * allocates nothing itself.
 *   - The text-row split count is lowered until the split partials fit in the 32 MiB; if one split
 *     of B * heads * n_text rows (4 * d + 8 bytes each) does not fit, the call returns
 *     CLEAR_ERR_WORKSPACE and launches nothing.
 *   - The first call on a device looks up the scratch array's device address (with that device
 *     current); make that first call before any stream capture, and before reserving the rest
 *     of device memory: the lookup can load the library's device code, which holds the array.
 *     A failed lookup returns CLEAR_ERR_CUDA, is not remembered (the next call tries again) and
 *     leaves no pending CUDA error behind.
 *   - All calls share the one array and it keeps the last call's contents. Nothing in it needs to
 *     start at zero: every value a call reads there is written earlier in the same call. Calls
 *     that overlap on the GPU (different streams, or different host threads) race on it.
 */
CLEAR_API clear_status_t clear_attn_fwd_noalloc(const clear_attn_params_t* params, const void* q, const void* k,
                                      const void* v, void* o, float* lse, void* stream);

/* Bytes of caller-provided device workspace clear_attn_fwd_host needs: device copies of q, k, v,
 * o and lse, plus clear_attn_fwd's workspace for one slice group. Returns 0 and sets *status (if
 * non-NULL) on invalid params. */
CLEAR_API size_t clear_attn_fwd_host_workspace_size(const clear_attn_params_t* params, clear_status_t* status);

/*
 * Forward from and to HOST memory, for callers whose tensors live on the host (the paper has no
 * counterpart; this is the transfer-overlapped form of clear_attn_fwd). The B * heads slices are
 * split into up to 24 groups of consecutive slices; each group's q, k, v are copied to the
 * device, its forward runs (one clear_attn_fwd call with B = 1, heads = group size), and its o
 * and lse are copied back. Copies run on two library-owned non-blocking streams per device
 * (created on first use, kept until exit), so the input copy of one group, the forward of the
 * previous one and the return copy of the one before overlap.
 *   q_host, k_host, v_host in : bf16 [B, heads, T, d] in page-locked host memory
 *   o_host                 out: bf16 [B, heads, T, d] in page-locked host memory
 *   lse_host               out: fp32 [B, heads, T] in page-locked host memory
 *   workspace              device scratch of at least clear_attn_fwd_host_workspace_size() bytes;
 *                          it receives the device copies, so its contents are undefined on return.
 *   stream                 the copies start after the work already queued on `stream`, and work
 *                          queued on `stream` after this call runs after o_host and lse_host are
 *                          written: synchronise `stream` before reading them on the host.
 * Results: those of clear_attn_fwd on the same inputs. Slices are independent and each group runs
 * the same kernels with the same text split count (it depends only on T).
 * Errors (nothing is launched): CLEAR_ERR_INVALID_ARG for a host pointer that is NULL, not 16-byte
 * aligned or not page-locked (pageable memory cannot overlap; cudaHostAlloc or cudaHostRegister
 * it), CLEAR_ERR_WORKSPACE for a missing or short workspace, and the argument errors of
 * clear_attn_fwd. CLEAR_ERR_CUDA if a copy, event or stream call fails.
 */
CLEAR_API clear_status_t clear_attn_fwd_host(const clear_attn_params_t* params, const void* q_host,
                                             const void* k_host, const void* v_host, void* o_host,
                                             float* lse_host, void* workspace, size_t workspace_bytes,
                                             void* stream);

/*
 * Backward of clear_attn_fwd with respect to q, k and v, given the upstream gradient dO and the
 * forward's o and lse (analytic softmax-attention gradient restricted to the mask):
 *   dV = P^T dO;  dP = dO V^T;  D = rowsum(dO o O);  dS = P o (dP - D);
 *   dQ = dS K / sqrt(d);  dK = dS^T Q / sqrt(d).
 *   q, k, v, o, dO  in : bf16 [B, heads, T, d];  lse in: fp32 [B, heads, T]
 *   dq, dk, dv      out: bf16 [B, heads, T, d]
 *   workspace       scratch of at least clear_attn_bwd_workspace_size() bytes.
 */
CLEAR_API clear_status_t clear_attn_bwd(const clear_attn_params_t* params, const void* q, const void* k,
                              const void* v, const void* o, const float* lse, const void* dO,
                              void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the current device.
 * Returns CLEAR_OK, CLEAR_ERR_DEVICE_TIMEOUT (a kernel gave up a bounded wait; its outputs are
 * invalid) or CLEAR_ERR_CUDA (the stream reported a CUDA error). */
CLEAR_API clear_status_t clear_attn_check(void* stream);

/* Context of the expired wait behind the last CLEAR_ERR_DEVICE_TIMEOUT that clear_attn_check()
 * returned on this host thread (zeros if none): {code (1 producer, 3 MMA, 4 softmax), wait site,
 * CTA index, thread index, phase parity (-1 for a polling loop), three site-specific counters}.
 * For diagnosis only; the layout may change between versions. */
CLEAR_API void clear_attn_device_diag(int* out8);

/* Self-test of the failure-detection path (the paper has no counterpart). Launches, on `stream`,
 * one small kernel whose single waiting thread waits on a shared-memory barrier that nothing ever
 * arrives on; after `limit_ms` milliseconds (1..5000) the wait gives up, records the expiry in the
 * same device error word and diagnostic record the attention kernels use (code 5, wait site 31)
 * and the kernel returns. Nothing faults or hangs, and the CUDA context stays usable. The caller
 * then sees CLEAR_ERR_DEVICE_TIMEOUT from clear_attn_check(stream), which also clears the word,
 * and the record from clear_attn_device_diag().
 * Returns CLEAR_OK once the kernel is launched, CLEAR_ERR_INVALID_ARG for a limit outside 1..5000
 * (checked before any CUDA call), CLEAR_ERR_UNSUPPORTED on a device other than sm_100,
 * CLEAR_ERR_CUDA if the launch fails. It shares the device error word with every other call on
 * the device: do not run it concurrently with attention calls whose status you need. */
CLEAR_API clear_status_t clear_attn_selftest_expiry(int limit_ms, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Host-only scheduler queries (no GPU needed). They expose the tile enumeration the kernels use,
 * so its coverage can be checked against a brute-force mask on the CPU.
 * --------------------------------------------------------------------------------------------- */

/* Work-list shape of the forward. The forward works on pairs of 128-row query tiles that share
 * their 64-key tiles: pairs of consecutive text tiles (split over key ranges) and 16 x 16 image
 * blocks (upper and lower 8 x 16 halves). Returns the numbers of text pairs (all splits) and image
 * pairs, the text split count S and the 64-key chunks per split. Any output may be NULL. */
CLEAR_API clear_status_t clear_sched_forward_shape(const clear_attn_params_t* params, long long* n_text_items,
                                         long long* n_image_items, int* splits,
                                         int* chunks_per_split);

/* Union key tiles visited by forward pair `item` (0 <= item < n_text_items + n_image_items), in
 * order. Each tile is 4 ints: kind (0 = linear chunk, 1 = image rectangle), a, b, flags.
 * Linear: tokens [a, a + 64), first b of them real. Rectangle: grid rows [a, a + 4) x columns
 * [b, b + 16). flags: bit 0 / bit 1 = half A / half B needs the tile (some kept pair), bit 2 /
 * bit 3 = every pair of half A / half B with the tile is kept (no mask). q_info = {is_text, bh,
 * q0 (first token of half A, or first grid row of the block), x0 (first grid column), half B
 * holds real queries}. Writes at most max_tiles tiles; the total count goes to *n_tiles. */
CLEAR_API clear_status_t clear_sched_item_tiles(const clear_attn_params_t* params, long long item,
                                      int* q_info, int* tiles, int max_tiles, int* n_tiles);

/* clear_sched_forward_shape and clear_sched_item_tiles for the forward of a stripe (see
 * clear_attn_fwd_stripe): image pairs cover query rows [q_row0, q_row1); text pairs visit the
 * stripe's text-row key ranges (the text tokens if text_keys, then rows [key_row0, key_row1), each
 * range in 64-token chunks from its own first token). */
CLEAR_API clear_status_t clear_sched_stripe_forward_shape(const clear_attn_params_t* params,
                                                          const clear_attn_stripe_t* stripe, long long* n_text_items,
                                                          long long* n_image_items, int* splits, int* chunks_per_split);
CLEAR_API clear_status_t clear_sched_stripe_item_tiles(const clear_attn_params_t* params,
                                                       const clear_attn_stripe_t* stripe, long long item, int* q_info,
                                                       int* tiles, int max_tiles, int* n_tiles);

/* Useful (kept-pair) and executed (padded-tile) multiply-add pair counts of one forward call,
 * summed over B and heads: useful = number of ones in the mask; executed = 128 x 64 per tile
 * product the forward issues (a half times a key tile it needs). FLOPs are 4 * d times these. */
CLEAR_API clear_status_t clear_sched_pair_counts(const clear_attn_params_t* params, long long* useful_pairs,
                                       long long* executed_pairs);

#ifdef __cplusplus
}
#endif

#endif /* CLEAR_ATTN_H_ */
