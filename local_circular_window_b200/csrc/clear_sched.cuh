// CLEAR tile scheduler: which key tiles each query tile must visit.
//
// The CLEAR mask (pith.science review of "CLEAR: Conv-Like Linearization Revs Pre-Trained
// Diffusion Transformers Up", section "Core claim") keeps (i, j) iff i is a text token, or j is a
// text token, or image tokens i and j lie at squared grid distance dx^2 + dy^2 < r^2. Text tokens
// come first; image token (y, x) sits at n_text + y*W + x.
//
// Work is cut into query tiles of 128 rows:
//   * image query tiles: an 8 x 16 rectangle of grid positions (kQH x kQW);
//   * text query tiles: 128 consecutive token rows starting at a multiple of 128 (rows past
//     n_text are computed and discarded).
// Key tiles are 128 keys:
//   * linear chunks (kind kLinear): keys [a, a + 128) in token order, `valid` of them real;
//   * image rectangles (kind kRect): grid rows [ky, ky + 8) x columns [kx, kx + 16).
//
// An image query tile visits the text chunks covering [0, n_text) and then, band by band (8 key
// rows at a time), the 16-column rectangles that cover the union of its queries' circular
// windows in that band. The band's column range is set by the band's smallest vertical distance
// to the query tile, so every key within radius of some query in the tile is visited exactly once,
// and rectangles the disc never reaches are skipped. A rectangle whose every (query, key) pair is
// within radius and inside the grid is flagged kFull (no mask needed).
//
// Text query tiles visit all linear chunks over [0, T), split into `S` contiguous ranges
// ("splits") so the 512 text rows can spread over many SMs; the splits are merged by a
// log-sum-exp combine.
//
// This header is compiled for both host and device: the kernels enumerate tiles on the fly with
// it, and the host-side query API exposes the same enumeration to the tests.
#pragma once
#include <cstdint>

#ifndef __CUDACC__
#define CLEAR_HD
#else
#define CLEAR_HD __host__ __device__ __forceinline__
#endif

namespace clear {

constexpr int kQH = 8;      // image query tile rows
constexpr int kQW = 16;     // image query tile columns
constexpr int kKH = 8;      // image key tile rows
constexpr int kKW = 16;     // image key tile columns
constexpr int kTile = 128;  // rows per query tile, keys per key tile
// The forward pairs two query tiles and visits 64-key tiles: 4 x 16 grid rectangles or 64-token
// chunks (half-size key tiles let each half double-buffer S in tensor memory).
constexpr int kFKH = 4;       // forward key rectangle rows
constexpr int kFChunk = 64;   // forward keys per tile

enum KeyKind : int { kLinear = 0, kRect = 1 };
enum KeyFlags : int { kNeedsMask = 0, kFull = 1 };

struct KeyTile {
  int kind;   // kLinear or kRect
  int a;      // kLinear: first token; kRect: first key row ky
  int b;      // kLinear: number of valid keys (1..128); kRect: first key column kx
  int flags;  // kFull or kNeedsMask
};

// Window shapes: the circle (CLEAR's mask, dx^2 + dy^2 < r^2), the square of the same radius
// (|dx| < r and |dy| < r), and the border-shifted square (the same square around a centre clamped
// to [r-1, n-r] per axis, so every query keeps (2r-1)^2 image keys; forward only). Everything
// downstream sees a window only through half_width / within, applied to window_center coordinates.
enum WindowShape : int { kCircle = 0, kSquare = 1, kShifted = 2 };

struct Geom {
  int B, heads, n_text, H, W, d, r;
  int window;        // WindowShape
  int T, BH;
  int nqy, nqx, nQ;  // image query tiles per (b, h): ceil(H/8) x ceil(W/16)
  int nTq;           // text query tiles: ceil(n_text / 128)
  int nTk;           // text key chunks: ceil(n_text / 128)
  int nC;            // linear key chunks over all T tokens: ceil(T / 128)
  int S;             // splits of a text query tile's key range
  int cps;           // chunks per split
  long long n_txt_items, n_img_items;
  // Forward pairs: two query tiles share every key tile they visit (a 16 x 16 image block, or
  // two consecutive 128-row text tiles); key tiles are 64 keys.
  int nqy2, nQ2;     // image blocks per (b, h): ceil((qy1 - qy0)/16) x ceil(W/16)
  int nTq2;          // text tile pairs: ceil(nTq / 2)
  int fnC;           // 64-key chunks a text query row visits (both key ranges below)
  int fnTk;          // 64-key chunks over the text tokens
  int fS, fcps;      // forward text splits and 64-key chunks per split
  int ftarget;       // chunks per forward text split aimed at (balance_forward_splits)
  long long n_txt_pairs, n_img_pairs;
  // Stripe mode (patch-parallel inference; the defaults are the whole problem): image query rows
  // are rows [qy0, qy1) of the grid only, and text query rows see the keys of token ranges
  // [ta_lo, ta_hi) and [tb_lo, tb_hi) (fnC = nca + ncb chunks of 64 keys, each range chunked from
  // its own start).
  int qy0, qy1;
  int ta_lo, ta_hi, tb_lo, tb_hi, nca;
  // Place in a packed batch (a mixed-resolution forward; the defaults are a problem of its own):
  // the item's tokens start at token t0 of rows that are tok_total tokens long, its text rows'
  // split partials start at partial row part_row0, and its text rows are rows
  // [crow0, crow0 + BH * n_text) of the batch's combine pass.
  int t0;
  long long tok_total, part_row0, crow0;
};

CLEAR_HD int cdiv(int a, int b) { return (a + b - 1) / b; }
CLEAR_HD int imin(int a, int b) { return a < b ? a : b; }
CLEAR_HD int imax(int a, int b) { return a > b ? a : b; }

// Largest w >= 0 with w*w < rem (rem >= 1); integer square root by correction of a float guess.
CLEAR_HD int isqrt_below(int rem) {
  int w = (int)sqrtf((float)(rem - 1));
  while (w > 0 && w * w > rem - 1) --w;
  while ((w + 1) * (w + 1) <= rem - 1) ++w;
  return w;
}

// Horizontal half-width of the window at vertical distance dy >= 0: the largest kept dx, or -1
// when no key at that vertical distance is kept. Circle: largest dx with dx^2 + dy^2 < r^2;
// square: r - 1 for dy < r.
CLEAR_HD int half_width(int r, int dy, int window = kCircle) {
  if (window != kCircle) return dy < r ? r - 1 : -1;
  int rem = r * r - dy * dy;
  return rem <= 0 ? -1 : isqrt_below(rem);
}

// Whether the offset (dx, dy), both >= 0, is inside the window.
CLEAR_HD bool within(int r, int window, int dx, int dy) {
  return window != kCircle ? (dx < r && dy < r) : (dx * dx + dy * dy < r * r);
}

// The grid coordinate (row or column, axis length n) the window is measured from: the query's own
// coordinate, or for the shifted window the centre clamped so the window stays inside the grid.
CLEAR_HD int window_center(int v, int r, int n, int window) {
  if (window != kShifted) return v;
  const int lo = r - 1, hi = n - r;
  return v < lo ? lo : (v > hi ? hi : v);
}

// Text split count: enough splits that each covers about `target` chunks, capped so the fp32
// partials stay small.
CLEAR_HD void choose_splits(int nC, int target, int max_splits, int* S, int* cps) {
  int s = cdiv(nC, target);
  if (s < 1) s = 1;
  if (s > max_splits) s = max_splits;
  int c = cdiv(nC, s);
  s = cdiv(nC, c);  // no empty split
  *S = s;
  *cps = c;
}

constexpr int kSplitTargetChunks = 64;
constexpr int kMaxSplits = 32;

// Text rows' key ranges: the text tokens (when text_keys) and image tokens [tk_lo, tk_hi); one range
// when they are adjacent.
CLEAR_HD void set_text_key_ranges(Geom* g, int text_keys, int tk_lo, int tk_hi) {
  if (text_keys && tk_lo == g->n_text) {
    g->ta_lo = 0; g->ta_hi = tk_hi; g->tb_lo = g->tb_hi = tk_hi;
  } else if (text_keys) {
    g->ta_lo = 0; g->ta_hi = g->n_text; g->tb_lo = tk_lo; g->tb_hi = tk_hi;
  } else {
    g->ta_lo = tk_lo; g->ta_hi = tk_hi; g->tb_lo = g->tb_hi = tk_hi;
  }
  g->nca = cdiv(g->ta_hi - g->ta_lo, kFChunk);
  g->fnC = g->nca + cdiv(g->tb_hi - g->tb_lo, kFChunk);
}

// Work counts that depend on the query rows and text-row key ranges (after set_text_key_ranges).
CLEAR_HD void set_forward_work(Geom* g, int qy0, int qy1) {
  g->qy0 = qy0;
  g->qy1 = qy1;
  g->nqy2 = cdiv(qy1 - qy0, 2 * kQH);
  g->nQ2 = g->nqy2 * g->nqx;
  g->ftarget = 2 * kSplitTargetChunks;
  choose_splits(g->fnC, g->ftarget, kMaxSplits, &g->fS, &g->fcps);
  g->n_txt_pairs = (long long)g->BH * g->nTq2 * g->fS;
  g->n_img_pairs = (long long)g->BH * g->nQ2;
}

CLEAR_HD void balance_forward_splits(Geom* g);

CLEAR_HD Geom make_geom(int B, int heads, int n_text, int H, int W, int d, int r, int window = kCircle) {
  Geom g;
  g.B = B; g.heads = heads; g.n_text = n_text; g.H = H; g.W = W; g.d = d; g.r = r;
  g.window = window;
  g.T = n_text + H * W;
  g.BH = B * heads;
  g.nqy = cdiv(H, kQH);
  g.nqx = cdiv(W, kQW);
  g.nQ = g.nqy * g.nqx;
  g.nTq = cdiv(n_text, kTile);
  g.nTk = cdiv(n_text, kTile);
  g.nC = cdiv(g.T, kTile);
  choose_splits(g.nC, kSplitTargetChunks, kMaxSplits, &g.S, &g.cps);
  g.n_txt_items = (long long)g.BH * g.nTq * g.S;
  g.n_img_items = (long long)g.BH * g.nQ;
  g.nTq2 = cdiv(g.nTq, 2);
  g.fnTk = cdiv(n_text, kFChunk);
  set_text_key_ranges(&g, 1, n_text, g.T);
  set_forward_work(&g, 0, H);
  balance_forward_splits(&g);
  g.t0 = 0;
  g.tok_total = g.T;
  g.part_row0 = 0;
  g.crow0 = 0;
  return g;
}

// One unit of forward work: a query tile of one (batch, head) and its key range.
struct WorkItem {
  int is_text;  // 1: text query tile (split partial), 0: image query tile
  int bh;
  int q0;       // text: first query token; image: query tile row y0
  int x0;       // image: query tile column x0
  int split;    // text: split index
  int c_begin, c_end;  // text: linear chunk range [c_begin, c_end)
};

// Text items come first (they are the longest), then image items.
CLEAR_HD WorkItem decode_work(const Geom& g, long long w) {
  WorkItem it;
  if (w < g.n_txt_items) {
    int s = (int)(w % g.S);
    long long t = w / g.S;
    int qt = (int)(t % g.nTq);
    it.is_text = 1;
    it.bh = (int)(t / g.nTq);
    it.q0 = qt * kTile;
    it.x0 = 0;
    it.split = s;
    it.c_begin = s * g.cps;
    it.c_end = imin(g.nC, (s + 1) * g.cps);
  } else {
    long long u = w - g.n_txt_items;
    int tile = (int)(u % g.nQ);
    it.is_text = 0;
    it.bh = (int)(u / g.nQ);
    it.q0 = (tile / g.nqx) * kQH;
    it.x0 = (tile % g.nqx) * kQW;
    it.split = 0;
    it.c_begin = 0;
    it.c_end = 0;
  }
  return it;
}

// Enumerates the key tiles of one work item, in visiting order.
struct KeyIter {
  // fixed per item
  const int* wtab;        // optional half-width table (device shared memory), entries [0, wtab_n)
  int wtab_n;
  int is_text, r, window, H, W, n_text, T;
  int y0, yl, x0, xl;     // image query tile, clipped to the grid (rows y0..yl, cols x0..xl)
  int ky_begin, ky_end;   // key rows that any query of the tile can reach
  // state
  int lin_next, lin_end;  // remaining linear chunks [lin_next, lin_end)
  int band_ky;            // current band's first key row
  int kx, kx_end;         // next rectangle column and the band's last needed column

  CLEAR_HD void init(const Geom& g, const WorkItem& it, const int* table = nullptr, int table_n = 0) {
    wtab = table;
    wtab_n = table_n;
    is_text = it.is_text; r = g.r; window = g.window; H = g.H; W = g.W; n_text = g.n_text; T = g.T;
    if (is_text) {
      lin_next = it.c_begin;
      lin_end = it.c_end;
      band_ky = 1; ky_end = 0;  // no bands
      kx = 1; kx_end = 0;
      y0 = yl = x0 = xl = 0; ky_begin = 0;
      return;
    }
    lin_next = 0;
    lin_end = g.nTk;
    y0 = it.q0; x0 = it.x0;
    yl = imin(y0 + kQH - 1, H - 1);
    xl = imin(x0 + kQW - 1, W - 1);
    ky_begin = imax(0, y0 - (r - 1));
    ky_end = imin(H - 1, yl + (r - 1));
    band_ky = ky_begin - kKH;  // first advance lands on ky_begin
    kx = 1; kx_end = 0;        // empty band: forces an advance
  }

  // Moves to the next band with at least one needed column; false when none is left.
  CLEAR_HD bool advance_band() {
    while (true) {
      band_ky += kKH;
      if (band_ky > ky_end) return false;
      int band_last = imin(band_ky + kKH - 1, H - 1);
      int dmin = imax(0, imax(y0 - band_last, band_ky - yl));
      int w = (dmin < wtab_n) ? wtab[dmin] : half_width(r, dmin, window);
      if (w < 0) continue;
      kx = imax(0, x0 - w);
      kx_end = imin(W - 1, xl + w);
      if (kx <= kx_end) return true;
    }
  }

  CLEAR_HD bool next(KeyTile* t) {
    if (lin_next < lin_end) {
      int a = lin_next * kTile;
      int lim = is_text ? T : n_text;
      t->kind = kLinear;
      t->a = a;
      t->b = imin(kTile, lim - a);
      t->flags = (t->b == kTile) ? kFull : kNeedsMask;
      ++lin_next;
      return true;
    }
    if (is_text) return false;
    if (kx > kx_end) {
      if (!advance_band()) return false;
    }
    t->kind = kRect;
    t->a = band_ky;
    t->b = kx;
    // Full when the rectangle is inside the grid and its farthest pair is within radius.
    bool inside = (band_ky + kKH - 1 <= H - 1) && (kx + kKW - 1 <= W - 1);
    int mdy = imax(band_ky + kKH - 1 - y0, yl - band_ky);
    int mdx = imax(kx + kKW - 1 - x0, xl - kx);
    t->flags = (inside && within(r, window, mdx, mdy)) ? kFull : kNeedsMask;
    kx += kKW;
    return true;
  }
};

// Number of key tiles an item visits (host-side cost estimates and tests).
CLEAR_HD int count_key_tiles(const Geom& g, const WorkItem& it, const int* table = nullptr, int table_n = 0) {
  KeyIter ki;
  ki.init(g, it, table, table_n);
  KeyTile t;
  int n = 0;
  while (ki.next(&t)) ++n;
  return n;
}

// ------------------------------------------------------------------------------------------------
// Pair work items for the forward: half A and half B of a pair share the key tiles.
// ------------------------------------------------------------------------------------------------
enum PairFlags : int { kNeedA = 1, kNeedB = 2, kFullA = 4, kFullB = 8 };

struct PairItem {
  int is_text;
  int bh;
  int q0;        // text: first token of half A (half B starts 128 later); image: block row y0
  int x0;        // image: block column x0
  int validB;    // half B holds at least one real query row
  int split, c_begin, c_end;  // text: split index and linear chunk range
};

CLEAR_HD PairItem decode_pair(const Geom& g, long long w) {
  PairItem it;
  if (w < g.n_txt_pairs) {
    int s = (int)(w % g.fS);
    long long t = w / g.fS;
    int qp = (int)(t % g.nTq2);
    it.is_text = 1;
    it.bh = (int)(t / g.nTq2);
    it.q0 = qp * 2 * kTile;
    it.x0 = 0;
    it.validB = (it.q0 + kTile) < g.n_text;
    it.split = s;
    it.c_begin = s * g.fcps;
    it.c_end = imin(g.fnC, (s + 1) * g.fcps);
  } else {
    long long u = w - g.n_txt_pairs;
    int blk = (int)(u % g.nQ2);
    it.is_text = 0;
    it.bh = (int)(u / g.nQ2);
    it.q0 = g.qy0 + (blk / g.nqx) * (2 * kQH);
    it.x0 = (blk % g.nqx) * kQW;
    it.validB = (it.q0 + kQH) < g.qy1;
    it.split = 0;
    it.c_begin = 0;
    it.c_end = 0;
  }
  return it;
}

// Union key tiles of a pair (64 keys each), with per-half need / full flags. Image blocks visit the
// 64-token text chunks, then band by band (4 key rows) the 16-column rectangles covering the union
// of both halves' windows; a tile is needed by a half iff some (query of that half, key of the
// tile) pair is kept.
struct PairKeyIter {
  const int* wtab;
  int wtab_n;
  int is_text, r, window, H, W, n_text, T, validB;
  int ta_lo, ta_hi, tb_lo, tb_hi, nca;  // text rows' key ranges (chunk i < nca: range a)
  int y0, x0, xl;             // block origin, last column
  int yA0, yAl, yB0, yBl;     // half rows (clipped); B rows only if validB
  int ky_begin, ky_end;
  int lin_next, lin_end;
  int band_ky, kx, kx_end;
  int band_step, n_bands;     // bands are visited ends-inward: 0, n-1, 1, n-2, ...

  CLEAR_HD void init(const Geom& g, const PairItem& it, const int* table = nullptr, int table_n = 0) {
    wtab = table;
    wtab_n = table_n;
    is_text = it.is_text; r = g.r; window = g.window; H = g.H; W = g.W; n_text = g.n_text; T = g.T;
    validB = it.validB;
    ta_lo = g.ta_lo; ta_hi = g.ta_hi; tb_lo = g.tb_lo; tb_hi = g.tb_hi; nca = g.nca;
    if (is_text) {
      lin_next = it.c_begin;
      lin_end = it.c_end;
      band_ky = 1; ky_end = 0; kx = 1; kx_end = 0;
      y0 = x0 = xl = yA0 = yAl = yB0 = yBl = 0; ky_begin = 0;
      band_step = n_bands = 0;
      return;
    }
    lin_next = 0;
    lin_end = g.fnTk;
    y0 = it.q0; x0 = it.x0;
    xl = imin(x0 + kQW - 1, W - 1);
    yA0 = y0; yAl = imin(y0 + kQH - 1, g.qy1 - 1);
    yB0 = y0 + kQH; yBl = imin(y0 + 2 * kQH - 1, g.qy1 - 1);
    if (window == kShifted) {  // clamping is monotone: a query rectangle maps to a centre rectangle
      x0 = window_center(x0, r, W, window); xl = window_center(xl, r, W, window);
      yA0 = window_center(yA0, r, H, window); yAl = window_center(yAl, r, H, window);
      yB0 = window_center(yB0, r, H, window); yBl = window_center(yBl, r, H, window);
      y0 = yA0;
    }
    const int ylast = validB ? yBl : yAl;
    ky_begin = imax(0, y0 - (r - 1));
    ky_end = imin(H - 1, ylast + (r - 1));
    n_bands = (ky_end - ky_begin) / kFKH + 1;
    band_step = 0;
    band_ky = ky_begin;
    kx = 1; kx_end = 0;
  }

  CLEAR_HD int hw(int dy) const { return (dy < wtab_n) ? wtab[dy] : half_width(r, dy, window); }

  // Next band with kept columns. The first and last bands are reached by one half only (the
  // top ones by half A, the bottom ones by half B); alternating from both ends keeps both halves
  // busy instead of leaving one idle at the start of the pair and the other at its end.
  CLEAR_HD bool advance_band() {
    const int ylast = validB ? yBl : yAl;
    while (true) {
      if (band_step >= n_bands) return false;
      const int k = (band_step & 1) ? n_bands - 1 - (band_step >> 1) : (band_step >> 1);
      ++band_step;
      band_ky = ky_begin + k * kFKH;
      const int band_last = imin(band_ky + kFKH - 1, H - 1);
      const int dmin = imax(0, imax(y0 - band_last, band_ky - ylast));
      const int w = hw(dmin);
      if (w < 0) continue;
      kx = imax(0, x0 - w);
      kx_end = imin(W - 1, xl + w);
      if (kx <= kx_end) return true;
    }
  }

  // need / full of rectangle [ky, ky+4) x [kx, kx+16) for query rows [qa, qb], columns [x0, xl].
  CLEAR_HD int half_flags(int ky, int kxx, int qa, int qb, int need_bit, int full_bit) const {
    const int kyl = imin(ky + kFKH - 1, H - 1);
    const int kxl = imin(kxx + kKW - 1, W - 1);
    const int dy = imax(0, imax(qa - kyl, ky - qb));
    const int dx = imax(0, imax(x0 - kxl, kxx - xl));
    if (!within(r, window, dx, dy)) return 0;
    const bool inside = (ky + kFKH - 1 <= H - 1) && (kxx + kKW - 1 <= W - 1);
    const int mdy = imax(ky + kFKH - 1 - qa, qb - ky);
    const int mdx = imax(kxx + kKW - 1 - x0, xl - kxx);
    return need_bit | ((inside && within(r, window, mdx, mdy)) ? full_bit : 0);
  }

  CLEAR_HD bool next(KeyTile* t) {
    if (lin_next < lin_end) {
      // Image blocks: the text keys from token 0. Text rows: chunk i of range a, or of range b.
      int a = lin_next * kFChunk, lim = n_text;
      if (is_text) {
        const bool in_a = lin_next < nca;
        a = in_a ? ta_lo + lin_next * kFChunk : tb_lo + (lin_next - nca) * kFChunk;
        lim = in_a ? ta_hi : tb_hi;
      }
      t->kind = kLinear;
      t->a = a;
      t->b = imin(kFChunk, lim - a);
      const int full = (t->b == kFChunk);
      t->flags = kNeedA | (full ? kFullA : 0) | (validB ? (kNeedB | (full ? kFullB : 0)) : 0);
      ++lin_next;
      return true;
    }
    if (is_text) return false;
    while (true) {
      if (kx > kx_end) {
        if (!advance_band()) return false;
      }
      const int f = half_flags(band_ky, kx, yA0, yAl, kNeedA, kFullA) |
                    (validB ? half_flags(band_ky, kx, yB0, yBl, kNeedB, kFullB) : 0);
      t->kind = kRect;
      t->a = band_ky;
      t->b = kx;
      t->flags = f;
      kx += kKW;
      if (f & (kNeedA | kNeedB)) return true;  // rectangles neither half reaches are skipped
    }
  }
};

// Needed tiles of one half (half = 0: A, 1: B) in a pair, and the union tile count.
CLEAR_HD void count_pair_tiles(const Geom& g, const PairItem& it, const int* table, int table_n, int* n_union,
                               int* n_a, int* n_b) {
  PairKeyIter ki;
  ki.init(g, it, table, table_n);
  KeyTile t;
  int nu = 0, na = 0, nb = 0;
  while (ki.next(&t)) {
    ++nu;
    na += (t.flags & kNeedA) ? 1 : 0;
    nb += (t.flags & kNeedB) ? 1 : 0;
  }
  *n_union = nu;
  *n_a = na;
  *n_b = nb;
}

// Text split count of the forward, chosen with a model of the static round-robin assignment
// (pair item w runs on CTA w mod kFwdModelSMs, one CTA per SM): an item costs the (key tile,
// half) products it issues plus a fixed cost per item (kFwdTextItemCost, kFwdImageItemCost; fitted
// to timings of split counts 1 to 7 on FLUX-shaped 64 x 64 and 128 x 128 grids, where the model
// then picks the measured best each time), and the split count with the smallest busiest CTA wins
// (the smaller count on ties). Candidates run from the plain rule (splits of at most
// 2 * kSplitTargetChunks chunks) up to 8 splits, never above kMaxSplits. With more than 64 image
// pairs per SM the plain rule is kept: the items are then many and small enough to balance.
constexpr int kFwdModelSMs = 148;
constexpr int kFwdTextItemCost = 16;
constexpr int kFwdImageItemCost = 24;

CLEAR_HD long long forward_makespan(const Geom& g, int S, const int* img_cost, int n_img_cost) {
  const int cps = cdiv(g.fnC, S);
  S = cdiv(g.fnC, cps);
  const long long n = (long long)g.BH * (g.nTq2 * S + n_img_cost);
  const int G = n < kFwdModelSMs ? (int)n : kFwdModelSMs;
  long long load[kFwdModelSMs] = {};
  int bin = 0;
  for (int pr = 0; pr < g.BH * g.nTq2; ++pr)  // text pairs, then their splits, as decode_pair orders them
    for (int sp = 0; sp < S; ++sp) {
      load[bin] += 2 * (imin(g.fnC, (sp + 1) * cps) - sp * cps) + kFwdTextItemCost;
      if (++bin == G) bin = 0;
    }
  for (int bh = 0; bh < g.BH; ++bh)
    for (int i = 0; i < n_img_cost; ++i) {
      load[bin] += img_cost[i] + kFwdImageItemCost;
      if (++bin == G) bin = 0;
    }
  long long mx = 0;
  for (int i = 0; i < G; ++i) mx = load[i] > mx ? load[i] : mx;
  return mx;
}

constexpr int kMaxModelPairs = 64 * kFwdModelSMs;

// (key tile, half) products of each image pair of head 0, g.nQ2 entries; every head has the same.
CLEAR_HD void image_pair_costs(const Geom& g, int* cost) {
  for (int blk = 0; blk < g.nQ2; ++blk) {
    const PairItem it = decode_pair(g, g.n_txt_pairs + blk);
    PairKeyIter ki;
    ki.init(g, it, nullptr, 0);
    KeyTile t;
    int c = 0;
    while (ki.next(&t)) c += ((t.flags & kNeedA) ? 1 : 0) + ((t.flags & kNeedB) ? 1 : 0);
    cost[blk] = c;
  }
}

// The plain rule: splits of at most 2 * kSplitTargetChunks chunks.
CLEAR_HD void plain_forward_splits(Geom* g) {
  g->ftarget = 2 * kSplitTargetChunks;
  choose_splits(g->fnC, g->ftarget, kMaxSplits, &g->fS, &g->fcps);
  g->n_txt_pairs = (long long)g->BH * g->nTq2 * g->fS;
}

CLEAR_HD void balance_forward_splits(Geom* g) {
  plain_forward_splits(g);
  if (g->n_text == 0 || g->nQ2 == 0 || (long long)g->BH * g->nQ2 > kMaxModelPairs || g->fS >= 8) return;
#ifndef __CUDA_ARCH__
  static thread_local int cost[kMaxModelPairs];
  image_pair_costs(*g, cost);
  int best_s = g->fS;
  long long best = forward_makespan(*g, g->fS, cost, g->nQ2);
  for (int s = g->fS + 1; s <= imin(8, kMaxSplits); ++s) {
    const long long m = forward_makespan(*g, s, cost, g->nQ2);
    if (m < best) { best = m; best_s = s; }
  }
  g->ftarget = cdiv(g->fnC, best_s);
  choose_splits(g->fnC, g->ftarget, kMaxSplits, &g->fS, &g->fcps);
  g->n_txt_pairs = (long long)g->BH * g->nTq2 * g->fS;
#endif
}

}  // namespace clear
