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

enum KeyKind : int { kLinear = 0, kRect = 1 };
enum KeyFlags : int { kNeedsMask = 0, kFull = 1 };

struct KeyTile {
  int kind;   // kLinear or kRect
  int a;      // kLinear: first token; kRect: first key row ky
  int b;      // kLinear: number of valid keys (1..128); kRect: first key column kx
  int flags;  // kFull or kNeedsMask
};

struct Geom {
  int B, heads, n_text, H, W, d, r;
  int T, BH;
  int nqy, nqx, nQ;  // image query tiles per (b, h): ceil(H/8) x ceil(W/16)
  int nTq;           // text query tiles: ceil(n_text / 128)
  int nTk;           // text key chunks: ceil(n_text / 128)
  int nC;            // linear key chunks over all T tokens: ceil(T / 128)
  int S;             // splits of a text query tile's key range
  int cps;           // chunks per split
  long long n_txt_items, n_img_items;
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

// Horizontal half-width of the window at vertical distance dy: largest dx with dx^2 + dy^2 < r^2,
// or -1 when no key at that vertical distance is within radius.
CLEAR_HD int half_width(int r, int dy) {
  int rem = r * r - dy * dy;
  return rem <= 0 ? -1 : isqrt_below(rem);
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

CLEAR_HD Geom make_geom(int B, int heads, int n_text, int H, int W, int d, int r) {
  Geom g;
  g.B = B; g.heads = heads; g.n_text = n_text; g.H = H; g.W = W; g.d = d; g.r = r;
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
  int is_text, r, H, W, n_text, T;
  int y0, yl, x0, xl;     // image query tile, clipped to the grid (rows y0..yl, cols x0..xl)
  int ky_begin, ky_end;   // key rows that any query of the tile can reach
  // state
  int lin_next, lin_end;  // remaining linear chunks [lin_next, lin_end)
  int band_ky;            // current band's first key row
  int kx, kx_end;         // next rectangle column and the band's last needed column

  CLEAR_HD void init(const Geom& g, const WorkItem& it) {
    is_text = it.is_text; r = g.r; H = g.H; W = g.W; n_text = g.n_text; T = g.T;
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
      int w = half_width(r, dmin);
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
    t->flags = (inside && mdy * mdy + mdx * mdx < r * r) ? kFull : kNeedsMask;
    kx += kKW;
    return true;
  }
};

// Number of key tiles an item visits (host-side cost estimates and tests).
CLEAR_HD int count_key_tiles(const Geom& g, const WorkItem& it) {
  KeyIter ki;
  ki.init(g, it);
  KeyTile t;
  int n = 0;
  while (ki.next(&t)) ++n;
  return n;
}

}  // namespace clear
