// Device helpers shared by the forward and backward kernels: tile loads, the circular-window row
// ranges used for masking, and the 1024-byte alignment of the dynamic shared-memory base.
#pragma once
#include <cuda_bf16.h>

#include "clear_sched.cuh"
#include "sm100_ptx.cuh"

namespace clear {

constexpr int kMaxRTable = 256;   // radius up to which the half-width table lives in smem
constexpr int kHalfBytes = kTile * 128;  // one 128-row x 64-element bf16 block (128B-swizzled)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Loads one 128-row tile (all 64-element column blocks) of q/k/v/dO: a linear chunk of 128 tokens
// (kind kLinear, first token a) or an 8 x 16 grid rectangle (kind kRect, rows from a, columns
// from b) of head bh.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* lin, const CUtensorMap* img,
                                          uint64_t* bar, int kind, int a, int b, int bh) {
  #pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    uint8_t* d = dst + h * kHalfBytes;
    if (kind == kLinear)
      tma_load_3d(d, lin, bar, h * 64, a, bh);
    else
      tma_load_4d(d, img, bar, h * 64, b, a, bh);
  }
}

// Half-width for |dy| beyond the shared-memory table (only for radii above kMaxRTable).
__device__ __noinline__ int half_width_slow(int r, int dy, int window) { return half_width(r, dy, window); }

// Kept column range [lo, hi] (tile-local, 0..15) of key row ky of a rectangle tile starting at
// column kx, seen from grid point (yq, xq): keys inside the grid with dx^2 + dy^2 < r^2. An empty
// range is returned as lo = 16, hi = -1, so that (unsigned)(c - lo) <= (unsigned)(hi - lo) is
// exactly "lo <= c <= hi" for every c in 0..15.
__device__ __forceinline__ void rect_row_range(const Geom& g, const int* wtab, int yq, int xq, int ky, int kx,
                                               int* lo_out, int* hi_out) {
  const int dy = ky - yq;
  const int ady = dy < 0 ? -dy : dy;
  int w = (ady < kMaxRTable) ? wtab[ady] : half_width_slow(g.r, ady, g.window);
  if ((unsigned)ky >= (unsigned)g.H) w = -1;
  int lo = imax(imax(xq - w, 0) - kx, 0);
  int hi = imin(imin(xq + w, g.W - 1) - kx, kKW - 1);
  if (w < 0 || lo > hi) { lo = kKW; hi = -1; }
  *lo_out = lo;
  *hi_out = hi;
}

// Largest |dy| the full half-width table needs: a query and a key row of the grid are at most
// H - 1 apart, and no row at |dy| >= r is kept, so min(r, H) entries cover every lookup.
constexpr int kMaxHwTable = 16384;
__host__ __device__ inline int hw_table_size(int r, int H) { return r < H ? r : H; }

// Branch-free kept range of one key row from the full half-width table (int16 entries, exactly
// hw_table_size(r, H) of them): same contract as rect_row_range.
__device__ __forceinline__ void row_range_tab(const Geom& g, const int16_t* tab, int tabn, int yq, int xq, int ky,
                                              int kx, int* lo_out, int* hi_out) {
  const int dy = ky - yq;
  const int ady = dy < 0 ? -dy : dy;
  int w = tab[ady < tabn ? ady : tabn - 1];
  w = (ady < tabn && (unsigned)ky < (unsigned)g.H) ? w : -1;
  int lo = imax(imax(xq - w, 0) - kx, 0);
  int hi = imin(imin(xq + w, g.W - 1) - kx, kKW - 1);
  const bool empty = (w < 0) | (lo > hi);
  *lo_out = empty ? kKW : lo;
  *hi_out = empty ? -1 : hi;
}

}  // namespace clear
