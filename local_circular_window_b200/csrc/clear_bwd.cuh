// CLEAR attention backward on sm_100a (tcgen05 + TMA), matching clear_fwd.cuh.
//
// The pages give no backward formula; CLEAR only fine-tunes the attention layers by gradient
// descent (pith.science review of "CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion
// Transformers Up", "The reading"), so this is the analytic gradient of the masked softmax
// attention forward:
//   P = softmax_M(scale * Q K^T), D_i = rowsum(dO_i o O_i), dP = dO V^T, dS = P o (dP - D),
//   dV = P^T dO,  dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Kernels (all deterministic, no floating-point atomics):
//   preprocess  D and LSE * log2(e) per row                             (CUDA cores, HBM-bound)
//   dq kernel   Q-stationary: per query tile, visit its 128-key tiles; S, dP -> TMEM,
//               dS -> smem (bf16), dQ += dS K in TMEM. One thread issues S and dP (the next key
//               tile's while the softmax works on this one), another the dQ products; V's ring
//               slot is released after dP, K's after dQ. Text query tiles are split over key
//               chunks into fp32 partials.
//   dkdv kernel KV-stationary: per key tile, visit the query tiles that keep it. The mask is
//               symmetric, so the same tile enumeration with the roles of query and key swapped
//               gives exactly those tiles. S^T, dP^T -> TMEM, per half of 64 partner queries;
//               P^T, dS^T written back over them (bf16); dV += P^T dO, dK += dS^T Q in TMEM with
//               the A operand read from TMEM, so one half's products overlap the other half's
//               softmax; partner Q / dO double-buffered. Text key tiles are split over query
//               chunks into fp32 partials.
// Both kernels split each tile's 128 columns over two softmax warpgroups (64 each); in dkdv they
// never wait for each other, in dq both arrive on the barriers that hand S / dP back and dS on.
//   reduce      sums the split partials of the text rows in a fixed order and writes bf16.
#pragma once
#include <cuda_bf16.h>

#include "clear_common.cuh"
#include "clear_sched.cuh"
#include "sm100_ptx.cuh"

namespace clear {

struct BwdWorkspace {
  size_t dvec_off, l2vec_off, dq_off, dk_off, dv_off, total;
};

inline size_t bwd_align256(size_t x) { return (x + 255) & ~size_t(255); }

inline BwdWorkspace bwd_workspace_layout(const Geom& g) {
  BwdWorkspace w{};
  const size_t rows = (size_t)g.BH * g.T;
  const size_t part = (size_t)g.S * g.BH * g.n_text * g.d * sizeof(float);
  w.dvec_off = 0;
  w.l2vec_off = bwd_align256(w.dvec_off + rows * sizeof(float));
  w.dq_off = bwd_align256(w.l2vec_off + rows * sizeof(float));
  w.dk_off = bwd_align256(w.dq_off + part);
  w.dv_off = bwd_align256(w.dk_off + part);
  w.total = bwd_align256(w.dv_off + part);
  return w;
}

struct BwdArgs {
  Geom g;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dO;
  const float* lse;
  __nv_bfloat16 *dq, *dk, *dv;
  char* ws;
  BwdWorkspace wl;
};

struct BwdParams {
  Geom g;
  float scale;         // 1/sqrt(d)
  float scale_log2;    // scale * log2(e)
  const float* dvec;   // [BH, T] rowsum(dO o O)
  const float* l2vec;  // [BH, T] lse * log2(e)
  __nv_bfloat16* out_a;  // dq (dq kernel) or dk (dkdv kernel)
  __nv_bfloat16* out_b;  // dv (dkdv kernel)
  float* part_a;         // [S, BH, n_text, d] split partials (dq, or dk)
  float* part_b;         // [S, BH, n_text, d] split partials (dv)
  long long n_work;
};

// 16-bit keep-mask of one row of a rectangle tile: columns [kx, kx + 16) of grid row ky, seen from
// grid point (yp, xp): bit c set iff (ky, kx + c) is inside the grid and within radius.
__device__ __forceinline__ uint32_t rect_row_bits(const Geom& g, const int* wtab, int yp, int xp, int ky,
                                                  int kx) {
  if (ky < 0 || ky >= g.H) return 0u;
  const int dy = ky - yp;
  const int ady = dy < 0 ? -dy : dy;
  if (ady >= g.r) return 0u;
  const int wdt = (ady < kMaxRTable) ? wtab[ady] : half_width(g.r, ady, g.window);
  if (wdt < 0) return 0u;
  int lo = imax(xp - wdt, 0) - kx;
  int hi = imin(xp + wdt, g.W - 1) - kx;
  lo = imax(lo, 0);
  hi = imin(hi, kKW - 1);
  if (lo > hi) return 0u;
  return ((2u << hi) - 1u) & ~((1u << lo) - 1u);
}

// Writes 128 bf16 values of one row into a 128 x 128 K-major, 128B-swizzled operand block
// (two 128 x 64 halves), the layout the tcgen05 A-operand descriptors expect.
__device__ __forceinline__ void store_row_sw128(uint32_t base, int row, const float* x) {
  #pragma unroll
  for (int ch = 0; ch < kTile / 8; ++ch) {
    const uint32_t addr = base + (ch >> 3) * (kTile * 128) + row * 128 +
                          ((((uint32_t)ch & 7u) ^ ((uint32_t)row & 7u)) << 4);
    st_shared_v4(addr, pack_bf16x2(x[ch * 8 + 0], x[ch * 8 + 1]), pack_bf16x2(x[ch * 8 + 2], x[ch * 8 + 3]),
                 pack_bf16x2(x[ch * 8 + 4], x[ch * 8 + 5]), pack_bf16x2(x[ch * 8 + 6], x[ch * 8 + 7]));
  }
}

// Writes 32 bf16 values (columns [32*ch, 32*ch + 32)) of one row into a 128 x 128 K-major,
// 128B-swizzled operand block.
__device__ __forceinline__ void store_chunk32_sw128(uint32_t base, int row, int ch, const float* x) {
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c8 = ch * 4 + q;  // 8-column chunk index 0..15
    const uint32_t addr = base + (c8 >> 3) * (kTile * 128) + row * 128 +
                          ((((uint32_t)c8 & 7u) ^ ((uint32_t)row & 7u)) << 4);
    st_shared_v4(addr, pack_bf16x2(x[q * 8 + 0], x[q * 8 + 1]), pack_bf16x2(x[q * 8 + 2], x[q * 8 + 3]),
                 pack_bf16x2(x[q * 8 + 4], x[q * 8 + 5]), pack_bf16x2(x[q * 8 + 6], x[q * 8 + 7]));
  }
}

__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* s) {
  uint32_t sr[4][32];
  tmem_ld32(taddr + 0, sr[0]);
  tmem_ld32(taddr + 32, sr[1]);
  tmem_ld32(taddr + 64, sr[2]);
  tmem_ld32(taddr + 96, sr[3]);
  tmem_wait_ld();
  #pragma unroll
  for (int c = 0; c < kTile; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Issues the K-dim loop of one 128 x N x D tile product with both operands K-major in smem.
template <int D>
__device__ __forceinline__ void mma_kmajor(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr, uint32_t idesc) {
  #pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * (kTile * 128) + (kk & 3) * 32;
    umma_ss(d_tmem, smem_desc_sw128(a_addr + off, 16, 1024), smem_desc_sw128(b_addr + off, 16, 1024), idesc,
            kk > 0);
  }
}

// Issues a 128 x D x 128 product: A (128 x 128, K-major, smem) times B (128 rows of D, MN-major).
template <int D>
__device__ __forceinline__ void mma_a_kmajor_b_mnmajor(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr,
                                                       uint32_t idesc, bool accumulate) {
  #pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk) {
    const uint32_t a_off = (kk >> 2) * (kTile * 128) + (kk & 3) * 32;
    umma_ss(d_tmem, smem_desc_sw128(a_addr + a_off, 16, 1024), smem_desc_sw128(b_addr + kk * 2048, kTile * 128, 1024),
            idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// ------------------------------------------------------------------------------------------------
// Preprocess: D = rowsum(dO o O), L2 = lse * log2(e). One warp per row.
// ------------------------------------------------------------------------------------------------
template <int D>
__global__ void clear_bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                                            const float* __restrict__ lse, float* __restrict__ dvec,
                                            float* __restrict__ l2vec, long long rows) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int kPer = D / 32;
  const __nv_bfloat16* a = o + row * D + lane * kPer;
  const __nv_bfloat16* b = dO + row * D + lane * kPer;
  float acc = 0.f;
  #pragma unroll
  for (int e = 0; e < kPer; ++e) acc += __bfloat162float(a[e]) * __bfloat162float(b[e]);
  #pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    dvec[row] = acc;
    l2vec[row] = lse[row] * 1.4426950408889634f;
  }
}

// ------------------------------------------------------------------------------------------------
// Reduce split partials of text rows: out[bh, t] = bf16(scale * sum_s part[s, bh, t]).
// ------------------------------------------------------------------------------------------------
template <int D>
__global__ void clear_bwd_reduce_kernel(const float* __restrict__ part, __nv_bfloat16* __restrict__ out, Geom g,
                                        float scale) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (long long)g.BH * g.n_text) return;
  const int bh = (int)(row / g.n_text);
  const int t = (int)(row % g.n_text);
  constexpr int kPer = D / 32;
  float acc[kPer];
  #pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  for (int s = 0; s < g.S; ++s) {
    const float* src = part + (((size_t)s * g.BH + bh) * g.n_text + t) * D + lane * kPer;
    #pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] += src[e];
  }
  __nv_bfloat16* dst = out + ((size_t)bh * g.T + t) * D + lane * kPer;
  #pragma unroll
  for (int e = 0; e < kPer; ++e) dst[e] = __float2bfloat16_rn(acc[e] * scale);
}

// ------------------------------------------------------------------------------------------------
// dQ kernel (Q-stationary)
// ------------------------------------------------------------------------------------------------
// 3 warpgroups: two softmax warpgroups (each owns 64 of the 128 key or query columns of a tile),
// then the TMA producer (warp 8), the MMA issuer / TMEM owner (warp 9) and two idle warps.
constexpr int kBwdThreads = 384;
// Launched at 168 registers per thread; the producer / MMA warpgroup drops to kBwdRegsLow and the
// softmax warpgroups grow to kBwdRegsHigh.
constexpr uint32_t kBwdRegsLow = 120;
constexpr uint32_t kBwdRegsHigh = 192;
static_assert(2 * 128 * kBwdRegsHigh + 128 * kBwdRegsLow <= 384 * 168, "register split exceeds the launch allocation");

template <int D, int NST>
struct DqLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTileBytes;
  static constexpr int kK = kDO + kTileBytes;
  static constexpr int kV = kK + NST * kTileBytes;
  static constexpr int kDS = kV + NST * kTileBytes;
  static constexpr int kBars = kDS + kTile * kTile * 2;
  static constexpr int bQFull = 0, bQEmpty = 1, bSdpFull = 2, bSdpFree = 3, bDsFull = 4, bDsEmpty = 5,
                       bAccDone = 6;
  // K and V ring slots are released separately: V after dP (its only reader), K after dQ.
  static constexpr int bKFull = 7, bVFull = bKFull + NST, bKEmpty = bVFull + NST, bVEmpty = bKEmpty + NST;
  static constexpr int kNumBars = bVEmpty + NST;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kWTab = kMisc + 16;
  static constexpr int kTotal = kWTab + kMaxRTable * 4;
  static constexpr int kAlloc = kTotal + 1024;
  static constexpr uint32_t kTmemS = 0, kTmemDP = 128, kTmemAcc = 256, kTmemCols = 512;
};

template <int D, int NST>
__global__ void __launch_bounds__(kBwdThreads, 1)
clear_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q_lin, const __grid_constant__ CUtensorMap tm_q_img,
                    const __grid_constant__ CUtensorMap tm_do_lin, const __grid_constant__ CUtensorMap tm_do_img,
                    const __grid_constant__ CUtensorMap tm_k_lin, const __grid_constant__ CUtensorMap tm_k_img,
                    const __grid_constant__ CUtensorMap tm_v_lin, const __grid_constant__ CUtensorMap tm_v_img,
                    const BwdParams p) {
  using L = DqLayout<D, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int* wtab = reinterpret_cast<int*>(smem + L::kWTab);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::bQFull], 1);
    mbar_init(&bars[L::bQEmpty], 1);
    mbar_init(&bars[L::bSdpFull], 1);
    mbar_init(&bars[L::bSdpFree], 256);
    mbar_init(&bars[L::bDsFull], 256);
    mbar_init(&bars[L::bDsEmpty], 1);
    mbar_init(&bars[L::bAccDone], 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars[L::bKFull + s], 1);
      mbar_init(&bars[L::bVFull + s], 1);
      mbar_init(&bars[L::bKEmpty + s], 1);
      mbar_init(&bars[L::bVEmpty + s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kMaxRTable; i += blockDim.x) wtab[i] = half_width(g.r, i, g.window);
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    regs_dec<kBwdRegsLow>();
    if (lane == 0) {
      int stage = 0;
      uint32_t ring_ph = 0, q_empty_ph = 0;
      bool first = true;
      for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
        const WorkItem it = decode_work(g, w);
        if (!first) {
          if (!mbar_wait(&bars[L::bQEmpty], q_empty_ph, abort_flag, kDevTimeoutTmaEmpty)) goto producer_done;
          q_empty_ph ^= 1;
        }
        first = false;
        mbar_arrive_expect_tx(&bars[L::bQFull], 2 * L::kTileBytes);
        load_tile<D>(smem + L::kQ, &tm_q_lin, &tm_q_img, &bars[L::bQFull], it.is_text ? kLinear : kRect, it.q0,
                     it.x0, it.bh);
        load_tile<D>(smem + L::kDO, &tm_do_lin, &tm_do_img, &bars[L::bQFull], it.is_text ? kLinear : kRect, it.q0,
                     it.x0, it.bh);
        KeyIter ki;
        ki.init(g, it);
        KeyTile t;
        while (ki.next(&t)) {
          // V first: its slot frees as soon as dP of the tile before has run, so only K's load
          // waits for the dQ product.
          if (!mbar_wait(&bars[L::bVEmpty + stage], ring_ph ^ 1, abort_flag, kDevTimeoutTmaEmpty)) goto producer_done;
          mbar_arrive_expect_tx(&bars[L::bVFull + stage], L::kTileBytes);
          load_tile<D>(smem + L::kV + stage * L::kTileBytes, &tm_v_lin, &tm_v_img, &bars[L::bVFull + stage], t.kind,
                       t.a, t.b, it.bh);
          if (!mbar_wait(&bars[L::bKEmpty + stage], ring_ph ^ 1, abort_flag, kDevTimeoutTmaEmpty)) goto producer_done;
          mbar_arrive_expect_tx(&bars[L::bKFull + stage], L::kTileBytes);
          load_tile<D>(smem + L::kK + stage * L::kTileBytes, &tm_k_lin, &tm_k_img, &bars[L::bKFull + stage], t.kind,
                       t.a, t.b, it.bh);
          if (++stage == NST) { stage = 0; ring_ph ^= 1; }
        }
      }
      for (int s = 0; s < NST; ++s) {
        if (!mbar_wait(&bars[L::bVEmpty + stage], ring_ph ^ 1, abort_flag, kDevTimeoutTmaEmpty)) break;
        if (!mbar_wait(&bars[L::bKEmpty + stage], ring_ph ^ 1, abort_flag, kDevTimeoutTmaEmpty)) break;
        if (++stage == NST) { stage = 0; ring_ph ^= 1; }
      }
    producer_done:;
    }
    __syncwarp();
  } else if (warp == 9) {
    regs_dec<kBwdRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t do_addr = smem_u32(smem + L::kDO);
      static_assert(NST == 2, "S and dP of the next key tile are issued while dQ still reads this one's K");
      int stage = 0;
      uint32_t ring_ph = 0, q_full_ph = 0, sdp_free_ph = 0;
      // dP = dO V^T and S = Q K^T of key tile j into TMEM (K/V ring slot `stage`), once the softmax
      // has read the previous pair. dP goes first: V arrives earlier than K (its slot is released
      // after dP, K's after dQ), and K's load overlaps dP's issue.
      auto issue_sdp = [&](int j, int n) -> bool {
        if (!mbar_wait(&bars[L::bSdpFree], sdp_free_ph ^ 1, abort_flag, kDevTimeoutMma)) return false;
        sdp_free_ph ^= 1;
        if (!mbar_wait(&bars[L::bVFull + stage], ring_ph, abort_flag, kDevTimeoutMma)) return false;
        tc_fence_after();
        mma_kmajor<D>(tmem + L::kTmemDP, do_addr, smem_u32(smem + L::kV + stage * L::kTileBytes), idesc_s);
        umma_commit(&bars[L::bVEmpty + stage]);
        if (!mbar_wait(&bars[L::bKFull + stage], ring_ph, abort_flag, kDevTimeoutMma)) return false;
        tc_fence_after();
        mma_kmajor<D>(tmem + L::kTmemS, q_addr, smem_u32(smem + L::kK + stage * L::kTileBytes), idesc_s);
        umma_commit(&bars[L::bSdpFull]);
        if (j == n - 1) umma_commit(&bars[L::bQEmpty]);  // Q and dO: last reads issued
        return true;
      };
      // This thread issues the score products (S, dP) of every tile; warp 10 issues the dQ
      // products, so that the two streams' issue costs overlap (a thread is held ~80 cycles per
      // tcgen05.mma, and the two share no TMEM columns: dQ reads dS and K from shared memory).
      for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
        const WorkItem it = decode_work(g, w);
        const int n = count_key_tiles(g, it);
        if (!mbar_wait(&bars[L::bQFull], q_full_ph, abort_flag, kDevTimeoutMma)) goto mma_done;
        q_full_ph ^= 1;
        tc_fence_after();
        for (int j = 0; j < n; ++j) {
          if (!issue_sdp(j, n)) goto mma_done;
          if (++stage == NST) { stage = 0; ring_ph ^= 1; }
        }
      }
    mma_done:;
    }
    __syncwarp();
  } else if (warp == 10) {
    regs_dec<kBwdRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t ds_addr = smem_u32(smem + L::kDS);
      int stage = 0;
      uint32_t ring_ph = 0, ds_full_ph = 0;
      for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
        const WorkItem it = decode_work(g, w);
        const int n = count_key_tiles(g, it);
        for (int j = 0; j < n; ++j) {
          // dQ += dS K, once the softmax has stored dS of tile j. K's slot cannot have been
          // reloaded (that waits for this product), so its full barrier still shows tile j's load.
          if (!mbar_wait(&bars[L::bDsFull], ds_full_ph, abort_flag, kDevTimeoutMma)) goto dq_done;
          ds_full_ph ^= 1;
          if (!mbar_wait(&bars[L::bKFull + stage], ring_ph, abort_flag, kDevTimeoutMma)) goto dq_done;
          tc_fence_after();
          mma_a_kmajor_b_mnmajor<D>(tmem + L::kTmemAcc, ds_addr, smem_u32(smem + L::kK + stage * L::kTileBytes),
                                    idesc_dq, j > 0);
          umma_commit(&bars[L::bDsEmpty]);
          umma_commit(&bars[L::bKEmpty + stage]);
          if (j == n - 1) umma_commit(&bars[L::bAccDone]);
          if (++stage == NST) { stage = 0; ring_ph ^= 1; }
        }
      }
    dq_done:;
    }
    __syncwarp();
  } else if (warp < 8) {
    regs_inc<kBwdRegsHigh>();
    const int wg = warp >> 2;                // key columns [64 wg, 64 wg + 64) of every tile
    const int row = threadIdx.x & 127;       // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    constexpr int kC = kTile / 2;
    constexpr int kHalfD = D / 2;            // output columns of this warpgroup
    const uint32_t ds_addr = smem_u32(smem + L::kDS);
    uint32_t sdp_full_ph = 0, ds_empty_ph = 0, acc_ph = 0;
    const float sl2 = p.scale_log2;
    bool ds_pending = false;  // a dQ MMA may still read the dS buffer
    for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
      const WorkItem it = decode_work(g, w);
      int yq = 0, xq = 0;
      bool row_valid;
      size_t grow;  // this query row in [BH, T]
      if (it.is_text) {
        row_valid = (it.q0 + row) < g.n_text;
        grow = (size_t)it.bh * g.T + (it.q0 + row);
      } else {
        yq = it.q0 + (row >> 4);
        xq = it.x0 + (row & 15);
        row_valid = (yq < g.H) && (xq < g.W);
        grow = (size_t)it.bh * g.T + g.n_text + (size_t)yq * g.W + xq;
      }
      const float lse2 = row_valid ? p.l2vec[grow] : INFINITY;
      const float dd = row_valid ? p.dvec[grow] : 0.f;
      KeyIter ki;
      ki.init(g, it);
      KeyTile t;
      while (ki.next(&t)) {
        if (!mbar_wait(&bars[L::bSdpFull], sdp_full_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
        sdp_full_ph ^= 1;
        tc_fence_after();
        float s[kC];
        {
          uint32_t sr[2][32];
          tmem_ld32(tmem + lane_base + L::kTmemS + kC * wg, sr[0]);
          tmem_ld32(tmem + lane_base + L::kTmemS + kC * wg + 32, sr[1]);
          tmem_wait_ld();
          #pragma unroll
          for (int c = 0; c < kC; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        // P = 2^(s * c - lse2) on kept pairs, 0 elsewhere (this warpgroup's four key rows / 64 keys)
        if (t.flags != kFull) {
          if (t.kind == kLinear) {
            #pragma unroll
            for (int c = 0; c < kC; ++c)
              if (kC * wg + c >= t.b) s[c] = -INFINITY;
          } else {
            #pragma unroll
            for (int kr = 0; kr < kKH / 2; ++kr) {
              const uint32_t bits = rect_row_bits(g, wtab, yq, xq, t.a + (kKH / 2) * wg + kr, t.b);
              #pragma unroll
              for (int c = 0; c < kKW; ++c)
                if (!((bits >> c) & 1u)) s[kr * kKW + c] = -INFINITY;
            }
          }
        }
        {
          const uint64_t sl2x2 = f32x2_pack(sl2, sl2), nlse2 = f32x2_pack(-lse2, -lse2);
          #pragma unroll
          for (int c = 0; c < kC; c += 2) {  // P = 2^(s c - lse2) on packed pairs (same results as scalar fp32)
            const uint64_t x = f32x2_fma(f32x2_pack(s[c], s[c + 1]), sl2x2, nlse2);
            s[c] = ex2_approx(f32x2_lo(x));
            s[c + 1] = ex2_approx(f32x2_hi(x));
          }
        }
        float dp[kC];
        {
          uint32_t dr[2][32];
          tmem_ld32(tmem + lane_base + L::kTmemDP + kC * wg, dr[0]);
          tmem_ld32(tmem + lane_base + L::kTmemDP + kC * wg + 32, dr[1]);
          tmem_wait_ld();
          #pragma unroll
          for (int c = 0; c < kC; ++c) dp[c] = __uint_as_float(dr[c >> 5][c & 31]);
        }
        tc_fence_before();
        mbar_arrive(&bars[L::bSdpFree]);
        {
          const uint64_t ndd2 = f32x2_pack(-dd, -dd);
          #pragma unroll
          for (int c = 0; c < kC; c += 2) {  // dS = P (dP - D)
            const uint64_t ds = f32x2_mul(f32x2_pack(s[c], s[c + 1]), f32x2_add(f32x2_pack(dp[c], dp[c + 1]), ndd2));
            s[c] = f32x2_lo(ds);
            s[c + 1] = f32x2_hi(ds);
          }
        }
        if (ds_pending) {
          if (!mbar_wait(&bars[L::bDsEmpty], ds_empty_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
          ds_empty_ph ^= 1;
        }
        store_chunk32_sw128(ds_addr, row, 2 * wg, s);
        store_chunk32_sw128(ds_addr, row, 2 * wg + 1, s + 32);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[L::bDsFull]);
        ds_pending = true;
      }
      // epilogue: this warpgroup's half of the dQ row
      if (!mbar_wait(&bars[L::bAccDone], acc_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
      acc_ph ^= 1;
      if (ds_pending) {  // the last dQ MMA has completed too
        if (!mbar_wait(&bars[L::bDsEmpty], ds_empty_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
        ds_empty_ph ^= 1;
        ds_pending = false;
      }
      tc_fence_after();
      {
        const uint32_t abase = tmem + lane_base + L::kTmemAcc + wg * kHalfD;
        #pragma unroll
        for (int c = 0; c < kHalfD / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(abase + c * 32, ov);
          tmem_wait_ld();
          if (!row_valid) continue;
          const int col = wg * kHalfD + c * 32;
          if (it.is_text) {
            float* dst = p.part_a + (((size_t)it.split * g.BH + it.bh) * g.n_text + it.q0 + row) * D + col;
            float4* d4 = reinterpret_cast<float4*>(dst);
            #pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                                  __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(p.out_a + grow * D + col);
            const float sc = p.scale;
            #pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pack_bf16x2(__uint_as_float(ov[8 * e + 0]) * sc, __uint_as_float(ov[8 * e + 1]) * sc),
                                 pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * sc, __uint_as_float(ov[8 * e + 3]) * sc),
                                 pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * sc, __uint_as_float(ov[8 * e + 5]) * sc),
                                 pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * sc, __uint_as_float(ov[8 * e + 7]) * sc));
          }
        }
      }
      tc_fence_before();
    }
  softmax_done:;
  } else {
    regs_dec<kBwdRegsLow>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// dK/dV kernel (KV-stationary)
// ------------------------------------------------------------------------------------------------
template <int D>
struct DkvLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytes;
  // Two buffers of the partner query tile's Q and dO, so the next tile loads during this one.
  static constexpr int kQ = kV + kTileBytes;             // + buf * kQStride
  static constexpr int kDO = kQ + kTileBytes;            // + buf * kQStride
  static constexpr int kQStride = 2 * kTileBytes;
  static constexpr int kVec = kQ + 2 * kQStride;         // float [tile parity][warpgroup][lse2 | D][64]
  static constexpr int kBars = kVec + 4 * kTile * 4;
  static constexpr int bKVFull = 0, bKVEmpty = 1, bQFull = 2 /* + buf */, bQEmpty = 4 /* + buf */,
                       bSFull = 6 /* + half */, bPFull = 8 /* + half */, bAccDone = 10;
  static constexpr int kNumBars = 11;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kWTab = kMisc + 16;
  static constexpr int kTotal = kWTab + kMaxRTable * 4;
  static constexpr int kAlloc = kTotal + 1024;
  // TMEM: S^T of the partner tile's two 64-query halves at columns 0 and 64, dP^T likewise at 128
  // and 192, and the dV, dK accumulators. Each warpgroup reads a 32-column chunk of each half and
  // writes its P^T (dS^T) as bf16 pairs over the first 16 columns of that same chunk.
  static constexpr uint32_t kTmemS = 0, kTmemDP = 128, kTmemDV = 256, kTmemDK = 256 + D, kTmemCols = 512;
};

// KV-stationary: one CTA holds a key tile's K and V and visits its partner query tiles (the
// mask is symmetric, so they are the key tiles KeyIter lists for a query tile at the same place):
// S^T = K Q^T and dP^T = V dO^T into TMEM, P^T = 2^(S^T c - lse2) and dS^T = P^T (dP^T - D)
// written back over them as bf16, then dV += P^T dO and dK += dS^T Q with the A operand read from
// TMEM. Partner Q / dO tiles are double-buffered. Each partner tile is taken as two halves of 64
// queries with barriers of their own, so that the tensor pipe works on one half (dV, dK of half a,
// then S^T, dP^T of the next tile's half a) while the softmax turns the other into P^T, dS^T.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
clear_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q_lin, const __grid_constant__ CUtensorMap tm_q_img,
                      const __grid_constant__ CUtensorMap tm_do_lin, const __grid_constant__ CUtensorMap tm_do_img,
                      const __grid_constant__ CUtensorMap tm_k_lin, const __grid_constant__ CUtensorMap tm_k_img,
                      const __grid_constant__ CUtensorMap tm_v_lin, const __grid_constant__ CUtensorMap tm_v_img,
                      const BwdParams p) {
  using L = DkvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  int* wtab = reinterpret_cast<int*>(smem + L::kWTab);
  float* vec = reinterpret_cast<float*>(smem + L::kVec);  // [buf][lse2 | dvec][128]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::bKVFull], 1);
    mbar_init(&bars[L::bKVEmpty], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[L::bQFull + b], 1);
      mbar_init(&bars[L::bQEmpty + b], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars[L::bSFull + h], 1);
      mbar_init(&bars[L::bPFull + h], 256);
    }
    mbar_init(&bars[L::bAccDone], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kMaxRTable; i += blockDim.x) wtab[i] = half_width(g.r, i, g.window);
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    regs_dec<kBwdRegsLow>();
    if (lane == 0) {
      uint32_t kv_empty_ph = 0, c = 0;  // c: partner tiles loaded so far
      bool first_item = true;
      for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
        const WorkItem it = decode_work(g, w);  // the stationary key tile
        if (!first_item) {
          if (!mbar_wait(&bars[L::bKVEmpty], kv_empty_ph, abort_flag, kDevTimeoutTmaEmpty)) goto producer_done;
          kv_empty_ph ^= 1;
        }
        first_item = false;
        mbar_arrive_expect_tx(&bars[L::bKVFull], 2 * L::kTileBytes);
        load_tile<D>(smem + L::kK, &tm_k_lin, &tm_k_img, &bars[L::bKVFull], it.is_text ? kLinear : kRect, it.q0,
                     it.x0, it.bh);
        load_tile<D>(smem + L::kV, &tm_v_lin, &tm_v_img, &bars[L::bKVFull], it.is_text ? kLinear : kRect, it.q0,
                     it.x0, it.bh);
        KeyIter ki;
        ki.init(g, it);
        KeyTile t;
        while (ki.next(&t)) {  // partner query tiles
          const uint32_t qb = c & 1;
          if (c >= 2 && !mbar_wait(&bars[L::bQEmpty + qb], ((c >> 1) - 1) & 1, abort_flag, kDevTimeoutTmaEmpty))
            goto producer_done;
          mbar_arrive_expect_tx(&bars[L::bQFull + qb], 2 * L::kTileBytes);
          load_tile<D>(smem + L::kQ + qb * L::kQStride, &tm_q_lin, &tm_q_img, &bars[L::bQFull + qb], t.kind, t.a,
                       t.b, it.bh);
          load_tile<D>(smem + L::kDO + qb * L::kQStride, &tm_do_lin, &tm_do_img, &bars[L::bQFull + qb], t.kind,
                       t.a, t.b, it.bh);
          ++c;
        }
      }
    producer_done:;
    }
    __syncwarp();
  } else if (warp == 9) {
    regs_dec<kBwdRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // one half: 64 partner queries
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      constexpr uint32_t kHalfRows = 64 * 128;  // bytes of 64 rows in each 64-column block of a tile
      uint32_t kv_full_ph = 0, p_full_ph[2] = {0, 0}, c = 0;
      // S^T and dP^T of half h of partner tile cc. They overwrite that half's P^T and dS^T of the
      // tile before, whose readers (dV, dK of the half) were issued before, by this thread, and
      // run first.
      auto scores = [&](uint32_t cc, int h) {
        const uint32_t qb = cc & 1;
        const uint32_t q_addr = smem_u32(smem + L::kQ + qb * L::kQStride) + h * kHalfRows;
        const uint32_t do_addr = smem_u32(smem + L::kDO + qb * L::kQStride) + h * kHalfRows;
        mma_kmajor<D>(tmem + L::kTmemS + 64 * h, k_addr, q_addr, idesc_s);    // S^T = K Q^T
        mma_kmajor<D>(tmem + L::kTmemDP + 64 * h, v_addr, do_addr, idesc_s);  // dP^T = V dO^T
        umma_commit(&bars[L::bSFull + h]);
      };
      // dV += P^T dO and dK += dS^T Q over the 64 partner queries of half h (four K16 steps each).
      // Step j's 16 queries are packed (8 columns) at the start of their warpgroup's 32-column chunk:
      // column 64 h + 32 (j / 2) + 8 (j % 2) of the S^T (P^T) and dP^T (dS^T) regions.
      auto accumulate = [&](uint32_t cc, int h, bool first) {
        const uint32_t qb = cc & 1;
        const uint64_t do_desc = smem_desc_sw128(smem_u32(smem + L::kDO + qb * L::kQStride), kHalfBytes, 1024);
        const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + L::kQ + qb * L::kQStride), kHalfBytes, 1024);
        #pragma unroll
        for (int j = 0; j < 4; ++j)
          umma_ts(tmem + L::kTmemDV, tmem + L::kTmemS + 64 * h + 32 * (j >> 1) + 8 * (j & 1),
                  do_desc + (uint64_t)(((4 * h + j) * 2048) >> 4), idesc_acc, (first && j == 0) ? 0u : 1u);
        #pragma unroll
        for (int j = 0; j < 4; ++j)
          umma_ts(tmem + L::kTmemDK, tmem + L::kTmemDP + 64 * h + 32 * (j >> 1) + 8 * (j & 1),
                  q_desc + (uint64_t)(((4 * h + j) * 2048) >> 4), idesc_acc, (first && j == 0) ? 0u : 1u);
      };
      for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
        const WorkItem it = decode_work(g, w);
        const int n = count_key_tiles(g, it);
        if (!mbar_wait(&bars[L::bKVFull], kv_full_ph, abort_flag, kDevTimeoutMma)) goto mma_done;
        kv_full_ph ^= 1;
        if (n > 0) {
          if (!mbar_wait(&bars[L::bQFull + (c & 1)], (c >> 1) & 1, abort_flag, kDevTimeoutMma)) goto mma_done;
          tc_fence_after();
          scores(c, 0);
          scores(c, 1);
        }
        for (int i = 0; i < n; ++i, ++c) {
          const bool more = i + 1 < n;
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(&bars[L::bPFull + h], p_full_ph[h], abort_flag, kDevTimeoutMma)) goto mma_done;
            p_full_ph[h] ^= 1;
            tc_fence_after();
            accumulate(c, h, i == 0 && h == 0);
            if (h == 1) umma_commit(&bars[L::bQEmpty + (c & 1)]);  // last reads of this Q / dO buffer issued
            if (more) {
              if (h == 0) {
                if (!mbar_wait(&bars[L::bQFull + ((c + 1) & 1)], ((c + 1) >> 1) & 1, abort_flag, kDevTimeoutMma))
                  goto mma_done;
                tc_fence_after();
              }
              scores(c + 1, h);
            }
          }
        }
        umma_commit(&bars[L::bAccDone]);
        umma_commit(&bars[L::bKVEmpty]);
      }
    mma_done:;
    }
    __syncwarp();
  } else if (warp < 8) {
    regs_inc<kBwdRegsHigh>();
    const int wg = warp >> 2;                // partner query columns [64 wg, 64 wg + 64) of every tile
    const int row = threadIdx.x & 127;       // key row of the stationary tile = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    constexpr int kHalfD = D / 2;            // output columns of this warpgroup
    uint32_t s_full_ph[2] = {0, 0}, acc_ph = 0;
    const float sl2 = p.scale_log2;
    uint32_t tile_counter = 0;
    for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
      const WorkItem it = decode_work(g, w);
      int yk = 0, xk = 0;
      bool row_valid;
      size_t grow;
      if (it.is_text) {
        row_valid = (it.q0 + row) < g.n_text;
        grow = (size_t)it.bh * g.T + (it.q0 + row);
      } else {
        yk = it.q0 + (row >> 4);
        xk = it.x0 + (row & 15);
        row_valid = (yk < g.H) && (xk < g.W);
        grow = (size_t)it.bh * g.T + g.n_text + (size_t)yk * g.W + xk;
      }
      KeyIter ki;
      ki.init(g, it);
      KeyTile t;
      while (ki.next(&t)) {
        // Row statistics of this warpgroup's 64 partner columns (its 32-column chunk of each half)
        // into its own block, [lse2 | D][64] per tile parity: thread r stores lse2 of local column r
        // (r < 64) or D of local column r - 64. Only this warpgroup reads them.
        float* lse_s = vec + ((tile_counter & 1) * 2 + wg) * 2 * 64;
        float* dv_s = lse_s + 64;
        ++tile_counter;
        {
          const int cl = row & 63;
          const int c = cl < 32 ? 32 * wg + cl : 32 + 32 * wg + cl;  // the tile's column
          bool ok;
          size_t qrow;
          if (t.kind == kLinear) {
            ok = c < t.b;
            qrow = (size_t)it.bh * g.T + t.a + c;
          } else {
            const int yq = t.a + (c >> 4), xq = t.b + (c & 15);
            ok = yq < g.H && xq < g.W && yq >= 0 && xq >= 0;
            qrow = ok ? (size_t)it.bh * g.T + g.n_text + (size_t)yq * g.W + xq : 0;
          }
          if (row < 64)
            lse_s[cl] = ok ? p.l2vec[qrow] : INFINITY;
          else
            dv_s[cl] = ok ? p.dvec[qrow] : 0.f;
        }
        named_bar_sync(1 + wg, 128);
        for (int h = 0; h < 2; ++h) {  // the tile's two 64-query halves
          if (!mbar_wait(&bars[L::bSFull + h], s_full_ph[h], abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
          s_full_ph[h] ^= 1;
          tc_fence_after();
          const int gch = 2 * h + wg;  // this warpgroup's 32-column chunk of the tile
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_base + L::kTmemS + 32 * gch, sr);
          tmem_ld32(tmem + lane_base + L::kTmemDP + 32 * gch, dr);
          tmem_wait_ld();
          // P^T = 2^(s c - lse2) on kept pairs, dS^T = P^T (dP^T - D), as bf16 pairs, written over
          // the first 16 columns of this warpgroup's own chunk (each thread only touches its own
          // TMEM lane, so the two warpgroups never wait for each other).
          uint32_t keep = 0xffffffffu;
          if (t.flags != kFull) {
            if (t.kind == kLinear) {
              const int lim = t.b - gch * 32;
              keep = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
            } else {
              keep = rect_row_bits(g, wtab, yk, xk, t.a + 2 * gch, t.b) |
                     (rect_row_bits(g, wtab, yk, xk, t.a + 2 * gch + 1, t.b) << 16);
            }
          }
          uint32_t pw[16], dw[16];
          const uint64_t sl2x2 = f32x2_pack(sl2, sl2);
          #pragma unroll
          for (int e = 0; e < 32; e += 2) {  // packed pairs: the same results as scalar fp32
            const int c = h * 32 + e;  // local column
            const float x0 = ((keep >> e) & 1u) ? __uint_as_float(sr[e]) : -INFINITY;
            const float x1 = ((keep >> (e + 1)) & 1u) ? __uint_as_float(sr[e + 1]) : -INFINITY;
            const uint64_t x = f32x2_fma(f32x2_pack(x0, x1), sl2x2, f32x2_pack(-lse_s[c], -lse_s[c + 1]));
            const float p0 = ex2_approx(f32x2_lo(x));
            const float p1 = ex2_approx(f32x2_hi(x));
            const uint64_t d = f32x2_mul(f32x2_pack(p0, p1),
                                         f32x2_add(f32x2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])),
                                                   f32x2_pack(-dv_s[c], -dv_s[c + 1])));
            pw[e / 2] = pack_bf16x2(p0, p1);
            dw[e / 2] = pack_bf16x2(f32x2_lo(d), f32x2_hi(d));
          }
          tmem_st16(tmem + lane_base + L::kTmemS + 32 * gch, pw);
          tmem_st16(tmem + lane_base + L::kTmemDP + 32 * gch, dw);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars[L::bPFull + h]);
        }
      }
      if (!mbar_wait(&bars[L::bAccDone], acc_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
      acc_ph ^= 1;
      tc_fence_after();
      #pragma unroll
      for (int which = 0; which < 2; ++which) {  // 0: dK, 1: dV; this warpgroup's half of each row
        const uint32_t abase = tmem + lane_base + (which == 0 ? L::kTmemDK : L::kTmemDV) + wg * kHalfD;
        const float sc = which == 0 ? p.scale : 1.f;
        #pragma unroll
        for (int c = 0; c < kHalfD / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(abase + c * 32, ov);
          tmem_wait_ld();
          if (!row_valid) continue;
          const int col = wg * kHalfD + c * 32;
          if (it.is_text) {
            float* part = which == 0 ? p.part_a : p.part_b;
            float* dst = part + (((size_t)it.split * g.BH + it.bh) * g.n_text + it.q0 + row) * D + col;
            float4* d4 = reinterpret_cast<float4*>(dst);
            #pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                                  __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
          } else {
            __nv_bfloat16* out = which == 0 ? p.out_a : p.out_b;
            uint4* d4 = reinterpret_cast<uint4*>(out + grow * D + col);
            #pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pack_bf16x2(__uint_as_float(ov[8 * e + 0]) * sc, __uint_as_float(ov[8 * e + 1]) * sc),
                                 pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * sc, __uint_as_float(ov[8 * e + 3]) * sc),
                                 pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * sc, __uint_as_float(ov[8 * e + 5]) * sc),
                                 pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * sc, __uint_as_float(ov[8 * e + 7]) * sc));
          }
        }
      }
      tc_fence_before();
    }
  softmax_done:;
  } else {
    regs_dec<kBwdRegsLow>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// Host launcher
// ------------------------------------------------------------------------------------------------
template <int D>
inline clear_status_t launch_bwd(const BwdArgs& a, const CUtensorMap& q_lin, const CUtensorMap& q_img,
                                 const CUtensorMap& k_lin, const CUtensorMap& k_img, const CUtensorMap& v_lin,
                                 const CUtensorMap& v_img, const CUtensorMap& do_lin, const CUtensorMap& do_img,
                                 int num_sms, cudaStream_t stream) {
  constexpr int NST = (DqLayout<D, 2>::kAlloc <= 232448) ? 2 : 1;
  using LQ = DqLayout<D, NST>;
  using LKV = DkvLayout<D>;
  static_assert(LKV::kAlloc <= 232448, "dkdv smem");
  const Geom& g = a.g;
  float* dvec = reinterpret_cast<float*>(a.ws + a.wl.dvec_off);
  float* l2vec = reinterpret_cast<float*>(a.ws + a.wl.l2vec_off);
  const long long rows = (long long)g.BH * g.T;
  clear_bwd_preprocess_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(a.o, a.dO, a.lse, dvec, l2vec, rows);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;

  BwdParams p{};
  p.g = g;
  p.scale = (float)(1.0 / std::sqrt((double)D));
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.dvec = dvec;
  p.l2vec = l2vec;
  p.n_work = g.n_txt_items + g.n_img_items;
  const long long grid = p.n_work < num_sms ? p.n_work : num_sms;

  // dQ
  p.out_a = a.dq;
  p.out_b = nullptr;
  p.part_a = reinterpret_cast<float*>(a.ws + a.wl.dq_off);
  p.part_b = nullptr;
  if (cudaFuncSetAttribute(clear_bwd_dq_kernel<D, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, LQ::kAlloc) !=
      cudaSuccess)
    return CLEAR_ERR_CUDA;
  clear_bwd_dq_kernel<D, NST><<<(unsigned)grid, kBwdThreads, LQ::kAlloc, stream>>>(q_lin, q_img, do_lin, do_img, k_lin,
                                                                                   k_img, v_lin, v_img, p);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;

  // dK, dV
  p.out_a = a.dk;
  p.out_b = a.dv;
  p.part_a = reinterpret_cast<float*>(a.ws + a.wl.dk_off);
  p.part_b = reinterpret_cast<float*>(a.ws + a.wl.dv_off);
  if (cudaFuncSetAttribute(clear_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LKV::kAlloc) !=
      cudaSuccess)
    return CLEAR_ERR_CUDA;
  clear_bwd_dkdv_kernel<D><<<(unsigned)grid, kBwdThreads, LKV::kAlloc, stream>>>(q_lin, q_img, do_lin, do_img, k_lin,
                                                                                 k_img, v_lin, v_img, p);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;

  if (g.n_text > 0) {
    const long long trows = (long long)g.BH * g.n_text;
    const unsigned blocks = (unsigned)((trows + 7) / 8);
    clear_bwd_reduce_kernel<D><<<blocks, 256, 0, stream>>>(reinterpret_cast<float*>(a.ws + a.wl.dq_off), a.dq, g,
                                                           p.scale);
    clear_bwd_reduce_kernel<D><<<blocks, 256, 0, stream>>>(reinterpret_cast<float*>(a.ws + a.wl.dk_off), a.dk, g,
                                                           p.scale);
    clear_bwd_reduce_kernel<D><<<blocks, 256, 0, stream>>>(reinterpret_cast<float*>(a.ws + a.wl.dv_off), a.dv, g, 1.f);
    if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  }
  return CLEAR_OK;
}

}  // namespace clear
