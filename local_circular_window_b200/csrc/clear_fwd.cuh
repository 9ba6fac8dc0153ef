// CLEAR attention forward on sm_100a: TMA -> shared memory -> tcgen05.mma (TMEM accumulators)
// -> masked online softmax in registers -> tcgen05.mma for P V.
//
// Semantics (pith.science review of "CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion
// Transformers Up", "Core claim" and "What carries the argument"): every query row takes one
// softmax over the keys the CLEAR mask keeps, scores scaled by 1/sqrt(d); text rows keep every
// key, image rows keep all text keys plus image keys with dx^2 + dy^2 < r^2.
//
// One CTA per SM, persistent over a static list of work items (clear_sched.cuh):
//   warps 0-3  softmax / epilogue: thread t owns query row t of the 128-row tile (TMEM lane t);
//   warp 4     TMA producer: Q tile once per item, then K and V tiles into a 2-stage ring;
//   warp 5     MMA issuer: S = Q K^T into one of two TMEM S buffers, O += P V into TMEM O.
// P goes from registers to shared memory as bf16 (128B-swizzled, K-major) for the P V MMA.
// The running max is rescaled lazily: O and l are only rescaled when a row's max grows by more
// than 2^8, which leaves the result exact up to rounding (the final division uses the same max).
#pragma once
#include <cuda_bf16.h>

#include "clear_sched.cuh"
#include "sm100_ptx.cuh"

namespace clear {

constexpr int kFwdStages = 2;
constexpr int kFwdThreads = 192;
constexpr int kMaxRTable = 256;      // radius up to which the half-width table lives in smem
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdParams {
  Geom g;
  float scale_log2;           // (1/sqrt(d)) * log2(e)
  __nv_bfloat16* o;           // [BH, T, d]
  float* lse;                 // [BH, T]
  float* opart;               // [S, BH, n_text, d] unnormalised partial O of text rows
  float2* ml;                 // [S, BH, n_text] (running max in scaled log2 units, sum)
  long long n_work;
};

template <int D>
struct FwdLayout {
  static constexpr int kHalves = D / 64;                 // 64-element (128 B) column blocks
  static constexpr int kTileBytes = kTile * D * 2;       // one 128-row bf16 tile
  static constexpr int kHalfBytes = kTile * 128;         // one 128 x 64 block
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kFwdStages * kTileBytes;
  static constexpr int kP = kV + kFwdStages * kTileBytes;
  static constexpr int kPBytes = kTile * kTile * 2;
  static constexpr int kBars = kP + kPBytes;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 1, bPFull = 2, bODone = 3;
  static constexpr int bKFull = 4;                       // + stage
  static constexpr int bVFull = bKFull + kFwdStages;     // + stage
  static constexpr int bKVEmpty = bVFull + kFwdStages;   // + stage
  static constexpr int bSFull = bKVEmpty + kFwdStages;   // + buffer (2)
  static constexpr int bSFree = bSFull + 2;              // + buffer (2)
  static constexpr int kNumBars = bSFree + 2;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kWTab = kMisc + 16;               // int[kMaxRTable]
  static constexpr int kTotal = kWTab + kMaxRTable * 4;
  static constexpr int kAlloc = kTotal + 1024;           // slack for 1024-byte alignment
  // TMEM columns
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO = 256, kTmemCols = 512;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Loads one 128-row tile (all 64-column halves) of q/k/v for a query or key tile.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* lin, const CUtensorMap* img,
                                          uint64_t* bar, int kind, int a, int b, int bh) {
  #pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    uint8_t* d = dst + h * FwdLayout<D>::kHalfBytes;
    if (kind == kLinear)
      tma_load_3d(d, lin, bar, h * 64, a, bh);
    else
      tma_load_4d(d, img, bar, h * 64, b, a, bh);
  }
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
clear_fwd_kernel(const __grid_constant__ CUtensorMap tm_q_lin, const __grid_constant__ CUtensorMap tm_q_img,
                 const __grid_constant__ CUtensorMap tm_k_lin, const __grid_constant__ CUtensorMap tm_k_img,
                 const __grid_constant__ CUtensorMap tm_v_lin, const __grid_constant__ CUtensorMap tm_v_img,
                 const FwdParams p) {
  using L = FwdLayout<D>;
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
    mbar_init(&bars[L::bPFull], 128);
    mbar_init(&bars[L::bODone], 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&bars[L::bKFull + s], 1);
      mbar_init(&bars[L::bVFull + s], 1);
      mbar_init(&bars[L::bKVEmpty + s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[L::bSFull + b], 1);
      mbar_init(&bars[L::bSFree + b], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Half-width table: wtab[dy] = largest dx with dx^2 + dy^2 < r^2 (or -1).
  for (int i = threadIdx.x; i < kMaxRTable; i += blockDim.x) wtab[i] = half_width(g.r, i);
  if (warp == 5) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q_lin); tma_prefetch_desc(&tm_q_img);
      tma_prefetch_desc(&tm_k_lin); tma_prefetch_desc(&tm_k_img);
      tma_prefetch_desc(&tm_v_lin); tma_prefetch_desc(&tm_v_img);
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
        mbar_arrive_expect_tx(&bars[L::bQFull], L::kTileBytes);
        load_tile<D>(smem + L::kQ, &tm_q_lin, &tm_q_img, &bars[L::bQFull],
                     it.is_text ? kLinear : kRect, it.q0, it.x0, it.bh);
        KeyIter ki;
        ki.init(g, it);
        KeyTile t;
        while (ki.next(&t)) {
          if (!mbar_wait(&bars[L::bKVEmpty + stage], ring_ph ^ 1, abort_flag, kDevTimeoutTmaEmpty))
            goto producer_done;
          mbar_arrive_expect_tx(&bars[L::bKFull + stage], L::kTileBytes);
          load_tile<D>(smem + L::kK + stage * L::kTileBytes, &tm_k_lin, &tm_k_img,
                       &bars[L::bKFull + stage], t.kind, t.a, t.b, it.bh);
          mbar_arrive_expect_tx(&bars[L::bVFull + stage], L::kTileBytes);
          load_tile<D>(smem + L::kV + stage * L::kTileBytes, &tm_v_lin, &tm_v_img,
                       &bars[L::bVFull + stage], t.kind, t.a, t.b, it.bh);
          if (++stage == kFwdStages) { stage = 0; ring_ph ^= 1; }
        }
      }
      // Drain: wait until the consumer has released every stage, so no copy is in flight.
      for (int s = 0; s < kFwdStages; ++s) {
        if (!mbar_wait(&bars[L::bKVEmpty + stage], ring_ph ^ 1, abort_flag, kDevTimeoutTmaEmpty)) break;
        if (++stage == kFwdStages) { stage = 0; ring_ph ^= 1; }
      }
    producer_done:;
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t p_addr = smem_u32(smem + L::kP);
      int stage = 0;
      uint32_t ring_ph = 0, q_full_ph = 0, p_full_ph = 0;
      uint32_t s_free_ph[2] = {0, 0};
      uint32_t J = 0;  // global key-tile counter (S buffer = J & 1)
      for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
        const WorkItem it = decode_work(g, w);
        const int n = count_key_tiles(g, it);
        if (!mbar_wait(&bars[L::bQFull], q_full_ph, abort_flag, kDevTimeoutMma)) goto mma_done;
        q_full_ph ^= 1;
        tc_fence_after();
        int st_j = stage;               // stage of tile j
        uint32_t ph_j = ring_ph;        // ring phase of tile j
        // QK for tile 0
        {
          const uint32_t b = J & 1;
          if (!mbar_wait(&bars[L::bSFree + b], s_free_ph[b] ^ 1, abort_flag, kDevTimeoutMma)) goto mma_done;
          s_free_ph[b] ^= 1;
          if (!mbar_wait(&bars[L::bKFull + st_j], ph_j, abort_flag, kDevTimeoutMma)) goto mma_done;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + L::kK + st_j * L::kTileBytes);
          #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kHalfBytes + (kk & 3) * 32;
            umma_ss(tmem + (b ? L::kTmemS1 : L::kTmemS0), smem_desc_sw128(q_addr + off, 16, 1024),
                    smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0);
          }
          umma_commit(&bars[L::bSFull + b]);
          if (n == 1) umma_commit(&bars[L::bQEmpty]);
        }
        for (int j = 0; j < n; ++j) {
          // next stage/phase
          int st_n = st_j + 1;
          uint32_t ph_n = ph_j;
          if (st_n == kFwdStages) { st_n = 0; ph_n ^= 1; }
          if (j + 1 < n) {
            const uint32_t b = (J + 1) & 1;
            if (!mbar_wait(&bars[L::bSFree + b], s_free_ph[b] ^ 1, abort_flag, kDevTimeoutMma)) goto mma_done;
            s_free_ph[b] ^= 1;
            if (!mbar_wait(&bars[L::bKFull + st_n], ph_n, abort_flag, kDevTimeoutMma)) goto mma_done;
            tc_fence_after();
            const uint32_t k_addr = smem_u32(smem + L::kK + st_n * L::kTileBytes);
            #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * L::kHalfBytes + (kk & 3) * 32;
              umma_ss(tmem + (b ? L::kTmemS1 : L::kTmemS0), smem_desc_sw128(q_addr + off, 16, 1024),
                      smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0);
            }
            umma_commit(&bars[L::bSFull + b]);
            if (j + 1 == n - 1) umma_commit(&bars[L::bQEmpty]);
          }
          // O += P_j V_j
          if (!mbar_wait(&bars[L::bPFull], p_full_ph, abort_flag, kDevTimeoutMma)) goto mma_done;
          p_full_ph ^= 1;
          if (!mbar_wait(&bars[L::bVFull + st_j], ph_j, abort_flag, kDevTimeoutMma)) goto mma_done;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(smem + L::kV + st_j * L::kTileBytes);
          #pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint32_t a_off = (kk >> 2) * L::kHalfBytes + (kk & 3) * 32;
            umma_ss(tmem + L::kTmemO, smem_desc_sw128(p_addr + a_off, 16, 1024),
                    smem_desc_sw128(v_addr + kk * 2048, L::kHalfBytes, 1024), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars[L::bODone]);
          umma_commit(&bars[L::bKVEmpty + st_j]);
          st_j = st_n;
          ph_j = ph_n;
          ++J;
        }
        stage = st_j;
        ring_ph = ph_j;
      }
    mma_done:;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x;  // 0..127 == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t p_addr = smem_u32(smem + L::kP);
    uint32_t s_full_ph[2] = {0, 0};
    uint32_t o_done_ph = 0;
    uint32_t J = 0;
    const float sl2 = p.scale_log2;
    for (long long w = blockIdx.x; w < p.n_work; w += gridDim.x) {
      const WorkItem it = decode_work(g, w);
      int yq = 0, xq = 0;
      bool row_valid;
      if (it.is_text) {
        row_valid = (it.q0 + row) < g.n_text;
      } else {
        yq = it.q0 + (row >> 4);
        xq = it.x0 + (row & 15);
        row_valid = (yq < g.H) && (xq < g.W);
      }
      float m_used = -INFINITY;  // running max, scaled log2 units
      float l = 0.f;
      KeyIter ki;
      ki.init(g, it);
      KeyTile t;
      int j = 0;
      while (ki.next(&t)) {
        const uint32_t b = J & 1;
        if (!mbar_wait(&bars[L::bSFull + b], s_full_ph[b], abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
        s_full_ph[b] ^= 1;
        tc_fence_after();
        float s[kTile];
        {
          uint32_t sr[4][32];
          const uint32_t sbase = tmem + lane_base + (b ? L::kTmemS1 : L::kTmemS0);
          tmem_ld32(sbase + 0, sr[0]);
          tmem_ld32(sbase + 32, sr[1]);
          tmem_ld32(sbase + 64, sr[2]);
          tmem_ld32(sbase + 96, sr[3]);
          tmem_wait_ld();
          #pragma unroll
          for (int c = 0; c < kTile; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        tc_fence_before();
        mbar_arrive(&bars[L::bSFree + b]);
        // ---- mask
        if (t.flags != kFull) {
          if (t.kind == kLinear) {
            #pragma unroll
            for (int c = 0; c < kTile; ++c)
              if (c >= t.b) s[c] = -INFINITY;
          } else {
            #pragma unroll
            for (int kr = 0; kr < kKH; ++kr) {
              const int ky = t.a + kr;
              const int dy = ky - yq;
              const int ady = dy < 0 ? -dy : dy;
              int wdt = -1;
              if (ky < g.H) wdt = (ady < kMaxRTable) ? (ady < g.r ? wtab[ady] : -1) : half_width(g.r, ady);
              int lo = imax(xq - wdt, 0) - t.b;
              int hi = imin(xq + wdt, g.W - 1) - t.b;
              lo = imax(lo, 0);
              hi = imin(hi, kKW - 1);
              uint32_t bits = 0;
              if (wdt >= 0 && lo <= hi) bits = ((2u << hi) - 1u) & ~((1u << lo) - 1u);
              #pragma unroll
              for (int c = 0; c < kKW; ++c)
                if (!((bits >> c) & 1u)) s[kr * kKW + c] = -INFINITY;
            }
          }
        }
        // ---- tile max
        float mt = s[0];
        #pragma unroll
        for (int c = 1; c < kTile; ++c) mt = fmaxf(mt, s[c]);
        const float mt_scaled = mt * sl2;
        // PV_{j-1} must be done before P is overwritten and before O is rescaled.
        if (j > 0) {
          if (!mbar_wait(&bars[L::bODone], o_done_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
          o_done_ph ^= 1;
          tc_fence_after();
        }
        float alpha = 1.f;
        bool need_rescale = false;
        if (m_used == -INFINITY) {
          m_used = mt_scaled;  // nothing accumulated yet (l == 0, O == 0)
        } else if (mt_scaled > m_used + kRescaleThreshold) {
          alpha = ex2_approx(m_used - mt_scaled);
          l *= alpha;
          m_used = mt_scaled;
          need_rescale = true;
        }
        if (j > 0 && __any_sync(0xffffffffu, need_rescale)) {
          const uint32_t obase = tmem + lane_base + L::kTmemO;
          #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(obase + c * 32, ov);
            tmem_wait_ld();
            #pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(obase + c * 32, ov);
          }
          tmem_wait_st();
        }
        // ---- P = 2^(s * scale_log2 - m), row sum, bf16 to smem (128B swizzle, K-major)
        const float base = (m_used == -INFINITY) ? 0.f : m_used;
        float lsum = 0.f;
        #pragma unroll
        for (int ch = 0; ch < kTile / 8; ++ch) {
          float e[8];
          #pragma unroll
          for (int u = 0; u < 8; ++u) {
            e[u] = ex2_approx(fmaf(s[ch * 8 + u], sl2, -base));
            lsum += e[u];
          }
          const uint32_t addr = p_addr + (ch >> 3) * L::kHalfBytes + row * 128 +
                                ((((uint32_t)ch & 7u) ^ ((uint32_t)row & 7u)) << 4);
          st_shared_v4(addr, pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]),
                       pack_bf16x2(e[4], e[5]), pack_bf16x2(e[6], e[7]));
        }
        l += lsum;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[L::bPFull]);
        ++J;
        ++j;
      }
      // ---- epilogue: wait for the last P V, then write O / l (or the split partial)
      if (!mbar_wait(&bars[L::bODone], o_done_ph, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
      o_done_ph ^= 1;
      tc_fence_after();
      {
        const uint32_t obase = tmem + lane_base + L::kTmemO;
        if (it.is_text) {
          const size_t prow = ((size_t)it.split * g.BH + it.bh) * g.n_text + (it.q0 + row);
          float* dst = p.opart + prow * D;
          #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(obase + c * 32, ov);
            tmem_wait_ld();
            if (row_valid) {
              float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
              #pragma unroll
              for (int e = 0; e < 8; ++e)
                d4[e] = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                                    __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
            }
          }
          if (row_valid) p.ml[prow] = make_float2(m_used, l);
        } else {
          const size_t orow = (size_t)it.bh * g.T + g.n_text + (size_t)yq * g.W + xq;
          const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
          __nv_bfloat16* dst = p.o + orow * D;
          #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(obase + c * 32, ov);
            tmem_wait_ld();
            if (row_valid) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
              #pragma unroll
              for (int e = 0; e < 4; ++e)
                d4[e] = make_uint4(
                    pack_bf16x2(__uint_as_float(ov[8 * e + 0]) * inv_l, __uint_as_float(ov[8 * e + 1]) * inv_l),
                    pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * inv_l, __uint_as_float(ov[8 * e + 3]) * inv_l),
                    pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * inv_l, __uint_as_float(ov[8 * e + 5]) * inv_l),
                    pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * inv_l, __uint_as_float(ov[8 * e + 7]) * inv_l));
            }
          }
          if (row_valid) p.lse[orow] = (m_used + __log2f(l)) * 0.69314718055994530942f;
        }
      }
      tc_fence_before();
    }
  softmax_done:;
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Merges the split partials of the text rows: m = max_s m_s, l = sum_s 2^(m_s - m) l_s,
// O = sum_s 2^(m_s - m) O_s / l, LSE = (m + log2 l) ln 2. One warp per text row.
template <int D>
__global__ void clear_fwd_combine_kernel(const FwdParams p) {
  const Geom& g = p.g;
  const int warps_per_block = blockDim.x / 32;
  const long long row_id = (long long)blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row_id >= (long long)g.BH * g.n_text) return;
  const int bh = (int)(row_id / g.n_text);
  const int tq = (int)(row_id % g.n_text);
  float m = -INFINITY;
  for (int s = 0; s < g.S; ++s) {
    const float2 v = p.ml[((size_t)s * g.BH + bh) * g.n_text + tq];
    if (v.y > 0.f) m = fmaxf(m, v.x);
  }
  constexpr int kPer = D / 32;
  float acc[kPer];
  #pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float l = 0.f;
  for (int s = 0; s < g.S; ++s) {
    const size_t prow = ((size_t)s * g.BH + bh) * g.n_text + tq;
    const float2 v = p.ml[prow];
    if (!(v.y > 0.f)) continue;
    const float f = exp2f(v.x - m);
    l += f * v.y;
    const float* src = p.opart + prow * D;
    #pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] += f * src[lane * kPer + e];
  }
  const float inv_l = 1.f / l;
  const size_t orow = (size_t)bh * g.T + tq;
  __nv_bfloat16* dst = p.o + orow * D + lane * kPer;
  #pragma unroll
  for (int e = 0; e < kPer; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv_l);
  if (lane == 0) p.lse[orow] = (m + log2f(l)) * 0.69314718055994530942f;
}

}  // namespace clear
