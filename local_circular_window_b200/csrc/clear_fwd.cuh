// CLEAR attention forward on sm_100a: TMA -> shared memory -> tcgen05.mma (TMEM accumulators)
// -> masked online softmax in registers -> P back into TMEM -> tcgen05.mma for P V.
//
// Semantics (pith.science review of "CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion
// Transformers Up", "Core claim" and "What carries the argument"): every query row takes one
// softmax over the keys the CLEAR mask keeps, scores scaled by 1/sqrt(d); text rows keep every
// key, image rows keep all text keys plus image keys with dx^2 + dy^2 < r^2.
//
// One CTA per SM, persistent over a static list of pair items (clear_sched.cuh). A pair is two
// 128-row query tiles ("halves" A and B: the upper and lower 8 x 16 rectangles of a 16 x 16 image
// block, or two consecutive text tiles) that share every key tile: each K/V tile is loaded once
// and multiplied by whichever halves reach it.
//   warps 0-3  softmax / epilogue of half A (thread t owns query row t = TMEM lane t);
//   warps 4-7  softmax / epilogue of half B;
//   warp 8     TMA producer: Q of both halves once per pair, K tiles into a 2-slot ring, V tiles
//              into a 2-slot ring; it polls the three streams and issues whatever has room;
//   warps 9/10 MMA issuers, one per half: S = Q K^T (TMEM), then, once the softmax has written P
//              over S (bf16, in TMEM), O += P V (A operand from TMEM). The two halves run
//              independently, so one half's products overlap the other half's softmax. A K/V slot
//              is released when both halves are done with it (barriers with two arrivals: a half
//              that skips a tile arrives once the tile has landed, keeping arrivals in phase);
//   warp 11    idle (it completes the third warpgroup, whose registers go to the softmax).
// TMEM columns: S_A [0,128), O_A [128,256), S_B [256,384), O_B [384,512).
// The running max is rescaled lazily: O and l are only rescaled when a row's max grows by more
// than 2^8, which leaves the result exact up to rounding (the final division uses the same max).
#pragma once
#include <cuda_bf16.h>

#include "clear_common.cuh"
#include "clear_sched.cuh"
#include "sm100_ptx.cuh"

namespace clear {

constexpr int kKStages = 2;   // K ring slots (a slot is freed once every Q K^T reading it is done)
constexpr int kVStages = 2;   // V ring slots (freed once every P V reading it is done)
constexpr int kFwdThreads = 384;           // 3 warpgroups: softmax A, softmax B, producer + MMA
// Launched at 168 registers per thread (65536 / 384, rounded to 8). The producer / MMA warpgroup
// drops to kRegsLow and the two softmax warpgroups grow to kRegsHigh:
// 2 * 128 * kRegsHigh + 128 * kRegsLow = 384 * 168.
constexpr uint32_t kRegsLow = 72;
constexpr uint32_t kRegsHigh = 216;
static_assert(2 * 128 * kRegsHigh + 128 * kRegsLow <= 384 * 168, "register split exceeds the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kLastTile = 16;              // mailbox flag: last needed tile of the half in this pair

struct FwdParams {
  Geom g;
  float scale_log2;           // (1/sqrt(d)) * log2(e)
  __nv_bfloat16* o;           // [BH, T, d]
  float* lse;                 // [BH, T]
  float* opart;               // [S, BH, n_text, d] unnormalised partial O of text rows
  float2* ml;                 // [S, BH, n_text] (running max in scaled log2 units, sum)
  long long n_work;           // pair items
};

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = kTile * D * 2;       // one 128-row bf16 tile
  static constexpr int kQ = 0;                           // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kBars = kV + kVStages * kTileBytes;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 1;
  static constexpr int bKFull = 2;                       // + slot
  static constexpr int bKEmpty = bKFull + kKStages;      // + slot
  static constexpr int bVFull = bKEmpty + kKStages;      // + slot
  static constexpr int bVEmpty = bVFull + kVStages;      // + slot
  static constexpr int bSFull = bVEmpty + kVStages;      // + half
  static constexpr int bPFull = bSFull + 2;              // + half
  static constexpr int bODone = bPFull + 2;              // + half
  static constexpr int bInfo = bODone + 2;               // + half: tile descriptor mailbox full
  static constexpr int kNumBars = bInfo + 2;
  static constexpr int kInfo = kBars + kNumBars * 8;     // int4[2]: {kind, a, b, flags | kLastTile}
  static constexpr int kMisc = kInfo + 32;
  static constexpr int kWTab = kMisc + 16;               // int[kMaxRTable] (tile enumeration)
  static constexpr int kHwTab = kWTab + kMaxRTable * 4;  // int16[hw_table_size(r, H)] (masks)
  static constexpr int kFixed = kHwTab + 1024;           // + slack for 1024-byte alignment
  static __host__ __device__ constexpr int alloc_bytes(int hw_entries) { return kFixed + ((hw_entries * 2 + 15) & ~15); }
  static constexpr uint32_t kTmemCols = 512;
  static __host__ __device__ constexpr uint32_t s_col(int half) { return half * 256; }
  static __host__ __device__ constexpr uint32_t o_col(int half) { return half * 256 + 128; }
};

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
  int16_t* hwtab = reinterpret_cast<int16_t*>(smem + L::kHwTab);
  int4* info = reinterpret_cast<int4*>(smem + L::kInfo);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::bQFull], 1);
    mbar_init(&bars[L::bQEmpty], 2);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars[L::bKFull + s], 1);
      mbar_init(&bars[L::bKEmpty + s], 2);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars[L::bVFull + s], 1);
      mbar_init(&bars[L::bVEmpty + s], 2);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars[L::bSFull + h], 1);
      mbar_init(&bars[L::bPFull + h], 128);
      mbar_init(&bars[L::bODone + h], 1);
      mbar_init(&bars[L::bInfo + h], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Half-width table: wtab[dy] = largest dx with dx^2 + dy^2 < r^2 (or -1).
  for (int i = threadIdx.x; i < kMaxRTable; i += blockDim.x) wtab[i] = half_width(g.r, i);
  const int hwn = hw_table_size(g.r, g.H);
  for (int i = threadIdx.x; i < hwn; i += blockDim.x) hwtab[i] = (int16_t)half_width(g.r, i);
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int wtn = imin(g.r, kMaxRTable);
  const long long stride = gridDim.x;
  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    regs_dec<kRegsLow>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q_lin); tma_prefetch_desc(&tm_q_img);
      tma_prefetch_desc(&tm_k_lin); tma_prefetch_desc(&tm_k_img);
      tma_prefetch_desc(&tm_v_lin); tma_prefetch_desc(&tm_v_img);
      long long wq = blockIdx.x;
      uint32_t q_loads = 0;
      long long wk = blockIdx.x, wv = blockIdx.x;
      PairItem itk{}, itv{};
      PairKeyIter kik, kiv;
      KeyTile tk{}, tv{};
      bool kval = wk < p.n_work, vval = kval;
      if (kval) { itk = decode_pair(g, wk); kik.init(g, itk, wtab, wtn); kik.next(&tk); itv = itk; kiv = kik; tv = tk; }
      uint32_t Gk = 0, Gv = 0;
      PollWatchdog wd;
      wd.start();
      while (wq < p.n_work || kval || vval) {
        bool prog = false;
        if (wq < p.n_work && (q_loads == 0 || mbar_test(&bars[L::bQEmpty], (q_loads - 1) & 1))) {
          const PairItem it = decode_pair(g, wq);
          mbar_arrive_expect_tx(&bars[L::bQFull], (it.validB ? 2 : 1) * L::kTileBytes);
          if (it.is_text) {
            load_tile<D>(smem + L::kQ, &tm_q_lin, &tm_q_img, &bars[L::bQFull], kLinear, it.q0, 0, it.bh);
            if (it.validB)
              load_tile<D>(smem + L::kQ + L::kTileBytes, &tm_q_lin, &tm_q_img, &bars[L::bQFull], kLinear,
                           it.q0 + kTile, 0, it.bh);
          } else {
            load_tile<D>(smem + L::kQ, &tm_q_lin, &tm_q_img, &bars[L::bQFull], kRect, it.q0, it.x0, it.bh);
            if (it.validB)
              load_tile<D>(smem + L::kQ + L::kTileBytes, &tm_q_lin, &tm_q_img, &bars[L::bQFull], kRect,
                           it.q0 + kQH, it.x0, it.bh);
          }
          ++q_loads;
          wq += stride;
          prog = true;
        }
        if (kval) {
          const uint32_t ks = Gk % kKStages;
          if (mbar_test(&bars[L::bKEmpty + ks], ((Gk / kKStages) & 1) ^ 1)) {
            mbar_arrive_expect_tx(&bars[L::bKFull + ks], L::kTileBytes);
            load_tile<D>(smem + L::kK + ks * L::kTileBytes, &tm_k_lin, &tm_k_img, &bars[L::bKFull + ks], tk.kind,
                         tk.a, tk.b, itk.bh);
            ++Gk;
            if (!kik.next(&tk)) {
              wk += stride;
              kval = wk < p.n_work;
              if (kval) { itk = decode_pair(g, wk); kik.init(g, itk, wtab, wtn); kik.next(&tk); }
            }
            prog = true;
          }
        }
        if (vval && Gv < Gk) {
          const uint32_t vs = Gv % kVStages;
          if (mbar_test(&bars[L::bVEmpty + vs], ((Gv / kVStages) & 1) ^ 1)) {
            mbar_arrive_expect_tx(&bars[L::bVFull + vs], L::kTileBytes);
            load_tile<D>(smem + L::kV + vs * L::kTileBytes, &tm_v_lin, &tm_v_img, &bars[L::bVFull + vs], tv.kind,
                         tv.a, tv.b, itv.bh);
            ++Gv;
            if (!kiv.next(&tv)) {
              wv += stride;
              vval = wv < p.n_work;
              if (vval) { itv = decode_pair(g, wv); kiv.init(g, itv, wtab, wtn); kiv.next(&tv); }
            }
            prog = true;
          }
        }
        if (!wd.tick(prog, abort_flag, kDevTimeoutTmaEmpty)) break;
      }
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------------ MMA issuers (one per half)
    regs_dec<kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const int h = warp - 9;
      const int need_bit = h == 0 ? kNeedA : kNeedB;
      const uint32_t q_addr = smem_u32(smem + L::kQ + h * L::kTileBytes);
      const uint32_t s_tm = tmem + L::s_col(h);
      const uint32_t o_tm = tmem + L::o_col(h);
      uint32_t G = 0, nq = 0, items = 0;
      for (long long w = blockIdx.x; w < p.n_work; w += stride, ++items) {
        const PairItem it = decode_pair(g, w);
        int nu, na, nb;
        count_pair_tiles(g, it, wtab, wtn, &nu, &na, &nb);
        const int n = h == 0 ? na : nb;
        if (n == 0) {  // this half has no queries in the pair: release Q once it has landed
          if (!mbar_wait(&bars[L::bQFull], items & 1, abort_flag, kDevTimeoutMma)) goto mma_done;
          mbar_arrive(&bars[L::bQEmpty]);
        }
        PairKeyIter ki;
        ki.init(g, it, wtab, wtn);
        KeyTile t;
        int j = 0;
        for (; ki.next(&t); ++G) {
          const uint32_t ks = G % kKStages, kph = (G / kKStages) & 1;
          const uint32_t vs = G % kVStages, vph = (G / kVStages) & 1;
          if (!(t.flags & need_bit)) {
            // Skipped tile: arrive on its empty barriers once it has landed (so the arrival
            // belongs to this use of the slot).
            if (!mbar_wait(&bars[L::bKFull + ks], kph, abort_flag, kDevTimeoutMma)) goto mma_done;
            mbar_arrive(&bars[L::bKEmpty + ks]);
            if (!mbar_wait(&bars[L::bVFull + vs], vph, abort_flag, kDevTimeoutMma)) goto mma_done;
            mbar_arrive(&bars[L::bVEmpty + vs]);
            continue;
          }
          // Hand the tile to this half's softmax (its previous descriptor was consumed before it
          // signalled the previous P, which this thread has waited for).
          info[h] = make_int4(t.kind, t.a, t.b, t.flags | (j == n - 1 ? kLastTile : 0));
          mbar_arrive(&bars[L::bInfo + h]);
          if (j == 0 && !mbar_wait(&bars[L::bQFull], items & 1, abort_flag, kDevTimeoutMma)) goto mma_done;
          if (!mbar_wait(&bars[L::bKFull + ks], kph, abort_flag, kDevTimeoutMma)) goto mma_done;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + L::kK + ks * L::kTileBytes);
          #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            umma_ss(s_tm, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
                    idesc_qk, kk > 0);
          }
          umma_commit(&bars[L::bSFull + h]);
          umma_commit(&bars[L::bKEmpty + ks]);
          if (j == n - 1) umma_commit(&bars[L::bQEmpty]);
          // O += P V once the softmax has written P over S
          if (!mbar_wait(&bars[L::bPFull + h], nq & 1, abort_flag, kDevTimeoutMma)) goto mma_done;
          if (!mbar_wait(&bars[L::bVFull + vs], vph, abort_flag, kDevTimeoutMma)) goto mma_done;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(smem + L::kV + vs * L::kTileBytes);
          #pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(o_tm, s_tm + kk * 8, smem_desc_sw128(v_addr + kk * 2048, kHalfBytes, 1024), idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars[L::bVEmpty + vs]);
          if (j == n - 1) umma_commit(&bars[L::bODone + h]);
          ++nq;
          ++j;
        }
      }
    mma_done:;
    }
    __syncwarp();
  } else if (warp == 11) {
    regs_dec<kRegsLow>();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    regs_inc<kRegsHigh>();
    const int half = warp >> 2;              // 0: A, 1: B
    const int row = threadIdx.x & 127;       // TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_tm = tmem + lane_base + L::s_col(half);
    const uint32_t o_tm = tmem + lane_base + L::o_col(half);
    const int full_bit = half == 0 ? kFullA : kFullB;
    uint32_t nq = 0, n_out = 0;
    const float sl2 = p.scale_log2;
    for (long long w = blockIdx.x; w < p.n_work; w += stride) {
      const PairItem it = decode_pair(g, w);
      if (half == 1 && !it.validB) continue;
      int yq = 0, xq = 0, tq = 0;
      bool row_valid;
      if (it.is_text) {
        tq = it.q0 + half * kTile + row;
        row_valid = tq < g.n_text;
      } else {
        yq = it.q0 + half * kQH + (row >> 4);
        xq = it.x0 + (row & 15);
        row_valid = (yq < g.H) && (xq < g.W);
      }
      float m_used = -INFINITY;  // running max, scaled log2 units
      float l = 0.f;
      int j = 0;
      bool last = false;
      while (!last) {
        if (!mbar_wait(&bars[L::bInfo + half], nq & 1, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
        const int4 ti = info[half];
        KeyTile t;
        t.kind = ti.x;
        t.a = ti.y;
        t.b = ti.z;
        t.flags = ti.w;
        last = (ti.w & kLastTile) != 0;
        if (!mbar_wait(&bars[L::bSFull + half], nq & 1, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
        tc_fence_after();
        float s[kTile];
        {
          uint32_t sr[4][32];
          tmem_ld32(s_tm + 0, sr[0]);
          tmem_ld32(s_tm + 32, sr[1]);
          tmem_ld32(s_tm + 64, sr[2]);
          tmem_ld32(s_tm + 96, sr[3]);
          tmem_wait_ld();
          #pragma unroll
          for (int c = 0; c < kTile; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        // ---- mask (branch-free selects; full tiles skip it)
        if (!(t.flags & full_bit)) {
          if (t.kind == kLinear) {
            const int lim = t.b;
            #pragma unroll
            for (int c = 0; c < kTile; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
          } else {
            // keep bits: word q holds key rows 2q (bits 0-15) and 2q+1 (bits 16-31)
            uint32_t keep[kKH / 2];
            #pragma unroll
            for (int q = 0; q < kKH / 2; ++q) {
              int lo0, hi0, lo1, hi1;
              row_range_tab(g, hwtab, hwn, yq, xq, t.a + 2 * q, t.b, &lo0, &hi0);
              row_range_tab(g, hwtab, hwn, yq, xq, t.a + 2 * q + 1, t.b, &lo1, &hi1);
              const int n0 = imax(hi0 - lo0 + 1, 0), n1 = imax(hi1 - lo1 + 1, 0);
              keep[q] = (((1u << n0) - 1u) << (lo0 & 15)) | ((((1u << n1) - 1u) << (lo1 & 15)) << 16);
            }
            #pragma unroll
            for (int c = 0; c < kTile; ++c)
              s[c] = (keep[c >> 5] & (1u << (c & 31))) ? s[c] : -INFINITY;
          }
        }
        // ---- tile max (8 independent chains of 3-input maxima)
        float mx[8];
        #pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmax3(s[u], s[u + 8], s[u + 16]);
        #pragma unroll
        for (int c = 24; c < kTile - 8; c += 16) {
          #pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmax3(mx[u], s[c + u], s[c + 8 + u]);
        }
        #pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], s[kTile - 8 + u]);
        const float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
        const float mt_scaled = mt * sl2;
        // S_j being ready means every earlier product of this CTA has completed, including this
        // half's P V of tile j-1: O may be rescaled in place.
        float alpha = 1.f;
        bool need_rescale = false;
        if (m_used == -INFINITY) {
          m_used = mt_scaled;  // nothing accumulated yet (l == 0)
        } else if (mt_scaled > m_used + kRescaleThreshold) {
          alpha = ex2_approx(m_used - mt_scaled);
          l *= alpha;
          m_used = mt_scaled;
          need_rescale = true;
        }
        if (j > 0 && __any_sync(0xffffffffu, need_rescale)) {
          #pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(o_tm + c * 32, ov);
            tmem_wait_ld();
            #pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(o_tm + c * 32, ov);
          }
        }
        // ---- P = 2^(s * scale_log2 - m), row sum, bf16 pairs written over S in TMEM
        const float base = (m_used == -INFINITY) ? 0.f : m_used;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        #pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t pw[32];
          #pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int c = hc * 64 + 2 * q;
            const float e0 = ex2_approx(fmaf(s[c], sl2, -base));
            const float e1 = ex2_approx(fmaf(s[c + 1], sl2, -base));
            acc[(2 * q) & 7] += e0;
            acc[(2 * q + 1) & 7] += e1;
            pw[q] = pack_bf16x2(e0, e1);
          }
          tmem_st32(s_tm + hc * 32, pw);
        }
        l += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[L::bPFull + half]);
        ++nq;
        ++j;
      }
      // ---- epilogue: wait for this half's last P V, then write O / l (or the split partial)
      if (j == 0) continue;
      if (!mbar_wait(&bars[L::bODone + half], n_out & 1, abort_flag, kDevTimeoutSoftmax)) goto softmax_done;
      ++n_out;
      tc_fence_after();
      if (it.is_text) {
        const size_t prow = ((size_t)it.split * g.BH + it.bh) * g.n_text + (row_valid ? tq : 0);
        float* dst = p.opart + prow * D;
        #pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(o_tm + c * 32, ov);
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
          tmem_ld32(o_tm + c * 32, ov);
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
      // The next pair's first P V overwrites O; it waits for this half's next P, which is
      // signalled after these TMEM reads.
      tc_fence_before();
    }
  softmax_done:;
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
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
