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
// block, or two consecutive text tiles) that share every 128-key tile: each K/V tile is loaded once
// and multiplied by whichever halves reach it. Every product is a full-width tensor-core step:
// S = Q K^T is M128 N128 (K = d), O += P V is M128 N=d (K = 128 keys), P read from TMEM.
//   warps 0-3   softmax / epilogue of half A (thread t owns query row t = TMEM lane t);
//   warps 4-7   softmax / epilogue of half B;
//   warp 8      TMA producer: Q of each half (its own buffer, reloaded as soon as that half has
//               issued its last score product of the pair), K and V tiles into 2-slot rings. It
//               enumerates each union tile once, publishes its descriptor (kind, origin, per-half
//               need / full bits, last-of-pair and last-needed-by-half bits, head) in a 16-entry
//               shared ring that the V stream and both MMA issuers read, and posts each half's
//               tiles (and the end of each pair) to that half's softmax through a 4-slot mailbox;
//   warps 9/10  MMA issuers, one per half, in a fixed order per needed tile:
//               S = Q K^T -> (softmax writes P over S) -> O += P V -> next tile's S. With a single S
//               buffer per half the two halves alternate on the tensor pipe: one half's P V and
//               next S run while the other half's softmax works. Tiles a half does not need are
//               still observed and released by that half, so each half sees every phase of every
//               ring slot in order, which keeps the parity-based waits exact;
//   warp 11     idle (it completes the third warpgroup, whose registers go to the softmax).
// TMEM columns of half h: S (fp32) / P (bf16 pairs, first 64 columns) [256h, 256h+128),
// O [256h+128, 256h+128+d). Products issued by one thread run in order, so an S product issued
// after the P V product that reads the same columns never overwrites P early, and the S-full
// commit of tile j also covers the P V of tile j-1 (the softmax may rescale O once S_j is ready).
// The running max is rescaled lazily: O and l are only rescaled when a row's max grows by more
// than 2^8, which leaves the result exact up to rounding (the final division uses the same max).
#pragma once
#include <cuda_bf16.h>

#include "clear_common.cuh"
#include "clear_sched.cuh"
#include "sm100_ptx.cuh"

namespace clear {

constexpr int kKStages = 2;   // K ring slots (128-key tiles)
constexpr int kVStages = 2;   // V ring slots
constexpr int kFwdThreads = 384;           // 3 warpgroups: softmax A, softmax B, producer + MMA
// Launched at 168 registers per thread (65536 / 384, rounded to 8). The producer / MMA warpgroup
// drops to kRegsLow and the two softmax warpgroups grow to kRegsHigh:
// 2 * 128 * kRegsHigh + 128 * kRegsLow <= 384 * 168.
constexpr uint32_t kRegsLow = 88;
constexpr uint32_t kRegsHigh = 208;
static_assert(2 * 128 * kRegsHigh + 128 * kRegsLow <= 384 * 168, "register split exceeds the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kTileRing = 16;              // union tile descriptors in flight (producer -> others)
// Descriptor ring entry x: kind | flags << 4 | these bits.
constexpr int kRingLastUnion = 1 << 12;    // last union tile of the pair
constexpr int kRingLastA = 1 << 13;        // last tile of the pair that half A needs
constexpr int kRingLastB = 1 << 14;        // last tile of the pair that half B needs
constexpr int kMsgSlots = 4;               // mailbox slots per half (producer -> softmax)
// Mailbox message kinds (producer -> softmax); tiles use their KeyKind (kLinear / kRect).
constexpr int kMsgEndPair = 2;             // the half's last tile of the current pair was posted
constexpr int kMsgEndAll = 3;              // no more pairs for this CTA

struct FwdParams {
  Geom g;
  float scale_log2;           // (1/sqrt(d)) * log2(e)
  __nv_bfloat16* o;           // [BH, T, d]
  float* lse;                 // [BH, T]
  float* opart;               // [fS, BH, n_text, d] unnormalised partial O of text rows
  float2* ml;                 // [fS, BH, n_text] (running max in scaled log2 units, sum)
  long long n_work;           // pair items
  int wide_o, wide_part;      // o / opart are 32-byte aligned: the epilogue may store 32 bytes at once
};

// Packed fp32 pairs (one 64-bit register, low word first): fma.rn.f32x2 / add.rn.f32x2 do two
// correctly rounded fp32 operations per instruction, with the same results as two fmaf / fadd.
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float f32x2_lo(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo;
}
__device__ __forceinline__ float f32x2_hi(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return hi;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x on the FMA pipe for two packed fp32 values, to take part of the exponentials off the
// MUFU unit (16 results per clock per SM, as many clocks per tile as the tensor core needs).
// Range reduction: x = j + f with j = round-to-nearest(x), |f| <= 1/2; j is read from the low
// mantissa bits of x + 1.5 * 2^23. 2^f is a degree-3 polynomial whose coefficients minimise the
// maximum relative error on [-1/2, 1/2] (Remez exchange; fit_exp2_poly.py next to this file),
// 7.5e-5 (2^-13.7), far below the bf16 rounding P gets next. 2^j is added to the exponent field
// (j * 2^23 added to the bit pattern). x is clamped below at -125 so that the result stays a
// normal float: a masked score (-inf) gives 2^-125 ~ 2.4e-38 instead of 0, which changes no
// sum or product at fp32 / bf16 precision.
constexpr float kExp2C0 = 0.99992806f, kExp2C1 = 0.69326097f, kExp2C2 = 0.24261113f, kExp2C3 = 0.05517167f;
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x) {
  const float x0 = fmaxf(f32x2_lo(x), -125.f), x1 = fmaxf(f32x2_hi(x), -125.f);
  const uint64_t xc = f32x2_pack(x0, x1);
  const uint64_t t = f32x2_add(xc, f32x2_pack(12582912.f, 12582912.f));    // 1.5 * 2^23: rounds to integer
  const uint64_t j = f32x2_add(t, f32x2_pack(-12582912.f, -12582912.f));   // round(x), exact
  const uint64_t f = f32x2_fma(j, f32x2_pack(-1.f, -1.f), xc);             // x - round(x), exact
  uint64_t q = f32x2_fma(f, f32x2_pack(kExp2C3, kExp2C3), f32x2_pack(kExp2C2, kExp2C2));
  q = f32x2_fma(q, f, f32x2_pack(kExp2C1, kExp2C1));
  q = f32x2_fma(q, f, f32x2_pack(kExp2C0, kExp2C0));
  const uint32_t r0 = __float_as_uint(f32x2_lo(q)) + (__float_as_uint(f32x2_lo(t)) << 23);
  const uint32_t r1 = __float_as_uint(f32x2_hi(q)) + (__float_as_uint(f32x2_hi(t)) << 23);
  return f32x2_pack(__uint_as_float(r0), __uint_as_float(r1));
}

// Which column pairs of each 32-column chunk take the polynomial exp2 instead of MUFU ex2
// (bit q: columns 2q and 2q + 1).
#ifndef CLEAR_FWD_EXP2_POLY_PAIRS
#define CLEAR_FWD_EXP2_POLY_PAIRS 0x0000u
#endif
// 1: P = 2^x through the MUFU's packed bf16 form: x rounded to bf16, two results per operation,
// already the bf16 pair the P V product reads; the row sum adds those bf16 values.
#ifndef CLEAR_FWD_EXP_BF16X2
#define CLEAR_FWD_EXP_BF16X2 0
#endif

// One 32-byte global store (the address must be 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* ptr, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t a4, uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

template <int D>
struct FwdLayout {
  static constexpr int kQTileBytes = kTile * D * 2;      // one 128-row bf16 query tile
  static constexpr int kKVTileBytes = kFChunk * D * 2;   // one 128-key bf16 tile
  static constexpr int kBlock = kTile * 128;             // 128 rows x 64 elements (128B-swizzled)
  static constexpr int kQ = 0;                           // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kQTileBytes;
  static constexpr int kV = kK + kKStages * kKVTileBytes;
  static constexpr int kBars = kV + kVStages * kKVTileBytes;
  // barrier indices
  static constexpr int bQFull = 0;                       // + half
  static constexpr int bQEmpty = bQFull + 2;             // + half
  static constexpr int bKFull = bQEmpty + 2;             // + slot
  static constexpr int bKEmpty = bKFull + kKStages;      // + slot
  static constexpr int bVFull = bKEmpty + kKStages;      // + slot
  static constexpr int bVEmpty = bVFull + kVStages;      // + slot
  static constexpr int bSFull = bVEmpty + kVStages;      // + half: S = Q K^T of the half's tile ready
  static constexpr int bPFull = bSFull + 2;              // + half: P written over S
  static constexpr int bMsgFull = bPFull + 2;            // + kMsgSlots * half + slot: mailbox message posted
  static constexpr int bMsgEmpty = bMsgFull + 2 * kMsgSlots;  // + kMsgSlots * half + slot: mailbox slot read
  static constexpr int bODone = bMsgEmpty + 2 * kMsgSlots;    // + half: last P V of the half's pair done
  static constexpr int bExpDone = bODone + 2;            // + half: the half's exponentials of a shared tile done
  static constexpr int kNumBars = bExpDone + 2;
  static constexpr int kMsg = kBars + kNumBars * 8;      // int4[2][kMsgSlots] mailbox: {kind, a, b, flags | ordinal << 8}
  static constexpr int kRing = kMsg + 2 * kMsgSlots * 16;  // int4[kTileRing]: {x bits, a, b, bh}
  static constexpr int kMisc = kRing + kTileRing * 16;
  static constexpr int kWTab = kMisc + 16;               // int[kMaxRTable] (tile enumeration)
  static constexpr int kHwTab = kWTab + kMaxRTable * 4;  // int16[hw_table_size(r, H)] (masks)
  static constexpr int kFixed = kHwTab + 1024;           // + slack for 1024-byte alignment
  static __host__ __device__ constexpr int alloc_bytes(int hw_entries) { return kFixed + ((hw_entries * 2 + 15) & ~15); }
  static constexpr uint32_t kTmemCols = 512;
  static __host__ __device__ constexpr uint32_t s_col(int half) { return half * 256; }
  static __host__ __device__ constexpr uint32_t o_col(int half) { return half * 256 + 128; }
};

// Tiles of a pair each half needs (the producer's last-needed bits).
__device__ __forceinline__ void pair_need_counts(const Geom& g, const PairItem& it, const int* wtab, int wtn, int* na,
                                              int* nb) {
  int nu;
  count_pair_tiles(g, it, wtab, wtn, &nu, na, nb);
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
  int16_t* hwtab = reinterpret_cast<int16_t*>(smem + L::kHwTab);
  int4* msg = reinterpret_cast<int4*>(smem + L::kMsg);
  int4* ring = reinterpret_cast<int4*>(smem + L::kRing);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Geom& g = p.g;

  if (threadIdx.x == 0) {
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars[L::bQFull + h], 1);
      mbar_init(&bars[L::bQEmpty + h], 1);
      mbar_init(&bars[L::bSFull + h], 1);
      mbar_init(&bars[L::bPFull + h], 128);
      mbar_init(&bars[L::bODone + h], 1);
      mbar_init(&bars[L::bExpDone + h], 128);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars[L::bKFull + s], 1);
      mbar_init(&bars[L::bKEmpty + s], 2);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars[L::bVFull + s], 1);
      mbar_init(&bars[L::bVEmpty + s], 2);
    }
    for (int i = 0; i < 2 * kMsgSlots; ++i) {
      mbar_init(&bars[L::bMsgFull + i], 1);
      mbar_init(&bars[L::bMsgEmpty + i], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Half-width tables: wtab[dy] (tile enumeration, first kMaxRTable rows) and the int16 table
  // hwtab[dy] for every |dy| < min(r, H) (masks).
  for (int i = threadIdx.x; i < kMaxRTable; i += blockDim.x) wtab[i] = half_width(g.r, i, g.window);
  const int hwn = hw_table_size(g.r, g.H);
  for (int i = threadIdx.x; i < hwn; i += blockDim.x) hwtab[i] = (int16_t)half_width(g.r, i, g.window);
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

  // The producer and issuer warps run their loops with all 32 lanes (warp-uniform state, barrier
  // results combined by votes) and issue each TMA copy, tcgen05 product or commit from one elected
  // lane: operands that are warp-uniform can then stay in uniform registers.
  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    regs_dec<kRegsLow>();
    if (elect_one()) {
      tma_prefetch_desc(&tm_q_lin); tma_prefetch_desc(&tm_q_img);
      tma_prefetch_desc(&tm_k_lin); tma_prefetch_desc(&tm_k_img);
      tma_prefetch_desc(&tm_v_lin); tma_prefetch_desc(&tm_v_img);
    }
    __syncwarp();
    // Q stream of each half: pair index and loads so far.
    long long wq0 = blockIdx.x, wq1 = blockIdx.x;
    uint32_t nq0 = 0, nq1 = 0;
    // K stream: the current union tile and a one-tile lookahead (for the last-of-pair bit), and
    // the tiles each half still needs in the pair (for its last-needed bit).
    long long wk = blockIdx.x;
    PairItem itk{};
    PairKeyIter kik;
    KeyTile tcur{}, tnext{};
    int remA = 0, remB = 0;
    bool kval = wk < p.n_work, next_in_pair = false;
    if (kval) {
      itk = decode_pair(g, wk);
      pair_need_counts(g, itk, wtab, wtn, &remA, &remB);
      kik.init(g, itk, wtab, wtn);
      kik.next(&tcur);
      next_in_pair = kik.next(&tnext);
    }
    uint32_t Gk = 0, Gv = 0;
    uint32_t nm0 = 0, nm1 = 0;   // mailbox messages posted to each half
    uint32_t pk = 0;             // pair ordinal of the K stream (this CTA's pairs, in order)
    bool end0 = false, end1 = false;
    // Slot n of half h's mailbox is free once the softmax has read the message kMsgSlots posts back.
    auto slot_free = [&](int h, uint32_t n) -> bool {
      return mbar_test(&bars[L::bMsgEmpty + kMsgSlots * h + n % kMsgSlots], ((n / kMsgSlots) & 1) ^ 1);
    };
    auto post = [&](int h, uint32_t n, int4 m) {  // called by the elected lane
      msg[kMsgSlots * h + n % kMsgSlots] = m;
      mbar_arrive(&bars[L::bMsgFull + kMsgSlots * h + n % kMsgSlots]);
    };
    PollWatchdog wd;
    wd.start();
    while (wq0 < p.n_work || wq1 < p.n_work || kval || Gv < Gk || !end0 || !end1) {
      bool prog = false;
      #pragma unroll
      for (int h = 0; h < 2; ++h) {
        long long& wq = h ? wq1 : wq0;
        uint32_t& nq = h ? nq1 : nq0;
        if (wq < p.n_work &&
            (nq == 0 || __any_sync(0xffffffffu, mbar_test(&bars[L::bQEmpty + h], (nq - 1) & 1)))) {
          const PairItem it = decode_pair(g, wq);
          if (elect_one()) {
            if (h == 0 || it.validB) {
              mbar_arrive_expect_tx(&bars[L::bQFull + h], L::kQTileBytes);
              if (it.is_text)
                load_tile<D>(smem + L::kQ + h * L::kQTileBytes, &tm_q_lin, &tm_q_img, &bars[L::bQFull + h], kLinear,
                             it.q0 + h * kTile, 0, it.bh);
              else
                load_tile<D>(smem + L::kQ + h * L::kQTileBytes, &tm_q_lin, &tm_q_img, &bars[L::bQFull + h], kRect,
                             it.q0 + h * kQH, it.x0, it.bh);
            } else {
              mbar_arrive(&bars[L::bQFull + h]);  // no query rows: the phase completes empty
            }
          }
          __syncwarp();
          ++nq;
          wq += stride;
          prog = true;
        }
      }
      if (kval && Gk - Gv < (uint32_t)kTileRing) {
        const uint32_t ks = Gk % kKStages;
        const bool needA = tcur.flags & kNeedA, needB = tcur.flags & kNeedB;
        const bool lastA = needA && remA == 1, lastB = needB && remB == 1;
        // The K slot and the mailbox slots this tile's messages take (the tile, and the end of the
        // pair after a half's last tile) must all be free.
        bool ready = mbar_test(&bars[L::bKEmpty + ks], ((Gk / kKStages) & 1) ^ 1);
        if (needA) ready = ready && slot_free(0, nm0) && (!lastA || slot_free(0, nm0 + 1));
        if (needB) ready = ready && slot_free(1, nm1) && (!lastB || slot_free(1, nm1 + 1));
        if (__all_sync(0xffffffffu, ready)) {
          int bits = tcur.kind | (tcur.flags << 4) | (next_in_pair ? 0 : kRingLastUnion);
          if (lastA) bits |= kRingLastA;
          if (lastB) bits |= kRingLastB;
          remA -= needA ? 1 : 0;
          remB -= needB ? 1 : 0;
          if (elect_one()) {
            const int4 m = make_int4(tcur.kind, tcur.a, tcur.b, tcur.flags | (int)(pk << 8));
            if (needA) post(0, nm0, m);
            if (lastA) post(0, nm0 + 1, make_int4(kMsgEndPair, 0, 0, 0));
            if (needB) post(1, nm1, m);
            if (lastB) post(1, nm1 + 1, make_int4(kMsgEndPair, 0, 0, 0));
            // Publish the descriptor before the load: the K barrier's completion makes it visible.
            ring[Gk % kTileRing] = make_int4(bits, tcur.a, tcur.b, itk.bh);
            mbar_arrive_expect_tx(&bars[L::bKFull + ks], L::kKVTileBytes);
            load_tile<D>(smem + L::kK + ks * L::kKVTileBytes, &tm_k_lin, &tm_k_img, &bars[L::bKFull + ks], tcur.kind,
                         tcur.a, tcur.b, itk.bh);
          }
          __syncwarp();
          nm0 += (needA ? 1 : 0) + (lastA ? 1 : 0);
          nm1 += (needB ? 1 : 0) + (lastB ? 1 : 0);
          ++Gk;
          if (next_in_pair) {
            tcur = tnext;
            next_in_pair = kik.next(&tnext);
          } else {
            ++pk;
            wk += stride;
            kval = wk < p.n_work;
            if (kval) {
              itk = decode_pair(g, wk);
              pair_need_counts(g, itk, wtab, wtn, &remA, &remB);
              kik.init(g, itk, wtab, wtn);
              kik.next(&tcur);
              next_in_pair = kik.next(&tnext);
            }
          }
          prog = true;
        }
      }
      if (!kval && (!end0 || !end1)) {  // every tile posted: tell both softmax warpgroups to stop
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
          bool& done = h ? end1 : end0;
          const uint32_t n = h ? nm1 : nm0;
          if (!done && __all_sync(0xffffffffu, slot_free(h, n))) {
            if (elect_one()) post(h, n, make_int4(kMsgEndAll, 0, 0, 0));
            __syncwarp();
            done = true;
            prog = true;
          }
        }
      }
      if (Gv < Gk) {
        const uint32_t vs = Gv % kVStages;
        if (__any_sync(0xffffffffu, mbar_test(&bars[L::bVEmpty + vs], ((Gv / kVStages) & 1) ^ 1))) {
          if (elect_one()) {
            const int4 e = ring[Gv % kTileRing];
            mbar_arrive_expect_tx(&bars[L::bVFull + vs], L::kKVTileBytes);
            load_tile<D>(smem + L::kV + vs * L::kKVTileBytes, &tm_v_lin, &tm_v_img, &bars[L::bVFull + vs], e.x & 15,
                         e.y, e.z, e.w);
          }
          __syncwarp();
          ++Gv;
          prog = true;
        }
      }
      const bool alive = wd.tick(prog, abort_flag, kDevTimeoutTmaEmpty, 1, (int)Gk, (int)Gv, (int)(nm0 | (nm1 << 16)));
      if (!__all_sync(0xffffffffu, alive)) break;
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------------ MMA issuers (one per half)
    regs_dec<kRegsLow>();
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kFChunk, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    const int h = warp - 9;
    const int need_bit = h == 0 ? kNeedA : kNeedB;
    const int last_bit = h == 0 ? kRingLastA : kRingLastB;
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t s_tm = tm + L::s_col(h);
    const uint32_t o_tm = tm + L::o_col(h);
    // Shared-memory matrix descriptors, advanced per 16-element K step with plain adds.
    const uint64_t qdesc = smem_desc_sw128(smem_u32(smem + L::kQ + h * L::kQTileBytes), 16, 1024);
    const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
    const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + L::kV), L::kBlock, 1024);
    const uint32_t n_pairs = (uint32_t)((p.n_work - blockIdx.x + stride - 1) / stride);
    uint32_t G = 0;     // union tiles observed
    uint32_t nS = 0;    // tiles this half multiplied (S / P phases)
    bool ok = true;
    // Bounded wait by every lane; the warp goes on only if all of them saw the phase.
    auto wait_all = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
      const bool r = mbar_wait(bar, parity, abort_flag, kDevTimeoutMma, site, (int)G, (int)nS);
      return __all_sync(0xffffffffu, r);
    };
    for (uint32_t pair = 0; ok && pair < n_pairs; ++pair) {
      // Every half observes every Q phase (a half without query rows gets an empty phase).
      if (!wait_all(&bars[L::bQFull + h], pair & 1, 4 + h)) {
        ok = false;
        break;
      }
      bool had = false, q_released = false, o_done = false;
      while (true) {
        const uint32_t ks = G % kKStages, vs = G % kVStages;
        if (!wait_all(&bars[L::bKFull + ks], (G / kKStages) & 1, 6 + h)) {
          ok = false;
          break;
        }
        const int ex = __shfl_sync(0xffffffffu, ring[G % kTileRing].x, 0);
        const int flags = (ex >> 4) & 255;
        const bool last_union = (ex & kRingLastUnion) != 0;
        if (flags & need_bit) {
          const bool last_h = (ex & last_bit) != 0;
          const uint64_t kd = kdesc0 + (uint64_t)((ks * L::kKVTileBytes) >> 4);
          if (elect_one()) {
            tc_fence_after();
            #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * L::kBlock + (kk & 3) * 32) >> 4;
              umma_ss(s_tm, qdesc + off, kd + off, idesc_qk, kk > 0);
            }
            umma_commit(&bars[L::bSFull + h]);
            umma_commit(&bars[L::bKEmpty + ks]);
            if (last_h) umma_commit(&bars[L::bQEmpty + h]);  // the half's Q may be reloaded for its next pair
          }
          __syncwarp();
          q_released |= last_h;
          if (!wait_all(&bars[L::bVFull + vs], (G / kVStages) & 1, 8 + h) ||
              !wait_all(&bars[L::bPFull + h], nS & 1, 18 + h)) {
            ok = false;
            break;
          }
          const uint64_t vd = vdesc0 + (uint64_t)((vs * L::kKVTileBytes) >> 4);
          if (elect_one()) {
            tc_fence_after();
            #pragma unroll
            for (int kk = 0; kk < kFChunk / 16; ++kk)
              umma_ts(o_tm, s_tm + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv, (had || kk > 0) ? 1u : 0u);
            umma_commit(&bars[L::bVEmpty + vs]);
            if (last_h) umma_commit(&bars[L::bODone + h]);
          }
          __syncwarp();
          had = true;
          ++nS;
          o_done |= last_h;
        } else {
          // Not needed by this half: observed and released (after its V load, so the slot's
          // phases stay in step with the other half).
          if (elect_one()) mbar_arrive(&bars[L::bKEmpty + ks]);
          __syncwarp();
          if (!wait_all(&bars[L::bVFull + vs], (G / kVStages) & 1, 8 + h)) {
            ok = false;
            break;
          }
          if (elect_one()) mbar_arrive(&bars[L::bVEmpty + vs]);
          __syncwarp();
        }
        ++G;
        if (last_union) break;
      }
      if (!ok) break;
      if (!q_released) {
        if (elect_one()) {
          if (had)
            umma_commit(&bars[L::bQEmpty + h]);
          else
            mbar_arrive(&bars[L::bQEmpty + h]);
        }
        __syncwarp();
      }
      if (had && !o_done) {  // not reached: the producer marks every half's last tile of a pair
        if (elect_one()) umma_commit(&bars[L::bODone + h]);
        __syncwarp();
      }
    }
  } else if (warp == 11) {
    regs_dec<kRegsLow>();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    regs_inc<kRegsHigh>();
    const int half = warp >> 2;              // 0: A, 1: B
    const int row = threadIdx.x & 127;       // TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t o_tm = tmem + lane_base + L::o_col(half);
    const uint32_t s_tm = tmem + lane_base + L::s_col(half);
    const int full_bit = half == 0 ? kFullA : kFullB;
    uint32_t nq = 0, n_out = 0, nmsg = 0;
    uint32_t nboth = 0;  // tiles both halves multiply, seen so far (exponential-phase turns)
    const float sl2 = p.scale_log2;
    // Per-pair state, set up at the pair's first tile.
    PairItem it{};
    int yq = 0, xq = 0, tq = 0;
    int yc = 0, xc = 0;  // the window's centre: (yq, xq), clamped inside the grid for shifted windows
    bool row_valid = false;
    float m_used = -INFINITY;  // running max, scaled log2 units
    float l = 0.f;
    int j = 0;
    while (true) {
      const uint32_t ms = nmsg % kMsgSlots;
      if (!mbar_wait(&bars[L::bMsgFull + kMsgSlots * half + ms], (nmsg / kMsgSlots) & 1, abort_flag,
                     kDevTimeoutSoftmax, 10 + half, (int)nmsg, j))
        goto softmax_done;
      const int4 mv = msg[kMsgSlots * half + ms];
      mbar_arrive(&bars[L::bMsgEmpty + kMsgSlots * half + ms]);
      ++nmsg;
      if (mv.x == kMsgEndAll) break;
      if (mv.x == kMsgEndPair) {
        // ---- epilogue: wait for this half's last P V, then write O / l (or the split partial)
        if (!mbar_wait(&bars[L::bODone + half], n_out & 1, abort_flag, kDevTimeoutSoftmax, 16 + half, (int)nq,
                       (int)n_out))
          goto softmax_done;
        ++n_out;
        tc_fence_after();
        if (it.is_text) {
          const size_t prow = ((size_t)it.split * g.BH + it.bh) * g.n_text + (row_valid ? tq : 0);
          float* dst = p.opart + prow * D;
          // Two TMEM loads per wait; each row's run is written 32 (or 16) bytes at a time.
          #pragma unroll
          for (int c = 0; c < D / 32; c += 2) {
            uint32_t ov[2][32];
            tmem_ld32(o_tm + c * 32, ov[0]);
            tmem_ld32(o_tm + c * 32 + 32, ov[1]);
            tmem_wait_ld();
            if (row_valid) {
              #pragma unroll
              for (int u = 0; u < 2; ++u) {
                float* d = dst + (c + u) * 32;
                if (p.wide_part) {
                  #pragma unroll
                  for (int e = 0; e < 4; ++e)
                    st_global_v8(d + e * 8, ov[u][8 * e], ov[u][8 * e + 1], ov[u][8 * e + 2], ov[u][8 * e + 3],
                                 ov[u][8 * e + 4], ov[u][8 * e + 5], ov[u][8 * e + 6], ov[u][8 * e + 7]);
                } else {
                  float4* d4 = reinterpret_cast<float4*>(d);
                  #pragma unroll
                  for (int e = 0; e < 8; ++e)
                    d4[e] = make_float4(__uint_as_float(ov[u][4 * e]), __uint_as_float(ov[u][4 * e + 1]),
                                        __uint_as_float(ov[u][4 * e + 2]), __uint_as_float(ov[u][4 * e + 3]));
                }
              }
            }
          }
          if (row_valid) p.ml[prow] = make_float2(m_used, l);
        } else {
          const size_t orow = (size_t)it.bh * g.T + g.n_text + (size_t)yq * g.W + xq;
          const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
          __nv_bfloat16* dst = p.o + orow * D;
          #pragma unroll
          for (int c = 0; c < D / 32; c += 2) {
            uint32_t ov[2][32];
            tmem_ld32(o_tm + c * 32, ov[0]);
            tmem_ld32(o_tm + c * 32 + 32, ov[1]);
            tmem_wait_ld();
            if (row_valid) {
              #pragma unroll
              for (int u = 0; u < 2; ++u) {
                uint32_t w[16];
                #pragma unroll
                for (int i = 0; i < 16; ++i)
                  w[i] = pack_bf16x2(__uint_as_float(ov[u][2 * i]) * inv_l, __uint_as_float(ov[u][2 * i + 1]) * inv_l);
                __nv_bfloat16* d = dst + (c + u) * 32;
                if (p.wide_o) {
                  st_global_v8(d, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                  st_global_v8(d + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
                } else {
                  uint4* d4 = reinterpret_cast<uint4*>(d);
                  #pragma unroll
                  for (int e = 0; e < 4; ++e) d4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                }
              }
            }
          }
          if (row_valid) p.lse[orow] = (m_used + __log2f(l)) * 0.69314718055994530942f;
        }
        // The next pair's first P V overwrites O; it waits for this half's next P, which is
        // signalled after these TMEM reads.
        tc_fence_before();
        j = 0;
        continue;
      }
      // ---- a tile: {kind, a, b, flags | pair ordinal << 8}
      KeyTile t;
      t.kind = mv.x;
      t.a = mv.y;
      t.b = mv.z;
      t.flags = mv.w & 255;
      if (j == 0) {  // first tile of a pair: its geometry, fresh statistics
        it = decode_pair(g, blockIdx.x + (long long)(mv.w >> 8) * stride);
        if (it.is_text) {
          tq = it.q0 + half * kTile + row;
          row_valid = tq < g.n_text;
        } else {
          yq = it.q0 + half * kQH + (row >> 4);
          xq = it.x0 + (row & 15);
          row_valid = (yq < g.H) && (xq < g.W);
          yc = window_center(yq, g.r, g.H, g.window);
          xc = window_center(xq, g.r, g.W, g.window);
        }
        m_used = -INFINITY;
        l = 0.f;
      }
      {
        if (!mbar_wait(&bars[L::bSFull + half], nq & 1, abort_flag, kDevTimeoutSoftmax, 12 + half, (int)nq, j))
          goto softmax_done;
        tc_fence_after();
        float s[kFChunk];
        {
          uint32_t sr[kFChunk / 32][32];
          #pragma unroll
          for (int c = 0; c < kFChunk / 32; ++c) tmem_ld32(s_tm + c * 32, sr[c]);
          tmem_wait_ld();
          #pragma unroll
          for (int c = 0; c < kFChunk; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        // ---- mask. kw[c]: keep bits of this row's columns 32c .. 32c+31 (a rectangle's key rows
        // 2c and 2c+1, 16 bits each). Each 32-column chunk is then classed over the warp: no thread
        // keeps any key (skipped: P = 0, no exponentials), every thread keeps every key (no
        // selects), or partly kept (masked scores set to -inf). The classes are warp-uniform, so the
        // branches do not diverge.
        constexpr uint32_t kAllChunks = (1u << (kFChunk / 32)) - 1u;
        uint32_t cany = kAllChunks;
        if (!(t.flags & full_bit)) {
          uint32_t kw[kFChunk / 32];
          if (t.kind == kLinear) {
            #pragma unroll
            for (int c = 0; c < kFChunk / 32; ++c) {
              const int n = t.b - 32 * c;  // valid keys of the chunk
              kw[c] = n >= 32 ? ~0u : (n <= 0 ? 0u : ((1u << n) - 1u));
            }
          } else {
            // Row ky keeps columns [xc - w, xc + w] of the grid, w = half-width at |ky - yc|
            // (none when |ky - yc| >= r or ky is past the grid): clipped to the rectangle's 16
            // columns and the grid, as a 16-bit run.
            const int xr = xc - t.b;
            const int hi_lim = imin(g.W - 1 - t.b, kKW - 1);
            #pragma unroll
            for (int c = 0; c < kFChunk / 32; ++c) {
              uint32_t word = 0;
              #pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int ky = t.a + 2 * c + u;
                const int dy = ky - yc;
                const int ady = dy < 0 ? -dy : dy;
                int w = hwtab[imin(ady, hwn - 1)];
                w = (ady < hwn && ky < g.H) ? w : -1;
                const int lo = imin(imax(xr - w, 0), kKW);
                const int hi = imax(imin(xr + w, hi_lim), -1);
                word |= ((0xFFFFu >> (15 - hi)) & (0xFFFFu << lo) & 0xFFFFu) << (16 * u);
              }
              kw[c] = word;
            }
          }
          uint32_t cfull = 0;
          cany = 0;
          #pragma unroll
          for (int c = 0; c < kFChunk / 32; ++c) {
            cany |= __any_sync(0xffffffffu, kw[c] != 0u) ? (1u << c) : 0u;
            cfull |= __all_sync(0xffffffffu, kw[c] == ~0u) ? (1u << c) : 0u;
          }
          #pragma unroll
          for (int c = 0; c < kFChunk / 32; ++c) {
            if (((cany & ~cfull) >> c) & 1u) {
              #pragma unroll
              for (int e = 0; e < 32; ++e) s[32 * c + e] = ((kw[c] >> e) & 1u) ? s[32 * c + e] : -INFINITY;
            }
          }
        }
        // ---- tile max over the chunks some thread keeps (8 independent chains of 3-input maxima)
        float mx[8];
        if (cany == kAllChunks) {  // straight-line: every chunk
          #pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmax3(s[u], s[u + 8], s[u + 16]);
          #pragma unroll
          for (int c = 24; c + 16 <= kFChunk - 8; c += 16) {
            #pragma unroll
            for (int u = 0; u < 8; ++u) mx[u] = fmax3(mx[u], s[c + u], s[c + 8 + u]);
          }
          #pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], s[kFChunk - 8 + u]);
        } else {
          #pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
          #pragma unroll
          for (int c = 0; c < kFChunk / 32; ++c) {
            if ((cany >> c) & 1u) {
              #pragma unroll
              for (int u = 0; u < 8; ++u) {
                mx[u] = fmax3(mx[u], s[32 * c + u], s[32 * c + 8 + u]);
                mx[u] = fmax3(mx[u], s[32 * c + 16 + u], s[32 * c + 24 + u]);
              }
            }
          }
        }
        const float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
        const float mt_scaled = mt * sl2;
        float alpha = 1.f;
        bool need_rescale = false;
        if (m_used == -INFINITY) {
          m_used = mt_scaled;  // nothing accumulated yet (l == 0)
        } else if (mt_scaled > m_used + kRescaleThreshold) {
          // Lazy rescale: only when the max grows by more than 2^kRescaleThreshold; the final
          // O / l and the LSE use the same m_used, so the result stays exact up to rounding.
          alpha = ex2_approx(m_used - mt_scaled);
          l *= alpha;
          m_used = mt_scaled;
          need_rescale = true;
        }
        // ---- The two halves take turns at the exponentials of a tile both of them multiply: half A
        // after half B's previous such tile, half B after half A's same tile. Each half then has
        // the MUFU unit to itself while the tensor core runs the other half's products, instead of
        // both halves computing at once and both waiting for the tensor core afterwards.
        const bool both = (t.flags & (kNeedA | kNeedB)) == (kNeedA | kNeedB);
        if (both && (half == 1 || nboth > 0)) {
          const uint32_t ph = half == 0 ? ((nboth - 1) & 1) : (nboth & 1);
          if (!mbar_wait(&bars[L::bExpDone + (half ^ 1)], ph, abort_flag, kDevTimeoutSoftmax, 20 + half, (int)nboth,
                         (int)nq))
            goto softmax_done;
        }
        // ---- P = 2^(s * scale_log2 - m), row sum, bf16 pairs written over S in TMEM
        const float base = (m_used == -INFINITY) ? 0.f : m_used;
        const uint64_t sl2x2 = f32x2_pack(sl2, sl2), nbase2 = f32x2_pack(-base, -base);
        uint64_t acc2[4] = {0, 0, 0, 0};
        // P for columns 32c .. 32c+31: 16 bf16 pairs, row-sum terms into acc2, stored over S.
        auto exp_chunk = [&](int c4) {
          uint32_t pw[16];
          #pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int c = 32 * c4 + 2 * q;
            const uint64_t x = f32x2_fma(f32x2_pack(s[c], s[c + 1]), sl2x2, nbase2);
            if (CLEAR_FWD_EXP_BF16X2) {
              const uint32_t pb = ex2_approx_bf16x2(pack_bf16x2(f32x2_lo(x), f32x2_hi(x)));
              acc2[q & 3] =
                  f32x2_add(acc2[q & 3], f32x2_pack(__uint_as_float(pb << 16), __uint_as_float(pb & 0xFFFF0000u)));
              pw[q] = pb;
            } else {
              float e0, e1;
              if ((CLEAR_FWD_EXP2_POLY_PAIRS >> q) & 1u) {
                const uint64_t e = exp2_poly_x2(x);
                e0 = f32x2_lo(e);
                e1 = f32x2_hi(e);
              } else {
                e0 = ex2_approx(f32x2_lo(x));
                e1 = ex2_approx(f32x2_hi(x));
              }
              acc2[q & 3] = f32x2_add(acc2[q & 3], f32x2_pack(e0, e1));
              pw[q] = pack_bf16x2(e0, e1);
            }
          }
          tmem_st16(s_tm + c4 * 16, pw);
        };
        if (cany == kAllChunks) {  // straight-line: every chunk
          #pragma unroll
          for (int c4 = 0; c4 < kFChunk / 32; ++c4) exp_chunk(c4);
        } else {
          #pragma unroll
          for (int c4 = 0; c4 < kFChunk / 32; ++c4) {
            if ((cany >> c4) & 1u) {
              exp_chunk(c4);
            } else {  // no thread keeps a key of this chunk: P = 0
              uint32_t pw[16];
              #pragma unroll
              for (int q = 0; q < 16; ++q) pw[q] = 0u;
              tmem_st16(s_tm + c4 * 16, pw);
            }
          }
        }
        if (both) {
          mbar_arrive(&bars[L::bExpDone + half]);
          ++nboth;
        }
        l += ((f32x2_lo(acc2[0]) + f32x2_hi(acc2[0])) + (f32x2_lo(acc2[1]) + f32x2_hi(acc2[1]))) +
             ((f32x2_lo(acc2[2]) + f32x2_hi(acc2[2])) + (f32x2_lo(acc2[3]) + f32x2_hi(acc2[3])));
        if (j > 0 && __any_sync(0xffffffffu, need_rescale)) {
          // O holds P V up to tile j-1, complete: the S-full commit of this tile was issued after
          // it. Rescale O in place; P V of this tile waits for the P-full signal below. (Done
          // after P is written, when the score registers are free.)
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
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[L::bPFull + half]);
        ++nq;
        ++j;
      }
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
  for (int s = 0; s < g.fS; ++s) {
    const float2 v = p.ml[((size_t)s * g.BH + bh) * g.n_text + tq];
    if (v.y > 0.f) m = fmaxf(m, v.x);
  }
  constexpr int kPer = D / 32;
  float acc[kPer];
  #pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float l = 0.f;
  for (int s = 0; s < g.fS; ++s) {
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
