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
// block, or two consecutive text tiles) that share every 64-key tile: each K/V tile is loaded once
// and multiplied by whichever halves reach it.
//   warps 0-3   softmax / epilogue of half A (thread t owns query row t = TMEM lane t);
//   warps 4-7   softmax / epilogue of half B;
//   warp 8      TMA producer: Q of both halves once per pair, K and V tiles into 4-slot rings. It
//               enumerates each union tile once and publishes its descriptor (kind, origin, per-half
//               need / full bits, last-of-pair bit, head) in a 16-entry shared ring that the V
//               stream and both MMA issuers read, so nobody else re-runs the enumeration;
//   warps 9/10  MMA issuers, one per half. Each polls two walks over the pair's union tiles: the
//               QK walk issues S_j = Q K_j^T into one of two 64-column TMEM buffers (up to one
//               needed tile ahead of P V) and posts the tile to its softmax through a two-slot
//               mailbox; the PV walk issues O += P_j V_j once the softmax has written P_j over S_j
//               (bf16, in TMEM; A operand from TMEM). Tiles a half does not need are still
//               observed (their "full" phase) and released by that half, so each half sees every
//               phase of every ring slot in order, which keeps the parity-based waits exact.
//               Polling (instead of blocking) keeps either walk from holding up the other, so
//               every wait depends only on earlier tiles. The end of a pair is posted to the
//               softmax as a mailbox message;
//   warp 11     idle (it completes the third warpgroup, whose registers go to the softmax).
// TMEM columns of half h: S buffers [256h, 256h+64) and [256h+64, 256h+128), O [256h+128, 256h+256).
// The running max is rescaled lazily: O and l are only rescaled when a row's max grows by more
// than 2^8, which leaves the result exact up to rounding (the final division uses the same max).
#pragma once
#include <cuda_bf16.h>

#include "clear_common.cuh"
#include "clear_sched.cuh"
#include "sm100_ptx.cuh"

namespace clear {

constexpr int kKStages = 4;   // K ring slots
constexpr int kVStages = 4;   // V ring slots
constexpr int kFwdThreads = 384;           // 3 warpgroups: softmax A, softmax B, producer + MMA
// Launched at 168 registers per thread (65536 / 384, rounded to 8). The producer / MMA warpgroup
// drops to kRegsLow and the two softmax warpgroups grow to kRegsHigh:
// 2 * 128 * kRegsHigh + 128 * kRegsLow <= 384 * 168.
constexpr uint32_t kRegsLow = 88;
constexpr uint32_t kRegsHigh = 208;
static_assert(2 * 128 * kRegsHigh + 128 * kRegsLow <= 384 * 168, "register split exceeds the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kTileRing = 16;              // union tile descriptors in flight (producer -> others)
// Mailbox message kinds (issuer -> softmax); tiles use their KeyKind (kLinear / kRect).
constexpr int kMsgEndPair = 2;             // the half's last tile of the current pair was posted
constexpr int kMsgEndAll = 3;              // no more pairs for this CTA

struct FwdParams {
  Geom g;
  float scale_log2;           // (1/sqrt(d)) * log2(e)
  __nv_bfloat16* o;           // row (b, h, t) at o + b * o_sb + h * o_sh + t * o_st (elements)
  long long o_sb, o_sh, o_st;
  // The kernel's kSplit parameter: q, k, v maps (and o) have separate head and batch axes; without
  // it one flat b*heads+h axis, and row (bh, t) of o sits at o + bh * o_sh + t * o_st.
  float* lse;                 // [BH, T]
  float* opart;               // [fS, BH, n_text, d] unnormalised partial O of text rows
  float2* ml;                 // [fS, BH, n_text] (running max in scaled log2 units, sum)
  long long n_work;           // pair items
  int wide_o, wide_part;      // o / opart are 32-byte aligned: the epilogue may store 32 bytes at once
  // Mixed-resolution batch (the kernel's kVar parameter): per-item geometry (Geom::t0, tok_total,
  // part_row0 and crow0 place the item in the packed tensors) and image tensor maps (q, k, v for
  // each item), in device memory; the batch's pairs are every item's text pairs, then every item's
  // image pairs: wbound[i] is the first pair of item i's text pairs, wbound[n_items + i] of its
  // image pairs, wbound[2 * n_items] the total. p.g then carries what the items share (heads, d,
  // r, window) and the largest H (the half-width table's size).
  const Geom* items;
  const CUtensorMap* item_maps;
  const long long* wbound;
  int n_items;
  // FP8 score products (the kernel's kF8 parameter): s_q * s_k of each (batch, head), the
  // dequantization of the E4M3 codes' products, folded into the score scale.
  const float* qk_descale;
};

// Item of pair w of a mixed-resolution batch, and w's index among the item's own pairs.
__device__ __forceinline__ int locate_pair(const FwdParams& p, long long w, long long* local) {
  int lo = 0, hi = 2 * p.n_items - 1;  // last k with wbound[k] <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.wbound + mid) <= w) lo = mid; else hi = mid - 1;
  }
  const int item = lo < p.n_items ? lo : lo - p.n_items;
  const long long off = w - __ldg(p.wbound + lo);
  *local = lo < p.n_items ? off : p.items[item].n_txt_pairs + off;
  return item;
}

// One 32-byte global store (the address must be 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* ptr, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t a4, uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

// kF8: q and k tiles hold E4M3 codes (one byte per element; one 128-byte row block at d = 128).
template <int D, bool kF8 = false>
struct FwdLayout {
  static constexpr int kQTileBytes = kTile * D * (kF8 ? 1 : 2);     // one 128-row query tile
  static constexpr int kKTileBytes = kFChunk * D * (kF8 ? 1 : 2);   // one 64-key k tile
  static constexpr int kVTileBytes = kFChunk * D * 2;               // one 64-key bf16 v tile
  static constexpr int kKVBlock = kFChunk * 128;         // 64 rows x 64 elements (128B-swizzled)
  static constexpr int kQ = 0;                           // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kQTileBytes;
  static constexpr int kV = kK + kKStages * kKTileBytes;
  static constexpr int kBars = kV + kVStages * kVTileBytes;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 1;
  static constexpr int bKFull = 2;                       // + slot
  static constexpr int bKEmpty = bKFull + kKStages;      // + slot
  static constexpr int bVFull = bKEmpty + kKStages;      // + slot
  static constexpr int bVEmpty = bVFull + kVStages;      // + slot
  static constexpr int bSFull = bVEmpty + kVStages;      // + 2 * half + buffer
  static constexpr int bPFull = bSFull + 4;              // + 2 * half + buffer
  static constexpr int bMsgFull = bPFull + 4;            // + 2 * half + slot: mailbox message posted
  static constexpr int bMsgEmpty = bMsgFull + 4;         // + 2 * half + slot: mailbox slot read
  static constexpr int bODone = bMsgEmpty + 4;           // + half: last P V of the half's pair done
  static constexpr int bOReady = bODone + 2;             // + half: every P V done (one phase per tile)
  static constexpr int kNumBars = bOReady + 2;
  static constexpr int kMsg = (kBars + kNumBars * 8 + 15) & ~15;  // int4[2][2] mailbox: {kind, a, b, flags | ordinal << 8}
  static constexpr int kRing = kMsg + 64;                // int4[kTileRing]: {kind | flags << 4 | last << 12, a, b, bh}
  static_assert(kMsg % 16 == 0 && kRing % 16 == 0, "int4 mailbox and ring need 16-byte alignment");
  static_assert(kQ % 1024 == 0 && kK % 1024 == 0 && kV % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static constexpr int kMisc = kRing + kTileRing * 16;
  static constexpr int kWTab = kMisc + 16;               // int[kMaxRTable] (tile enumeration)
  static constexpr int kHwTab = kWTab + kMaxRTable * 4;  // int16[hw_table_size(r, H)] (masks)
  static constexpr int kFixed = kHwTab + 1024;           // + slack for 1024-byte alignment
  static __host__ __device__ constexpr int alloc_bytes(int hw_entries) { return kFixed + ((hw_entries * 2 + 15) & ~15); }
  static constexpr uint32_t kTmemCols = 512;
  static __host__ __device__ constexpr uint32_t s_col(int half, int buf) { return half * 256 + buf * 64; }
  static __host__ __device__ constexpr uint32_t o_col(int half) { return half * 256 + 128; }
};

// The forward's tensor maps view q, k, v with one flat b*heads+h axis when the layout allows it
// (batch stride = heads x head stride, or B = 1): linear (d, T, B*heads) and image (d, W, H,
// B*heads) maps. Otherwise (split_bh) they have separate head and batch axes, so any token, head and
// batch strides (multiples of 16 bytes) are read in place: (d, T, heads, B) and (d, W, H, heads, B),
// and a tile's (head, batch) coordinates come from its bh = b * heads + h.
// Loads one 64-key tile (all 64-element column blocks) of k or v: a 64-token chunk (kind kLinear,
// first token a) or a 4 x 16 grid rectangle (kind kRect, rows from a, columns from b).
template <int D, bool kSplit>
__device__ __forceinline__ void load_kv64(uint8_t* dst, const CUtensorMap* lin, const CUtensorMap* img, uint64_t* bar,
                                          int kind, int a, int b, int bh, int heads) {
  #pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    uint8_t* d = dst + h * FwdLayout<D>::kKVBlock;
    if (!kSplit) {
      if (kind == kLinear)
        tma_load_3d(d, lin, bar, h * 64, a, bh);
      else
        tma_load_4d(d, img, bar, h * 64, b, a, bh);
    } else {
      const int hh = bh % heads, bb = bh / heads;
      if (kind == kLinear)
        tma_load_4d(d, lin, bar, h * 64, a, hh, bb);
      else
        tma_load_5d(d, img, bar, h * 64, b, a, hh, bb);
    }
  }
}

// Loads one 128-row query tile (all 64-element column blocks): 128 tokens from a (kind kLinear) or
// an 8 x 16 grid rectangle (kind kRect, rows from a, columns from b).
template <int D, bool kSplit>
__device__ __forceinline__ void load_q128(uint8_t* dst, const CUtensorMap* lin, const CUtensorMap* img, uint64_t* bar,
                                          int kind, int a, int b, int bh, int heads) {
  if (!kSplit) {
    load_tile<D>(dst, lin, img, bar, kind, a, b, bh);
    return;
  }
  const int hh = bh % heads, bb = bh / heads;
  #pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    uint8_t* d = dst + h * kHalfBytes;
    if (kind == kLinear)
      tma_load_4d(d, lin, bar, h * 64, a, hh, bb);
    else
      tma_load_5d(d, img, bar, h * 64, b, a, hh, bb);
  }
}

template <int D, bool kSplit, bool kVar, bool kF8 = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
clear_fwd_kernel(const __grid_constant__ CUtensorMap tm_q_lin, const __grid_constant__ CUtensorMap tm_q_img,
                 const __grid_constant__ CUtensorMap tm_k_lin, const __grid_constant__ CUtensorMap tm_k_img,
                 const __grid_constant__ CUtensorMap tm_v_lin, const __grid_constant__ CUtensorMap tm_v_img,
                 const FwdParams p) {
  using L = FwdLayout<D, kF8>;
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
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars[L::bSFull + i], 1);
      mbar_init(&bars[L::bPFull + i], 128);
      mbar_init(&bars[L::bMsgFull + i], 1);
      mbar_init(&bars[L::bMsgEmpty + i], 128);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars[L::bODone + h], 1);
      mbar_init(&bars[L::bOReady + h], 1);
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

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    regs_dec<kRegsLow>();
    if (lane == 0) {
      tma_prefetch_desc(&tm_q_lin); tma_prefetch_desc(&tm_q_img);
      tma_prefetch_desc(&tm_k_lin); tma_prefetch_desc(&tm_k_img);
      tma_prefetch_desc(&tm_v_lin); tma_prefetch_desc(&tm_v_img);
      long long wq = blockIdx.x;
      uint32_t q_loads = 0;
      // K stream: the current union tile and a one-tile lookahead (for the last-of-pair bit).
      long long wk = blockIdx.x;
      PairItem itk{};
      PairKeyIter kik;
      KeyTile tcur{}, tnext{};
      bool kval = wk < p.n_work, next_in_pair = false;
      int ik = 0;  // the K stream's batch item (mixed-resolution batches)
      auto start_k_pair = [&]() {
        long long lw = wk;
        if constexpr (kVar) ik = locate_pair(p, wk, &lw);
        const Geom& gk = kVar ? p.items[ik] : g;
        itk = decode_pair(gk, lw);
        kik.init(gk, itk, wtab, wtn);
        kik.next(&tcur);
        next_in_pair = kik.next(&tnext);
      };
      if (kval) start_k_pair();
      uint32_t Gk = 0, Gv = 0;
      PollWatchdog wd;
      wd.start();
      while (wq < p.n_work || kval || Gv < Gk) {
        bool prog = false;
        if (wq < p.n_work && (q_loads == 0 || mbar_test(&bars[L::bQEmpty], (q_loads - 1) & 1))) {
          long long lw = wq;
          int iq = 0;
          if constexpr (kVar) iq = locate_pair(p, wq, &lw);
          const Geom& gq = kVar ? p.items[iq] : g;
          const CUtensorMap* qimg = kVar ? p.item_maps + 3 * iq : &tm_q_img;
          const int t0 = kVar ? gq.t0 : 0;  // the item's first token in the packed batch
          const PairItem it = decode_pair(gq, lw);
          mbar_arrive_expect_tx(&bars[L::bQFull], (it.validB ? 2 : 1) * L::kQTileBytes);
          if constexpr (kF8) {  // one 128-byte row block per tile
            uint8_t* qa = smem + L::kQ;
            if (it.is_text) {
              tma_load_3d(qa, &tm_q_lin, &bars[L::bQFull], 0, it.q0, it.bh);
              if (it.validB) tma_load_3d(qa + L::kQTileBytes, &tm_q_lin, &bars[L::bQFull], 0, it.q0 + kTile, it.bh);
            } else {
              tma_load_4d(qa, &tm_q_img, &bars[L::bQFull], 0, it.x0, it.q0, it.bh);
              if (it.validB) tma_load_4d(qa + L::kQTileBytes, &tm_q_img, &bars[L::bQFull], 0, it.x0, it.q0 + kQH, it.bh);
            }
          } else if (it.is_text) {
            load_q128<D, kSplit>(smem + L::kQ, &tm_q_lin, qimg, &bars[L::bQFull], kLinear, t0 + it.q0, 0, it.bh, g.heads);
            if (it.validB)
              load_q128<D, kSplit>(smem + L::kQ + L::kQTileBytes, &tm_q_lin, qimg, &bars[L::bQFull], kLinear,
                           t0 + it.q0 + kTile, 0, it.bh, g.heads);
          } else {
            load_q128<D, kSplit>(smem + L::kQ, &tm_q_lin, qimg, &bars[L::bQFull], kRect, it.q0, it.x0, it.bh, g.heads);
            if (it.validB)
              load_q128<D, kSplit>(smem + L::kQ + L::kQTileBytes, &tm_q_lin, qimg, &bars[L::bQFull], kRect,
                           it.q0 + kQH, it.x0, it.bh, g.heads);
          }
          ++q_loads;
          wq += stride;
          prog = true;
        }
        if (kval && Gk - Gv < (uint32_t)kTileRing) {
          const uint32_t ks = Gk % kKStages;
          if (mbar_test(&bars[L::bKEmpty + ks], ((Gk / kKStages) & 1) ^ 1)) {
            // Publish the descriptor before the load: the K barrier's completion makes it visible.
            // Linear tiles carry item-local tokens; bits 16+ of the first word hold the batch item.
            ring[Gk % kTileRing] = make_int4(tcur.kind | (tcur.flags << 4) | (next_in_pair ? 0 : (1 << 12)) | (ik << 16),
                                             tcur.a, tcur.b, itk.bh);
            mbar_arrive_expect_tx(&bars[L::bKFull + ks], L::kKTileBytes);
            if constexpr (kF8) {  // one 128-byte row block per tile
              if (tcur.kind == kLinear)
                tma_load_3d(smem + L::kK + ks * L::kKTileBytes, &tm_k_lin, &bars[L::bKFull + ks], 0, tcur.a, itk.bh);
              else
                tma_load_4d(smem + L::kK + ks * L::kKTileBytes, &tm_k_img, &bars[L::bKFull + ks], 0, tcur.b, tcur.a, itk.bh);
            } else
            load_kv64<D, kSplit>(smem + L::kK + ks * L::kKTileBytes, &tm_k_lin,
                                 kVar ? p.item_maps + 3 * ik + 1 : &tm_k_img, &bars[L::bKFull + ks], tcur.kind,
                                 tcur.kind == kLinear && kVar ? p.items[ik].t0 + tcur.a : tcur.a, tcur.b, itk.bh, g.heads);
            ++Gk;
            if (next_in_pair) {
              tcur = tnext;
              next_in_pair = kik.next(&tnext);
            } else {
              wk += stride;
              kval = wk < p.n_work;
              if (kval) start_k_pair();
            }
            prog = true;
          }
        }
        if (Gv < Gk) {
          const uint32_t vs = Gv % kVStages;
          if (mbar_test(&bars[L::bVEmpty + vs], ((Gv / kVStages) & 1) ^ 1)) {
            const int4 e = ring[Gv % kTileRing];
            const int iv = e.x >> 16;
            mbar_arrive_expect_tx(&bars[L::bVFull + vs], L::kVTileBytes);
            load_kv64<D, kSplit>(smem + L::kV + vs * L::kVTileBytes, &tm_v_lin,
                                 kVar ? p.item_maps + 3 * iv + 2 : &tm_v_img, &bars[L::bVFull + vs], e.x & 15,
                                 (e.x & 15) == kLinear && kVar ? p.items[iv].t0 + e.y : e.y, e.z, e.w, g.heads);
            ++Gv;
            prog = true;
          }
        }
        if (!wd.tick(prog, abort_flag, kDevTimeoutTmaEmpty, 1, (int)Gk, (int)Gv, (int)q_loads)) break;
      }
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------------ MMA issuers (one per half)
    regs_dec<kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kFChunk, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const int h = warp - 9;
      const int need_bit = h == 0 ? kNeedA : kNeedB;
      const uint32_t q_addr = smem_u32(smem + L::kQ + h * L::kQTileBytes);
      const uint32_t o_tm = tmem + L::o_col(h);
      // Shared-memory matrix descriptors, advanced per 16-element K step with plain adds.
      const uint64_t qdesc = smem_desc_sw128(q_addr, 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + L::kV), L::kKVBlock, 1024);
      const uint32_t n_pairs = (uint32_t)((p.n_work - blockIdx.x + stride - 1) / stride);
      // QK walk over the union tiles (union index Gq); pairs are observed in order.
      uint32_t pair = 0, Gq = 0, nqk = 0, nmsg = 0;
      bool q_seen = false, had = false, end_pending = false, all_posted = false;
      // PV walk: union index Gp; up to two needed tiles whose Q K^T is issued and P V is not.
      uint32_t Gp = 0, npv = 0;
      // The pending tiles form a two-entry FIFO kept in registers (head h*, tail t*): union index,
      // and flags (bit 0: first of the pair, overwrite O; bit 1: commit o_done after its P V).
      uint32_t hG = 0, tG = 0;
      int hF = 0, tF = 0;
      int pend = 0;
      PollWatchdog wd;
      wd.start();
      while (!all_posted || Gp < Gq || pend > 0) {
        bool prog = false;
        // ---- PV walk step (tiles the QK walk has passed, in order). It goes first: a ready P V
        // frees the S buffer the next Q K^T needs.
        if (Gp < Gq) {
          const uint32_t vs = Gp % kVStages;
          const bool needed = pend > 0 && hG == Gp;
          if (!needed) {
            if (mbar_test(&bars[L::bVFull + vs], (Gp / kVStages) & 1)) {
              mbar_arrive(&bars[L::bVEmpty + vs]);  // observed and released
              ++Gp;
              prog = true;
            }
          } else {
            const uint32_t b = npv & 1;
            const bool pr = mbar_test(&bars[L::bPFull + 2 * h + b], (npv >> 1) & 1);
            const bool vr = mbar_test(&bars[L::bVFull + vs], (Gp / kVStages) & 1);
            if (pr && vr) {
              tc_fence_after();
              const uint64_t vd = vdesc0 + (uint64_t)((vs * L::kVTileBytes) >> 4);
              const uint32_t s_tm = tmem + L::s_col(h, b);
              const bool first = hF & 1;
              #pragma unroll
              for (int kk = 0; kk < kFChunk / 16; ++kk)
                umma_ts(o_tm, s_tm + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                        (!first || kk > 0) ? 1u : 0u);
              umma_commit(&bars[L::bVEmpty + vs]);
              umma_commit(&bars[L::bOReady + h]);
              if (hF & 2) umma_commit(&bars[L::bODone + h]);
              ++npv;
              --pend;
              hG = tG;
              hF = tF;
              ++Gp;
              prog = true;
            }
          }
        }
        // ---- QK walk step
        if (end_pending || (pair >= n_pairs && !all_posted)) {
          // Post an end-of-pair (or end-of-work) message once the mailbox slot is free.
          const uint32_t ms = nmsg & 1;
          if (mbar_test(&bars[L::bMsgEmpty + 2 * h + ms], ((nmsg >> 1) & 1) ^ 1)) {
            msg[2 * h + ms] = make_int4(end_pending ? kMsgEndPair : kMsgEndAll, 0, 0, 0);
            mbar_arrive(&bars[L::bMsgFull + 2 * h + ms]);
            ++nmsg;
            if (end_pending) end_pending = false; else all_posted = true;
            prog = true;
          }
        } else if (pair < n_pairs) {
          if (!q_seen) {
            if (mbar_test(&bars[L::bQFull], pair & 1)) {  // every half observes every Q phase
              q_seen = true;
              had = false;
              prog = true;
            }
          } else {
            const uint32_t ks = Gq % kKStages;
            const uint32_t ms = nmsg & 1;
            // The K barrier, the ring entry and the mailbox are read back to back so their
            // latencies overlap; the test's acquire orders the ring read, and the entry is used
            // only once the test has passed.
            const bool kr = mbar_test(&bars[L::bKFull + ks], (Gq / kKStages) & 1);
            const int4 e = ring[Gq % kTileRing];
            const bool mr = mbar_test(&bars[L::bMsgEmpty + 2 * h + ms], ((nmsg >> 1) & 1) ^ 1);
            if (kr) {
              const int flags = (e.x >> 4) & 255;
              const bool last_of_pair = (e.x >> 12) & 1;
              const bool needed = (flags & need_bit) != 0;
              bool done_tile = false;
              if (!needed) {
                mbar_arrive(&bars[L::bKEmpty + ks]);  // observed and released
                done_tile = true;
              } else if (pend < 2 && mr) {
                const uint32_t b = nqk & 1;
                msg[2 * h + ms] = make_int4(e.x & 15, e.y, e.z, flags | (int)(pair << 8));
                mbar_arrive(&bars[L::bMsgFull + 2 * h + ms]);
                ++nmsg;
                tc_fence_after();
                const uint64_t kd = kdesc0 + (uint64_t)((ks * L::kKTileBytes) >> 4);
                if constexpr (kF8) {
                  // 32 one-byte elements per step, all inside the tile's single 128-byte row block
                  constexpr uint32_t idesc_f8 = idesc_e4m3_f32(128, kFChunk);
                  #pragma unroll
                  for (int kk = 0; kk < D / 32; ++kk)
                    umma_ss_f8(tmem + L::s_col(h, b), qdesc + (uint32_t)((kk * 32) >> 4), kd + (uint32_t)((kk * 32) >> 4),
                               idesc_f8, kk > 0);
                } else {
                  #pragma unroll
                  for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t qoff = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
                    const uint32_t koff = ((kk >> 2) * L::kKVBlock + (kk & 3) * 32) >> 4;
                    umma_ss(tmem + L::s_col(h, b), qdesc + qoff, kd + koff, idesc_qk, kk > 0);
                  }
                }
                umma_commit(&bars[L::bSFull + 2 * h + b]);
                umma_commit(&bars[L::bKEmpty + ks]);
                if (pend == 0) {
                  hG = Gq;
                  hF = had ? 0 : 1;
                } else {
                  tG = Gq;
                  tF = had ? 0 : 1;
                }
                ++pend;
                ++nqk;
                had = true;
                done_tile = true;
              }
              if (done_tile) {
                ++Gq;
                prog = true;
                if (last_of_pair) {
                  // Pair finished for this half: release Q, arrange o_done, tell the softmax.
                  if (had) {
                    umma_commit(&bars[L::bQEmpty]);
                    // o_done follows this half's last P V of the pair: mark it if still pending
                    // (it is the most recent needed tile), else commit now.
                    if (pend == 2)
                      tF |= 2;
                    else if (pend == 1)
                      hF |= 2;
                    else
                      umma_commit(&bars[L::bODone + h]);
                    end_pending = true;
                  } else {
                    mbar_arrive(&bars[L::bQEmpty]);
                  }
                  ++pair;
                  q_seen = false;
                }
              }
            }
          }
        }
        if (!wd.tick(prog, abort_flag, kDevTimeoutMma, 2 + h, (int)Gq, (int)(Gp | (npv << 16)),
                     pend | (end_pending ? 4 : 0) | (all_posted ? 8 : 0) | (q_seen ? 16 : 0) | ((int)pair << 8))) break;
      }
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
    const uint32_t o_tm = tmem + lane_base + L::o_col(half);
    const int full_bit = half == 0 ? kFullA : kFullB;
    uint32_t nq = 0, n_out = 0, nmsg = 0;
    float sl2 = p.scale_log2;  // with kF8, times the pair's s_q * s_k (set at each pair's first tile)
    // Per-pair state, set up at the pair's first tile. gs: the pair's geometry (its batch item's in a
    // mixed-resolution batch).
    Geom gv = g;
    const Geom& gs = kVar ? gv : g;
    PairItem it{};
    int yq = 0, xq = 0, tq = 0;
    int yc = 0, xc = 0;  // the window's centre: (yq, xq), clamped inside the grid for shifted windows
    bool row_valid = false;
    float m_used = -INFINITY;  // running max, scaled log2 units
    float l = 0.f;
    int j = 0;
    while (true) {
      const uint32_t ms = nmsg & 1;
      if (!mbar_wait(&bars[L::bMsgFull + 2 * half + ms], (nmsg >> 1) & 1, abort_flag, kDevTimeoutSoftmax, 10 + half,
                     (int)nmsg, j))
        goto softmax_done;
      const int4 mv = msg[2 * half + ms];
      mbar_arrive(&bars[L::bMsgEmpty + 2 * half + ms]);
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
          const size_t prow = (size_t)gs.part_row0 + ((size_t)it.split * gs.BH + it.bh) * gs.n_text + (row_valid ? tq : 0);
          float* dst = p.opart + prow * D;
          // Two TMEM loads per wait; each row's 512-byte run is written 32 (or 16) bytes at a time.
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
          const long long tok = (long long)gs.t0 + gs.n_text + (long long)yq * gs.W + xq;  // token in the batch
          const size_t orow = (size_t)it.bh * gs.tok_total + tok;                            // lse row
          const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
          __nv_bfloat16* dst = p.o + tok * p.o_st +
                               (kSplit ? (long long)(it.bh / g.heads) * p.o_sb + (long long)(it.bh % g.heads) * p.o_sh
                                       : (long long)it.bh * p.o_sh);
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
        long long lw = blockIdx.x + (long long)(mv.w >> 8) * stride;
        if constexpr (kVar) gv = p.items[locate_pair(p, lw, &lw)];
        it = decode_pair(gs, lw);
        if constexpr (kF8) sl2 = p.scale_log2 * __ldg(p.qk_descale + it.bh);
        if (it.is_text) {
          tq = it.q0 + half * kTile + row;
          row_valid = tq < gs.n_text;
        } else {
          yq = it.q0 + half * kQH + (row >> 4);
          xq = it.x0 + (row & 15);
          row_valid = (yq < gs.qy1) && (xq < gs.W);
          yc = window_center(yq, gs.r, gs.H, gs.window);
          xc = window_center(xq, gs.r, gs.W, gs.window);
        }
        m_used = -INFINITY;
        l = 0.f;
      }
      {
        const uint32_t b = nq & 1, ph = (nq >> 1) & 1;
        if (!mbar_wait(&bars[L::bSFull + 2 * half + b], ph, abort_flag, kDevTimeoutSoftmax, 12 + half, (int)nq, j))
          goto softmax_done;
        tc_fence_after();
        const uint32_t s_tm = tmem + lane_base + L::s_col(half, b);
        float s[kFChunk];
        {
          uint32_t sr[2][32];
          tmem_ld32(s_tm + 0, sr[0]);
          tmem_ld32(s_tm + 32, sr[1]);
          tmem_wait_ld();
          #pragma unroll
          for (int c = 0; c < kFChunk; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
        }
        // ---- mask (branch-free selects; full tiles skip it)
        if (!(t.flags & full_bit)) {
          if (t.kind == kLinear) {
            const int lim = t.b;
            #pragma unroll
            for (int c = 0; c < kFChunk; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
          } else {
            // keep bits: word q holds key rows 2q (bits 0-15) and 2q+1 (bits 16-31)
            uint32_t keep[kFKH / 2];
            #pragma unroll
            for (int q = 0; q < kFKH / 2; ++q) {
              int lo0, hi0, lo1, hi1;
              row_range_tab(gs, hwtab, hwn, yc, xc, t.a + 2 * q, t.b, &lo0, &hi0);
              row_range_tab(gs, hwtab, hwn, yc, xc, t.a + 2 * q + 1, t.b, &lo1, &hi1);
              const int n0 = imax(hi0 - lo0 + 1, 0), n1 = imax(hi1 - lo1 + 1, 0);
              keep[q] = (((1u << n0) - 1u) << (lo0 & 15)) | ((((1u << n1) - 1u) << (lo1 & 15)) << 16);
            }
            #pragma unroll
            for (int c = 0; c < kFChunk; ++c)
              s[c] = (keep[c >> 5] & (1u << (c & 31))) ? s[c] : -INFINITY;
          }
        }
        // ---- tile max (8 independent chains of 3-input maxima)
        float mx[8];
        #pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmax3(s[u], s[u + 8], s[u + 16]);
        #pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmax3(mx[u], s[u + 24], s[u + 32]);
        #pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmax3(mx[u], s[u + 40], s[u + 48]);
        #pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], s[u + 56]);
        const float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
        const float mt_scaled = mt * sl2;
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
          // O holds P V up to tile j-1: wait for that product (the one for tile j cannot start
          // before this tile's P is signalled), then rescale O in place.
          if (!mbar_wait(&bars[L::bOReady + half], (nq - 1) & 1, abort_flag, kDevTimeoutSoftmax, 14 + half, (int)nq, j))
            goto softmax_done;
          tc_fence_after();
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
        const uint64_t sl2x2 = f32x2_pack(sl2, sl2), nbase2 = f32x2_pack(-base, -base);
        uint64_t acc2[4] = {0, 0, 0, 0};
        uint32_t pw[32];
        #pragma unroll
        for (int q = 0; q < 32; ++q) {
          const uint64_t x = f32x2_fma(f32x2_pack(s[2 * q], s[2 * q + 1]), sl2x2, nbase2);
          const float e0 = ex2_approx(f32x2_lo(x));
          const float e1 = ex2_approx(f32x2_hi(x));
          acc2[q & 3] = f32x2_add(acc2[q & 3], f32x2_pack(e0, e1));
          pw[q] = pack_bf16x2(e0, e1);
        }
        tmem_st32(s_tm, pw);
        l += ((f32x2_lo(acc2[0]) + f32x2_hi(acc2[0])) + (f32x2_lo(acc2[1]) + f32x2_hi(acc2[1]))) +
             ((f32x2_lo(acc2[2]) + f32x2_hi(acc2[2])) + (f32x2_lo(acc2[3]) + f32x2_hi(acc2[3])));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[L::bPFull + 2 * half + b]);
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
// O = sum_s 2^(m_s - m) O_s / l, LSE = (m + log2 l) ln 2. One warp per text row: text row tq of
// head bh of the problem (or batch item) g.
template <int D, bool kSplit>
__device__ __forceinline__ void combine_text_row(const FwdParams& p, const Geom& g, int bh, int tq, int lane) {
  float m = -INFINITY;
  for (int s = 0; s < g.fS; ++s) {
    const float2 v = p.ml[(size_t)g.part_row0 + ((size_t)s * g.BH + bh) * g.n_text + tq];
    if (v.y > 0.f) m = fmaxf(m, v.x);
  }
  constexpr int kPer = D / 32;
  float acc[kPer];
  #pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float l = 0.f;
  for (int s = 0; s < g.fS; ++s) {
    const size_t prow = (size_t)g.part_row0 + ((size_t)s * g.BH + bh) * g.n_text + tq;
    const float2 v = p.ml[prow];
    if (!(v.y > 0.f)) continue;
    const float f = exp2f(v.x - m);
    l += f * v.y;
    const float* src = p.opart + prow * D;
    #pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] += f * src[lane * kPer + e];
  }
  const float inv_l = 1.f / l;
  const long long tok = (long long)g.t0 + tq;       // token in the (packed) tensors
  const size_t orow = (size_t)bh * g.tok_total + tok;  // lse row
  __nv_bfloat16* dst = p.o + tok * p.o_st + lane * kPer +
                       (kSplit ? (long long)(bh / g.heads) * p.o_sb + (long long)(bh % g.heads) * p.o_sh
                               : (long long)bh * p.o_sh);
  #pragma unroll
  for (int e = 0; e < kPer; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv_l);
  if (lane == 0) p.lse[orow] = (m + log2f(l)) * 0.69314718055994530942f;
}

template <int D, bool kSplit>
__global__ void clear_fwd_combine_kernel(const FwdParams p) {
  const Geom& g = p.g;
  const int warps_per_block = blockDim.x / 32;
  const long long row_id = (long long)blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  if (row_id >= (long long)g.BH * g.n_text) return;
  combine_text_row<D, kSplit>(p, g, (int)(row_id / g.n_text), (int)(row_id % g.n_text), threadIdx.x & 31);
}

// The same merge for every text row of a mixed-resolution batch (rows of item i: [crow0_i,
// crow0_i + BH * n_text_i)).
template <int D>
__global__ void clear_fwd_combine_varlen_kernel(const FwdParams p, long long rows) {
  const int warps_per_block = blockDim.x / 32;
  const long long row_id = (long long)blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  if (row_id >= rows) return;
  int lo = 0, hi = p.n_items - 1;  // last item with crow0 <= row_id (items without text rows share the next one's)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.items[mid].crow0 <= row_id) lo = mid; else hi = mid - 1;
  }
  const Geom& g = p.items[lo];
  const long long r0 = row_id - g.crow0;
  combine_text_row<D, false>(p, g, (int)(r0 / g.n_text), (int)(r0 % g.n_text), threadIdx.x & 31);
}

}  // namespace clear

namespace clear {

// Merges text query rows computed by P patches (parts) of a patch-parallel forward. Part p gives
// its rows normalised over its own keys, O_p, and their log-sum-exp L_p (natural log).
//   mode 0 (exact): L = log sum_p exp(L_p), O = sum_p exp(L_p - L) O_p: the softmax over the union
//                   of the parts' key sets, which must be disjoint;
//   mode 1 (the patch-wise average of Eq. 7 in the CLEAR paper): O = (1/P) sum_p O_p, each part's
//                   keys being the text tokens plus that patch's image tokens; L is written as in
//                   mode 0.
// One warp per text row; parts with no key (L_p = -inf) carry no weight.
template <int D>
__global__ void clear_text_merge_kernel(int rows, int parts, int mode, const __nv_bfloat16* __restrict__ o_parts,
                                        const float* __restrict__ lse_parts, __nv_bfloat16* __restrict__ o,
                                        float* __restrict__ lse) {
  const int warps_per_block = blockDim.x / 32;
  const long long row = (long long)blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int pp = 0; pp < parts; ++pp) m = fmaxf(m, lse_parts[(size_t)pp * rows + row]);
  constexpr int kPer = D / 32;
  float acc[kPer];
  #pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float z = 0.f;
  for (int pp = 0; pp < parts; ++pp) {
    const float lp = lse_parts[(size_t)pp * rows + row];
    const float w = (lp == -INFINITY) ? 0.f : expf(lp - m);
    z += w;
    const float f = mode == 0 ? w : 1.f;
    const __nv_bfloat16* src = o_parts + ((size_t)pp * rows + row) * D + lane * kPer;
    #pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] += f * __bfloat162float(src[e]);
  }
  const float inv = mode == 0 ? 1.f / z : 1.f / (float)parts;
  __nv_bfloat16* dst = o + (size_t)row * D + lane * kPer;
  #pragma unroll
  for (int e = 0; e < kPer; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0) lse[row] = m + logf(z);
}

}  // namespace clear
