// Axial 2D rotary position embedding of q and k on sm_100a: one streaming pass over each tensor,
// ahead of the CLEAR forward.
//
// Semantics: RoFormer's rotary embedding with NTK-aware scaled RoPE (the pith.science review of
// "CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion Transformers Up", "Assumptions & free
// parameters", lists an NTK-aware RoPE scale factor of 10 for the high-resolution runs), read for
// the token grid as axial 2D RoPE: image token (y, x) turns dims [0, d/2) by its row y and dims
// [d/2, d) by its column x, pair (2i, 2i+1) of an axis by position * base^(-2i/(d/2)) with the base
// theta * ntk^((d/2)/(d/2 - 2)): (a, b) -> (a cos - b sin, a sin + b cos). Text tokens are left
// as they are.
//
// HBM-bound: every 16-byte chunk (eight dims, four pairs) is read once and written once. Both axes
// share one (cos, sin) table, [positions][d/4 pairs] of (cos, sin), i.e. per 16-byte chunk of an
// axis two float4 {cos0, sin0, cos1, sin1}, {cos2, sin2, cos3, sin3}; it is built on the device in
// double (clear_rope_table_kernel) and stored as fp32, and read through the read-only path, where
// a grid of a few thousand positions stays resident in L1 and L2. The data itself moves by bulk
// copies through shared memory. The rotated values are rounded to bf16 once.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace clear {

constexpr int kRopeThreads = 256;  // table kernel
constexpr int kRopeMaxPairs = 32;  // pairs per axis at d = 128

struct RopeTableParams {
  float2* tab;                       // [n][np] (cos, sin)
  int n, np;                         // positions, pairs per axis (d/4)
  double inv_freq[kRopeMaxPairs];    // rotation rate of pair i: base^(-2i/(d/2))
};

// Entry (pos, i) = (cos, sin) of pos * inv_freq[i], evaluated in double and rounded to fp32.
__global__ void __launch_bounds__(kRopeThreads) clear_rope_table_kernel(const RopeTableParams p) {
  const int e = blockIdx.x * kRopeThreads + threadIdx.x;
  if (e >= p.n * p.np) return;
  const int pos = e / p.np, i = e - pos * p.np;
  double s, c;
  sincos((double)pos * p.inv_freq[i], &s, &c);
  p.tab[e] = make_float2((float)c, (float)s);
}

__device__ __forceinline__ uint32_t rope_pair(uint32_t w, float co, float si) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xffff0000u);
  const __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(a, co, -b * si), fmaf(a, si, b * co));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// ------------------------------------------------------------------------------------------------
// The rotation, streamed through shared memory with bulk asynchronous copies so that the bytes in
// flight do not live in registers: per block a ring of kRopeStages pieces of 16 KB (a contiguous
// stretch of q or k). Warp 8 loads each piece with one cp.async.bulk, the 256 threads of warps
// 0-7 rotate it in place (four independent 16-byte chunks each), and one of them writes it back
// with one bulk store. A stage goes back to the loader once its store has read it. Every wait is
// bounded.
// ------------------------------------------------------------------------------------------------
constexpr int kRopeBulkThreads = 288;  // warps 0-7 rotate, warp 8 loads
constexpr int kRopeRotThreads = 256;
constexpr int kRopePiece = 16384;
constexpr int kRopeStages = 4;  // 64 KB per block, three blocks per SM
constexpr int kRopeBulkSmem = kRopeStages * kRopePiece + 2 * kRopeStages * 8 + 16;
static_assert(kRopePiece % (128 * 2) == 0 && kRopePiece % (64 * 2) == 0, "pieces must start on token boundaries");

struct RopeBulkParams {
  const uint8_t* src[2];  // q, k: bf16 [BH][T][D] contiguous
  uint8_t* dst[2];        // rotated q, k, same layout (may be src: in place)
  const float4* tab;      // (cos, sin) table, see the top of this file
  long long bytes;        // bytes per tensor: BH * T * D * 2
  long long pieces;       // pieces per tensor: ceil(bytes / kRopePiece)
  int T, n_text, W;
  float sin_sign;
};

__device__ __forceinline__ void bulk_load_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void bulk_store_s2g(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(gdst), "r"(smem_u32(smem_src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Named barrier 1 over the 256 rotating threads; the _and form also returns whether every one of
// them passed true, so that they all leave the loop together when one wait has given up.
__device__ __forceinline__ void rope_bar_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool rope_bar_and(bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((uint32_t)v) : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(kRopeBulkThreads, 3) clear_rope_bulk_kernel(const RopeBulkParams p) {
  constexpr int kC = D / 8, kCAxis = kC / 2;
  extern __shared__ __align__(16) uint8_t rsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(rsm + kRopeStages * kRopePiece);
  uint64_t* empty = full + kRopeStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kRopeStages);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRopeStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const long long total = 2 * p.pieces;
  if (threadIdx.x >= kRopeRotThreads) {
    // ---- loader (one thread)
    if (threadIdx.x == kRopeRotThreads) {
      int j = 0;
      for (long long g = blockIdx.x; g < total; g += gridDim.x, ++j) {
        const int s = j % kRopeStages;
        if (!mbar_wait(&empty[s], ((j / kRopeStages) & 1) ^ 1, abort_flag, kDevTimeoutTmaEmpty, 26, j)) break;
        const int which = g >= p.pieces;
        const long long off = (which ? g - p.pieces : g) * kRopePiece;
        const uint32_t bytes = (uint32_t)(p.bytes - off < kRopePiece ? p.bytes - off : kRopePiece);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load_g2s(rsm + s * kRopePiece, (which ? p.src[1] : p.src[0]) + off, bytes, &full[s]);
      }
    }
    return;
  }
  // ---- rotation (warps 0-7) and the write-back (thread 0)
  const int tid = threadIdx.x;
  int j = 0;
  for (long long g = blockIdx.x; g < total; g += gridDim.x, ++j) {
    const int s = j % kRopeStages;
    const bool ok = mbar_wait(&full[s], (j / kRopeStages) & 1, abort_flag, kDevTimeoutTmaFull, 27, j);
    if (!rope_bar_and(ok)) break;
    const int which = g >= p.pieces;
    const long long off = (which ? g - p.pieces : g) * kRopePiece;
    const uint32_t bytes = (uint32_t)(p.bytes - off < kRopePiece ? p.bytes - off : kRopePiece);
    uint4* piece = reinterpret_cast<uint4*>(rsm + s * kRopePiece);
    // A piece starts on a token boundary (kRopePiece is a multiple of D * 2 bytes), so this thread's
    // chunks c = tid + 256 i (i < 4) keep one column and step 256 / kC tokens at a time.
    constexpr int kPer = kRopePiece / 16 / kRopeRotThreads;
    const int col = tid % kC;
    const int axis = col >= kCAxis;
    const int nch = (int)(bytes / 16);
    int t = (int)((off / (D * 2)) % p.T) + tid / kC;
    while (t >= p.T) t -= p.T;
    int tok[kPer];
    #pragma unroll
    for (int i = 0; i < kPer; ++i) {
      tok[i] = t;
      t += kRopeRotThreads / kC;
      while (t >= p.T) t -= p.T;
    }
    uint4 v[kPer];
    float4 c01[kPer], c23[kPer];
    bool rot[kPer];
    #pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int c = tid + i * kRopeRotThreads;
      rot[i] = c < nch && tok[i] >= p.n_text;
      if (rot[i]) {
        const int pi = tok[i] - p.n_text, y = pi / p.W, x = pi - y * p.W;
        const float4* e = p.tab + ((long long)(axis ? x : y) * kCAxis + (col - axis * kCAxis)) * 2;
        c01[i] = __ldg(e);
        c23[i] = __ldg(e + 1);
        v[i] = piece[c];
      }
    }
    const float sg = p.sin_sign;
    #pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (!rot[i]) continue;
      uint4 w = v[i];
      w.x = rope_pair(w.x, c01[i].x, sg * c01[i].y);
      w.y = rope_pair(w.y, c01[i].z, sg * c01[i].w);
      w.z = rope_pair(w.z, c23[i].x, sg * c23[i].y);
      w.w = rope_pair(w.w, c23[i].z, sg * c23[i].w);
      piece[tid + i * kRopeRotThreads] = w;
    }
    fence_proxy_async_smem();  // the rotated words, for the bulk store's reads
    rope_bar_sync();
    if (tid == 0) {
      bulk_store_s2g((which ? p.dst[1] : p.dst[0]) + off, piece, bytes);
      bulk_commit();
      bulk_wait_read<1>();  // the previous piece's store has read its stage: the loader may refill it
      if (j > 0) mbar_arrive(&empty[(j - 1) % kRopeStages]);
    }
  }
  if (tid == 0) bulk_wait_all();  // every store written before the kernel ends
}

}  // namespace clear
