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
// a grid of a few thousand positions stays resident in L1 and L2. The data loads bypass L1 so that
// they do not evict it. The rotated values are rounded to bf16 once.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace clear {

struct RopeParams {
  const uint4* src[2];  // q, k: bf16 [BH][T][D] contiguous, as 16-byte chunks
  uint4* dst[2];        // rotated q, k, same layout
  const float4* tab;    // (cos, sin) table, see above
  long long chunks;     // chunks per tensor: BH * T * D / 8
  int T, n_text, W;     // tokens per (b, h), text tokens, grid width
};

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;
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

__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t rope_pair(uint32_t w, float co, float si) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xffff0000u);
  const __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(a, co, -b * si), fmaf(a, si, b * co));
  return *reinterpret_cast<const uint32_t*>(&r);
}

template <int D>
__global__ void __launch_bounds__(kRopeThreads) clear_rope_kernel(const RopeParams p) {
  constexpr int kC = D / 8;        // chunks per token
  constexpr int kCAxis = kC / 2;   // chunks per axis
  const long long total = 2 * p.chunks;
  const long long stride = (long long)gridDim.x * kRopeThreads;
  for (long long base = (long long)blockIdx.x * kRopeThreads + threadIdx.x; base < total;
       base += kRopeUnroll * stride) {
    uint4 w[kRopeUnroll];
    float4 c01[kRopeUnroll], c23[kRopeUnroll];
    bool rot[kRopeUnroll];
    #pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const long long i = base + u * stride;
      rot[u] = false;
      if (i >= total) continue;
      const int which = i >= p.chunks;
      const long long j = which ? i - p.chunks : i;
      w[u] = ld_stream_v4((which ? p.src[1] : p.src[0]) + j);
      const int c = (int)(j % kC);
      const int t = (int)((j / kC) % p.T);
      if (t >= p.n_text) {
        const int pi = t - p.n_text, y = pi / p.W, x = pi - y * p.W;
        const int axis = c >= kCAxis;
        const float4* e = p.tab + ((long long)(axis ? x : y) * kCAxis + (c - axis * kCAxis)) * 2;
        c01[u] = __ldg(e);
        c23[u] = __ldg(e + 1);
        rot[u] = true;
      }
    }
    #pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const long long i = base + u * stride;
      if (i >= total) continue;
      uint4 v = w[u];
      if (rot[u]) {
        v.x = rope_pair(v.x, c01[u].x, c01[u].y);
        v.y = rope_pair(v.y, c01[u].z, c01[u].w);
        v.z = rope_pair(v.z, c23[u].x, c23[u].y);
        v.w = rope_pair(v.w, c23[u].z, c23[u].w);
      }
      if (i >= p.chunks)
        p.dst[1][i - p.chunks] = v;
      else
        p.dst[0][i] = v;
    }
  }
}

}  // namespace clear
