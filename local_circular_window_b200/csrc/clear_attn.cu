// Host side of libclear_attn.so: argument validation, TMA tensor-map encoding, kernel launches and
// the host-only scheduler queries. The C ABI is declared in include/clear_attn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "clear_attn.h"
#include "clear_bwd.cuh"
#include "clear_fwd.cuh"
#include "clear_rope.cuh"
#include "clear_sched.cuh"

using namespace clear;

// Scratch of the allocation-free forward (clear_attn_fwd_noalloc): the text-row split partials.
// Every device that loads this library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kVersion = 112;  // 0.1.2: forward from host buffers

// ------------------------------------------------------------------------------------------------
// Validation
// ------------------------------------------------------------------------------------------------
struct Checked {
  clear_status_t st;
  Geom g;
};

// Radius beyond which every pair of the grid is kept; larger radii are clamped to it. Circle: the
// smallest r with r^2 above the squared diagonal; square: max(H, W).
int full_radius(int H, int W, int window) {
  if (window == kSquare) return H > W ? H : W;
  long long d2 = (long long)(H - 1) * (H - 1) + (long long)(W - 1) * (W - 1);
  long long r = (long long)std::sqrt((double)d2);
  while (r * r > d2) --r;
  while ((r + 1) * (r + 1) <= d2) ++r;
  return (int)(r + 1);  // (r+1)^2 > d2
}

Checked check_params(const clear_attn_params_t* p) {
  Checked c{};
  c.st = CLEAR_ERR_INVALID_ARG;
  if (!p) return c;
  if (p->B < 1 || p->heads < 1 || p->n_text < 0 || p->H < 1 || p->W < 1 || p->r < 1) return c;
  if (p->window != kCircle && p->window != kSquare && p->window != kShifted) return c;
  // The shifted window must fit in the grid: it is never clamped to a smaller radius.
  if (p->window == kShifted && (2 * (long long)p->r - 1 > p->H || 2 * (long long)p->r - 1 > p->W)) return c;
  if (p->d != 64 && p->d != 128) {
    c.st = CLEAR_ERR_UNSUPPORTED;
    return c;
  }
  const long long N = (long long)p->H * p->W;
  const long long T = N + p->n_text;
  const long long BH = (long long)p->B * p->heads;
  if (N > (1ll << 28) || p->n_text > (1 << 24) || T > (1ll << 30) || BH > (1ll << 20)) return c;
  if (BH * T * p->d >= (1ll << 40)) return c;
  const int rfull = p->window == kShifted ? p->r : full_radius(p->H, p->W, p->window);
  const int r = p->r < rfull ? p->r : rfull;
  if (hw_table_size(r, p->H) > kMaxHwTable) {  // half-width table must fit in shared memory
    c.st = CLEAR_ERR_UNSUPPORTED;
    return c;
  }
  c.g = make_geom(p->B, p->heads, p->n_text, p->H, p->W, p->d, r, p->window);
  c.st = CLEAR_OK;
  return c;
}

bool aligned16(const void* ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// The forward restricted to a stripe of the grid (patch-parallel inference): image query rows
// [q_row0, q_row1); text query rows see grid rows [key_row0, key_row1) and, if text_keys, the text
// tokens. The shifted window is not offered (its centre clamping would need the whole grid).
Checked check_stripe(const clear_attn_params_t* p, const clear_attn_stripe_t* s) {
  Checked c = check_params(p);
  if (c.st != CLEAR_OK) return c;
  c.st = CLEAR_ERR_INVALID_ARG;
  if (!s) return c;
  if (p->window == kShifted) {
    c.st = CLEAR_ERR_UNSUPPORTED;
    return c;
  }
  if (s->q_row0 < 0 || s->q_row0 >= s->q_row1 || s->q_row1 > p->H) return c;
  if (s->key_row0 < 0 || s->key_row0 > s->key_row1 || s->key_row1 > p->H) return c;
  if (s->text_keys != 0 && s->text_keys != 1) return c;
  if (p->n_text > 0 && !s->text_keys && s->key_row0 == s->key_row1) return c;  // text rows without keys
  const int tk_lo = p->n_text + s->key_row0 * p->W, tk_hi = p->n_text + s->key_row1 * p->W;
  set_text_key_ranges(&c.g, s->text_keys, tk_lo, tk_hi);
  set_forward_work(&c.g, s->q_row0, s->q_row1);
  balance_forward_splits(&c.g);
  c.st = CLEAR_OK;
  return c;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct FwdWorkspace {
  size_t opart_off, ml_off, total;
};

FwdWorkspace fwd_workspace_layout(const Geom& g) {
  FwdWorkspace w{};
  if (g.n_text == 0) return w;
  const size_t rows = (size_t)g.fS * g.BH * g.n_text;
  w.opart_off = 0;
  w.ml_off = align256(rows * g.d * sizeof(float));
  w.total = align256(w.ml_off + rows * sizeof(float2));
  return w;
}

// ------------------------------------------------------------------------------------------------
// Device checks and TMA descriptors
// ------------------------------------------------------------------------------------------------
clear_status_t check_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CLEAR_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  if (major != 10) return CLEAR_ERR_UNSUPPORTED;
  if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  return CLEAR_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [BH, T, d] viewed as a 3D tensor (d, T, BH); box = 64 x rows x 1, 128-byte swizzle.
bool make_linear_map(CUtensorMap* m, const void* base, const Geom& g, int rows = kTile) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.T, (cuuint64_t)g.BH};
  cuuint64_t strides[2] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.T * g.d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Image part of [BH, T, d] viewed as a 4D tensor (d, W, H, BH) starting at token n_text;
// box = 64 x 16 x rows x 1 (a rows x 16 grid rectangle), 128-byte swizzle, zero fill outside
// the grid.
bool make_image_map(CUtensorMap* m, const void* base, const Geom& g, int rows = kKH) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const char* img = static_cast<const char*>(base) + (size_t)g.n_text * g.d * 2;
  cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.BH};
  cuuint64_t strides[3] = {(cuuint64_t)g.d * 2, (cuuint64_t)g.W * g.d * 2, (cuuint64_t)g.T * g.d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)kKW, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<char*>(img), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct QKVMaps {
  CUtensorMap q_lin, q_img, k_lin, k_img, v_lin, v_img;
};

bool make_qkv_maps(QKVMaps* m, const void* q, const void* k, const void* v, const Geom& g) {
  return make_linear_map(&m->q_lin, q, g) && make_image_map(&m->q_img, q, g) &&
         make_linear_map(&m->k_lin, k, g) && make_image_map(&m->k_img, k, g) &&
         make_linear_map(&m->v_lin, v, g) && make_image_map(&m->v_img, v, g);
}

// Element strides of one [B, heads, T, d] view: batch, head, token (d is contiguous).
struct TensorStrides {
  long long sb, sh, st;
};

TensorStrides contiguous_strides(const Geom& g) {
  return TensorStrides{(long long)g.heads * g.T * g.d, (long long)g.T * g.d, (long long)g.d};
}

// Whether b*heads+h can be one axis of stride sh (then the forward uses the flat maps).
bool flat_bh(const TensorStrides& t, const Geom& g) { return g.B == 1 || t.sb == (long long)g.heads * t.sh; }

// Forward view of q, k or v. Flat: linear (d, T, B*heads) with box 64 x rows x 1 and image
// (d, W, H, B*heads) from token n_text with box 64 x 16 x rows x 1. Split: the same with separate
// head and batch axes, (d, T, heads, B) and (d, W, H, heads, B).
bool make_fwd_tensor_maps(CUtensorMap* lin, CUtensorMap* img, const void* base, const TensorStrides& t, const Geom& g,
                          int lin_rows, int img_rows, bool split) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t e = 2;  // bytes per element
  if (!split) {
    cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.T, (cuuint64_t)g.BH};
    cuuint64_t strides[2] = {(cuuint64_t)t.st * e, (cuuint64_t)t.sh * e};
    cuuint32_t box[3] = {64, (cuuint32_t)lin_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(lin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
    const char* ib = static_cast<const char*>(base) + (size_t)g.n_text * t.st * e;
    cuuint64_t idims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.BH};
    cuuint64_t istrides[3] = {(cuuint64_t)t.st * e, (cuuint64_t)g.W * t.st * e, (cuuint64_t)t.sh * e};
    cuuint32_t ibox[4] = {64, (cuuint32_t)kKW, (cuuint32_t)img_rows, 1};
    cuuint32_t iestr[4] = {1, 1, 1, 1};
    return enc(img, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<char*>(ib), idims, istrides, ibox, iestr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  {
    cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.T, (cuuint64_t)g.heads, (cuuint64_t)g.B};
    cuuint64_t strides[3] = {(cuuint64_t)t.st * e, (cuuint64_t)t.sh * e, (cuuint64_t)t.sb * e};
    cuuint32_t box[4] = {64, (cuuint32_t)lin_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(lin, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  const char* ib = static_cast<const char*>(base) + (size_t)g.n_text * t.st * e;
  cuuint64_t dims[5] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.heads, (cuuint64_t)g.B};
  cuuint64_t strides[4] = {(cuuint64_t)t.st * e, (cuuint64_t)g.W * t.st * e, (cuuint64_t)t.sh * e, (cuuint64_t)t.sb * e};
  cuuint32_t box[5] = {64, (cuuint32_t)kKW, (cuuint32_t)img_rows, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(img, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<char*>(ib), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Forward maps: 128-row query tiles, 64-key K/V tiles (64-token chunks and 4 x 16 rectangles).
bool make_fwd_maps(QKVMaps* m, const void* q, const void* k, const void* v, const TensorStrides* st,
                   const Geom& g, bool split) {
  return make_fwd_tensor_maps(&m->q_lin, &m->q_img, q, st[0], g, kTile, kQH, split) &&
         make_fwd_tensor_maps(&m->k_lin, &m->k_img, k, st[1], g, kFChunk, kFKH, split) &&
         make_fwd_tensor_maps(&m->v_lin, &m->v_img, v, st[2], g, kFChunk, kFKH, split);
}

// Strides the forward accepts: positive multiples of 8 elements (16 bytes, the TMA stride rule), so
// that every token row starts 16-byte aligned when the base is.
bool strides_ok(const TensorStrides& t) {
  return t.sb > 0 && t.sh > 0 && t.st > 0 && t.sb % 8 == 0 && t.sh % 8 == 0 && t.st % 8 == 0 &&
         t.sb < (1ll << 39) && t.sh < (1ll << 39) && t.st < (1ll << 39);
}

template <int D, bool kSplit>
clear_status_t launch_fwd(const Geom& g, const QKVMaps& m, void* o, const TensorStrides& os, float* lse, void* ws,
                          int num_sms, cudaStream_t stream) {
  using L = FwdLayout<D>;
  const int smem_bytes = L::alloc_bytes(hw_table_size(g.r, g.H));
  if (smem_bytes > 232448) return CLEAR_ERR_UNSUPPORTED;  // guarded by check_params
  FwdParams p{};
  p.g = g;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sb = os.sb;
  p.o_sh = os.sh;
  p.o_st = os.st;
  p.lse = lse;
  const FwdWorkspace wl = fwd_workspace_layout(g);
  p.opart = g.n_text ? reinterpret_cast<float*>(static_cast<char*>(ws) + wl.opart_off) : nullptr;
  p.wide_o = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 && os.sb % 16 == 0 && os.sh % 16 == 0 && os.st % 16 == 0;
  p.wide_part = (reinterpret_cast<uintptr_t>(p.opart) & 31u) == 0;
  p.ml = g.n_text ? reinterpret_cast<float2*>(static_cast<char*>(ws) + wl.ml_off) : nullptr;
  p.n_work = g.n_txt_pairs + g.n_img_pairs;
  if (cudaFuncSetAttribute(clear_fwd_kernel<D, kSplit, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_bytes) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  const long long grid = p.n_work < num_sms ? p.n_work : num_sms;
  clear_fwd_kernel<D, kSplit, false><<<(unsigned)grid, kFwdThreads, smem_bytes, stream>>>(
      m.q_lin, m.q_img, m.k_lin, m.k_img, m.v_lin, m.v_img, p);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  if (g.n_text > 0) {
    const long long rows = (long long)g.BH * g.n_text;
    const int wpb = 8;
    clear_fwd_combine_kernel<D, kSplit><<<(unsigned)((rows + wpb - 1) / wpb), wpb * 32, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  }
  return CLEAR_OK;
}

// E4M3 q or k (one byte per element, contiguous [B, heads, T, d] with d = 128): linear view
// (d, T, B*heads) with lin_rows-token boxes and image view (d, W, H, B*heads) with img_rows x 16
// boxes, each box one 128-byte row block (128-byte swizzle), as the bf16 maps but with one block.
bool make_e4m3_maps(CUtensorMap* lin, CUtensorMap* img, const void* base, const Geom& g, int lin_rows, int img_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.T, (cuuint64_t)g.BH};
  cuuint64_t strides[2] = {(cuuint64_t)g.d, (cuuint64_t)g.T * g.d};
  cuuint32_t box[3] = {(cuuint32_t)g.d, (cuuint32_t)lin_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (enc(lin, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const char* ib = static_cast<const char*>(base) + (size_t)g.n_text * g.d;
  cuuint64_t idims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.BH};
  cuuint64_t istrides[3] = {(cuuint64_t)g.d, (cuuint64_t)g.W * g.d, (cuuint64_t)g.T * g.d};
  cuuint32_t ibox[4] = {(cuuint32_t)g.d, (cuuint32_t)kKW, (cuuint32_t)img_rows, 1};
  cuuint32_t iestr[4] = {1, 1, 1, 1};
  return enc(img, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<char*>(ib), idims, istrides, ibox, iestr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The forward with E4M3 q, k (score products of kind::f8f6f4) and bf16 v; contiguous tensors.
clear_status_t launch_fwd_f8(const Geom& g, const void* q8, const void* k8, const void* v, const float* qk_descale,
                             void* o, float* lse, void* ws, int num_sms, cudaStream_t stream) {
  constexpr int D = 128;
  using L = FwdLayout<D, true>;
  QKVMaps m;
  const TensorStrides cs = contiguous_strides(g);
  if (!make_e4m3_maps(&m.q_lin, &m.q_img, q8, g, kTile, kQH) || !make_e4m3_maps(&m.k_lin, &m.k_img, k8, g, kFChunk, kFKH) ||
      !make_fwd_tensor_maps(&m.v_lin, &m.v_img, v, cs, g, kFChunk, kFKH, false))
    return CLEAR_ERR_CUDA;
  const int smem_bytes = L::alloc_bytes(hw_table_size(g.r, g.H));
  if (smem_bytes > 232448) return CLEAR_ERR_UNSUPPORTED;
  FwdParams p{};
  p.g = g;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sb = cs.sb;
  p.o_sh = cs.sh;
  p.o_st = cs.st;
  p.lse = lse;
  const FwdWorkspace wl = fwd_workspace_layout(g);
  p.opart = g.n_text ? reinterpret_cast<float*>(static_cast<char*>(ws) + wl.opart_off) : nullptr;
  p.ml = g.n_text ? reinterpret_cast<float2*>(static_cast<char*>(ws) + wl.ml_off) : nullptr;
  p.wide_o = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  p.wide_part = (reinterpret_cast<uintptr_t>(p.opart) & 31u) == 0;
  p.n_work = g.n_txt_pairs + g.n_img_pairs;
  p.qk_descale = qk_descale;
  if (cudaFuncSetAttribute(clear_fwd_kernel<D, false, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_bytes) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  const long long grid = p.n_work < num_sms ? p.n_work : num_sms;
  clear_fwd_kernel<D, false, false, true><<<(unsigned)grid, kFwdThreads, smem_bytes, stream>>>(
      m.q_lin, m.q_img, m.k_lin, m.k_img, m.v_lin, m.v_img, p);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  if (g.n_text > 0) {
    const long long rows = (long long)g.BH * g.n_text;
    const int wpb = 8;
    clear_fwd_combine_kernel<D, false><<<(unsigned)((rows + wpb - 1) / wpb), wpb * 32, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  }
  return CLEAR_OK;
}

// Rotary embedding: one (cos, sin) table for both axes, [max(H, W) positions][d/4 pairs]; pair i of
// an axis turns by position * base^(-2i/(d/2)) with the NTK-aware base theta * ntk^((d/2)/(d/2 - 2)).
struct RopeTable {
  int n = 0;
  size_t bytes = 0;
};

RopeTable rope_table_shape(const Geom& g) {
  RopeTable t;
  t.n = g.H > g.W ? g.H : g.W;
  t.bytes = (size_t)t.n * (g.d / 4) * sizeof(float2);
  return t;
}

// Workspace of the rotary forward: the forward's own, the table, the rotated q, the rotated k.
struct RopeWorkspace {
  size_t tab_off, q_off, k_off, total;
};

RopeWorkspace rope_workspace_layout(const Geom& g) {
  RopeWorkspace w;
  const size_t qk = (size_t)g.BH * g.T * g.d * sizeof(__nv_bfloat16);
  w.tab_off = align256(fwd_workspace_layout(g).total);
  w.q_off = w.tab_off + align256(rope_table_shape(g).bytes);
  w.k_off = w.q_off + align256(qk);
  w.total = w.k_off + align256(qk);
  return w;
}

size_t rope_workspace_bytes(const Geom& g) { return rope_workspace_layout(g).total; }

// The rotation streamed through shared memory: as many blocks as are resident at once (two per SM
// at 96 KB of shared memory each), each walking its pieces of q and k round-robin.
template <int D>
clear_status_t launch_rope_bulk(const RopeBulkParams& p, int num_sms, cudaStream_t stream) {
  if (cudaFuncSetAttribute(clear_rope_bulk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRopeBulkSmem) !=
      cudaSuccess)
    return CLEAR_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, clear_rope_bulk_kernel<D>, kRopeBulkThreads,
                                                    kRopeBulkSmem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const long long cap = (long long)num_sms * per_sm;
  const long long grid = 2 * p.pieces < cap ? 2 * p.pieces : cap;
  clear_rope_bulk_kernel<D><<<(unsigned)grid, kRopeBulkThreads, kRopeBulkSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? CLEAR_OK : CLEAR_ERR_CUDA;
}

// The (cos, sin) table into tab (rope_table_shape(g).bytes, 16-byte aligned), then q and k rotated
// into q_out and k_out (which may be q and k themselves: every 16-byte chunk is read and written by
// the same thread). inverse turns every pair back by the negated angle.
clear_status_t launch_rope(const Geom& g, const clear_attn_rope_t& rope, bool inverse, const void* q, const void* k,
                           void* q_out, void* k_out, void* tab, int num_sms, cudaStream_t stream) {
  RopeTableParams tp{};
  tp.tab = static_cast<float2*>(tab);
  tp.n = rope_table_shape(g).n;
  tp.np = g.d / 4;
  const int da = g.d / 2;
  const double rope_base = (double)rope.theta * std::pow((double)rope.ntk, (double)da / (da - 2.0));
  for (int i = 0; i < tp.np; ++i) tp.inv_freq[i] = std::pow(rope_base, -2.0 * i / da);
  clear_rope_table_kernel<<<(unsigned)((tp.n * tp.np + kRopeThreads - 1) / kRopeThreads), kRopeThreads, 0, stream>>>(
      tp);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  RopeBulkParams p{};
  p.src[0] = static_cast<const uint8_t*>(q);
  p.src[1] = static_cast<const uint8_t*>(k);
  p.dst[0] = static_cast<uint8_t*>(q_out);
  p.dst[1] = static_cast<uint8_t*>(k_out);
  p.tab = static_cast<const float4*>(tab);
  p.bytes = (long long)g.BH * g.T * g.d * 2;
  p.pieces = (p.bytes + kRopePiece - 1) / kRopePiece;
  p.T = g.T;
  p.n_text = g.n_text;
  p.W = g.W;
  p.sin_sign = inverse ? -1.f : 1.f;
  if (p.bytes == 0) return CLEAR_OK;
  return g.d == 128 ? launch_rope_bulk<128>(p, num_sms, stream) : launch_rope_bulk<64>(p, num_sms, stream);
}

bool rope_ok(const clear_attn_rope_t* rope) {
  return rope && std::isfinite(rope->theta) && rope->theta > 1.f && std::isfinite(rope->ntk) && rope->ntk > 0.f;
}

// Device address of g_noalloc_scratch on the current device. The symbol's name is only a host-side
// stand-in; the address is looked up with that device current and kept once the lookup succeeded.
// A failed lookup (e.g. the module could not be loaded because device memory was exhausted, or a
// capture was in progress) is not cached: the next call tries again. The error the failed call
// left behind is cleared so that it is not reported by an unrelated later call.
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

clear_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CLEAR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CLEAR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return CLEAR_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return CLEAR_OK;
}

// The forward's schedule with its text-row split count lowered until the partials fit in the
// static scratch; CLEAR_ERR_WORKSPACE when even one split does not fit.
clear_status_t noalloc_geom(Geom* g) {
  if (g->n_text == 0) return CLEAR_OK;
  for (int cap = g->fS; cap >= 1; --cap) {
    Geom t = *g;
    choose_splits(t.fnC, t.ftarget, cap, &t.fS, &t.fcps);
    t.n_txt_pairs = (long long)t.BH * t.nTq2 * t.fS;
    if (fwd_workspace_layout(t).total <= kNoAllocScratchBytes) {
      *g = t;
      return CLEAR_OK;
    }
  }
  return CLEAR_ERR_WORKSPACE;
}

// One thread waits on a barrier that nothing arrives on, gives up after limit_ns and records the
// expiry exactly as a timed-out wait of the attention kernels does (failure-detection self-test).
__global__ void clear_selftest_expiry_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t a = smem_u32(&bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, 0)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        record_timeout(&abort_flag, kDevTimeoutOther, 31, 0, (int)(limit_ns / 1000000ull), 0, 0);
        break;
      }
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------------------------------------
// Forward from host buffers: (batch, head) slices are split into groups; the host-to-device copy of
// group i+1, the forward of group i and the device-to-host copy of group i-1 run concurrently on
// two library-owned copy streams and the caller's stream.
// ------------------------------------------------------------------------------------------------
constexpr long long kHostMaxGroups = 24;

struct HostPlan {
  long long slices = 0, group = 0, n_groups = 0;
  size_t slice_bytes = 0, slice_lse_bytes = 0;  // one slice of q (k, v, o) and of lse
  size_t lse_group_bytes = 0;                   // one group's lse block on the device (256-aligned)
  size_t q_off = 0, k_off = 0, v_off = 0, o_off = 0, lse_off = 0, fws_off = 0, fws_bytes = 0, total = 0;
};

// Params of one group: `n` consecutive slices of the flat [B * heads] axis, as B = 1, heads = n.
clear_attn_params_t group_params(const clear_attn_params_t* p, long long n) {
  clear_attn_params_t gp = *p;
  gp.B = 1;
  gp.heads = (int)n;
  return gp;
}

bool host_plan(const clear_attn_params_t* p, const Geom& g, HostPlan* hp) {
  hp->slices = g.BH;
  hp->group = (g.BH + kHostMaxGroups - 1) / kHostMaxGroups;
  hp->n_groups = (g.BH + hp->group - 1) / hp->group;
  hp->slice_bytes = (size_t)g.T * g.d * 2;
  hp->slice_lse_bytes = (size_t)g.T * sizeof(float);
  const size_t tens = align256(hp->slice_bytes * g.BH);
  hp->q_off = 0;
  hp->k_off = tens;
  hp->v_off = 2 * tens;
  hp->o_off = 3 * tens;
  hp->lse_off = 4 * tens;
  // Each group's lse gets its own aligned block: a slice of lse (T floats) is not a multiple of
  // 16 bytes in general, and the forward wants an aligned lse pointer.
  hp->lse_group_bytes = align256(hp->slice_lse_bytes * hp->group);
  hp->fws_off = hp->lse_off + hp->lse_group_bytes * hp->n_groups;
  const clear_attn_params_t gp = group_params(p, hp->group);
  const Checked c = check_params(&gp);
  if (c.st != CLEAR_OK) return false;
  hp->fws_bytes = fwd_workspace_layout(c.g).total;  // the largest group's; reused group after group
  hp->total = hp->fws_off + align256(hp->fws_bytes);
  return true;
}

// True iff both ends of [ptr, ptr + bytes) lie in page-locked host memory (cudaHostAlloc'd or
// cudaHostRegister'ed), which asynchronous copies need to overlap anything.
bool page_locked(const void* ptr, size_t bytes) {
  const char* ends[2] = {static_cast<const char*>(ptr), static_cast<const char*>(ptr) + bytes - 1};
  for (const char* a : ends) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, a) != cudaSuccess) {
      cudaGetLastError();  // clear the error state the failed query leaves behind
      return false;
    }
    if (at.type != cudaMemoryTypeHost) return false;
  }
  return true;
}

// Two non-blocking copy streams per device, created on first use and kept for the process.
clear_status_t copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static cudaStream_t streams[kMaxDevices][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CLEAR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CLEAR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 2; ++i)
    if (!streams[dev][i] && cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking) != cudaSuccess)
      return CLEAR_ERR_CUDA;
  *h2d = streams[dev][0];
  *d2h = streams[dev][1];
  return CLEAR_OK;
}

// The forward on tensors with the given strides (q, k, v, o), once the arguments are checked.
clear_status_t run_fwd(const Geom& g, const TensorStrides* st4, const void* q, const void* k, const void* v, void* o,
                       float* lse, void* workspace, cudaStream_t s) {
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  const bool split = !(flat_bh(st4[0], g) && flat_bh(st4[1], g) && flat_bh(st4[2], g) && flat_bh(st4[3], g));
  QKVMaps maps;
  if (!make_fwd_maps(&maps, q, k, v, st4, g, split)) return CLEAR_ERR_CUDA;
  if (split)
    return g.d == 128 ? launch_fwd<128, true>(g, maps, o, st4[3], lse, workspace, num_sms, s)
                      : launch_fwd<64, true>(g, maps, o, st4[3], lse, workspace, num_sms, s);
  return g.d == 128 ? launch_fwd<128, false>(g, maps, o, st4[3], lse, workspace, num_sms, s)
                    : launch_fwd<64, false>(g, maps, o, st4[3], lse, workspace, num_sms, s);
}

// ------------------------------------------------------------------------------------------------
// Mixed-resolution batch: items of their own (n_text, H, W) packed along the token axis of
// [heads, tok_total, d] tensors, all of them in one forward launch.
// ------------------------------------------------------------------------------------------------
constexpr int kMaxVarlenItems = 4096;

struct VarlenPlan {
  std::vector<Geom> items;
  std::vector<long long> wbound;  // 2 * n + 1 pair bounds (text pairs of each item, then image pairs, then the total)
  Geom shared;                    // what the items share, with the largest H (the half-width table's size)
  long long n_pairs = 0, text_rows = 0, part_rows = 0;
  size_t maps_off = 0, bound_off = 0, opart_off = 0, ml_off = 0, staged = 0, total = 0;
};

clear_status_t plan_varlen(const clear_attn_params_t* p, int n_items, const int* shapes, VarlenPlan* v) {
  if (!p || !shapes || n_items < 1 || n_items > kMaxVarlenItems) return CLEAR_ERR_INVALID_ARG;
  // One radius for every item: the request clamped to the largest full-grid radius among them. An
  // item whose own full radius is smaller keeps all its pairs either way.
  int rmax_full = 1;
  long long tok = 0;
  int max_h = 1;
  for (int i = 0; i < n_items; ++i) {
    clear_attn_params_t ip = *p;
    ip.B = 1;
    ip.n_text = shapes[3 * i];
    ip.H = shapes[3 * i + 1];
    ip.W = shapes[3 * i + 2];
    const Checked c = check_params(&ip);
    if (c.st != CLEAR_OK) return c.st;
    if (p->window != kShifted) {
      const int rf = full_radius(ip.H, ip.W, p->window);
      rmax_full = rf > rmax_full ? rf : rmax_full;
    }
    tok += c.g.T;
    max_h = ip.H > max_h ? ip.H : max_h;
  }
  if (tok > (1ll << 30) || (long long)p->heads * tok * p->d >= (1ll << 40)) return CLEAR_ERR_INVALID_ARG;
  const int r = p->window == kShifted ? p->r : (p->r < rmax_full ? p->r : rmax_full);
  if (hw_table_size(r, max_h) > kMaxHwTable) return CLEAR_ERR_UNSUPPORTED;
  v->items.resize(n_items);
  // Text splits by the plain rule: the launch deals every item's pairs round-robin as one list, so
  // there are many items per SM and the split-balancing model (made for one item alone) only adds
  // partial writes; measured on five FLUX-shaped mixes, the plain rule was as fast or 0.2-5 % faster.
  for (int i = 0; i < n_items; ++i) {
    v->items[i] = make_geom(1, p->heads, shapes[3 * i], shapes[3 * i + 1], shapes[3 * i + 2], p->d, r, p->window);
    plain_forward_splits(&v->items[i]);
  }
  v->wbound.assign(2 * (size_t)n_items + 1, 0);
  long long t0 = 0, part = 0, crow = 0, wt = 0;
  for (int i = 0; i < n_items; ++i) {
    Geom g = v->items[i];
    g.t0 = (int)t0;
    g.tok_total = tok;
    g.part_row0 = part;
    g.crow0 = crow;
    t0 += g.T;
    part += (long long)g.fS * g.BH * g.n_text;
    crow += (long long)g.BH * g.n_text;
    v->wbound[i] = wt;
    wt += g.n_txt_pairs;
    v->items[i] = g;
  }
  for (int i = 0; i < n_items; ++i) {
    v->wbound[n_items + i] = wt;
    wt += v->items[i].n_img_pairs;
  }
  v->wbound[2 * n_items] = wt;
  v->n_pairs = wt;
  v->text_rows = crow;
  v->part_rows = part;
  v->shared = make_geom(1, p->heads, 0, max_h, 1, p->d, r, p->window);
  v->shared.tok_total = tok;
  // Workspace: the item geometries, the image tensor maps (q, k, v per item), the pair bounds (all
  // three copied from the host before the launch), then the text rows' split partials.
  v->maps_off = align256(sizeof(Geom) * n_items);
  v->bound_off = align256(v->maps_off + sizeof(CUtensorMap) * 3 * (size_t)n_items);
  v->staged = v->bound_off + sizeof(long long) * v->wbound.size();
  v->opart_off = align256(v->staged);
  v->ml_off = align256(v->opart_off + (size_t)part * p->d * sizeof(float));
  v->total = align256(v->ml_off + (size_t)part * sizeof(float2));
  return CLEAR_OK;
}

template <int D>
clear_status_t launch_fwd_varlen(const VarlenPlan& v, const QKVMaps& maps, void* o, float* lse, void* ws, int num_sms,
                                 cudaStream_t stream) {
  using L = FwdLayout<D>;
  const Geom& g = v.shared;
  const int smem_bytes = L::alloc_bytes(hw_table_size(g.r, g.H));
  if (smem_bytes > 232448) return CLEAR_ERR_UNSUPPORTED;
  FwdParams p{};
  p.g = g;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sh = g.tok_total * D;
  p.o_sb = (long long)g.heads * p.o_sh;
  p.o_st = D;
  p.lse = lse;
  char* w = static_cast<char*>(ws);
  p.opart = v.part_rows ? reinterpret_cast<float*>(w + v.opart_off) : nullptr;
  p.ml = v.part_rows ? reinterpret_cast<float2*>(w + v.ml_off) : nullptr;
  p.wide_o = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  p.wide_part = (reinterpret_cast<uintptr_t>(p.opart) & 31u) == 0;
  p.n_work = v.n_pairs;
  p.items = reinterpret_cast<const Geom*>(w);
  p.item_maps = reinterpret_cast<const CUtensorMap*>(w + v.maps_off);
  p.wbound = reinterpret_cast<const long long*>(w + v.bound_off);
  p.n_items = (int)v.items.size();
  if (cudaFuncSetAttribute(clear_fwd_kernel<D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_bytes) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  const long long grid = p.n_work < num_sms ? p.n_work : num_sms;
  clear_fwd_kernel<D, false, true><<<(unsigned)grid, kFwdThreads, smem_bytes, stream>>>(
      maps.q_lin, maps.q_img, maps.k_lin, maps.k_img, maps.v_lin, maps.v_img, p);
  if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  if (v.text_rows > 0) {
    const int wpb = 8;
    clear_fwd_combine_varlen_kernel<D><<<(unsigned)((v.text_rows + wpb - 1) / wpb), wpb * 32, 0, stream>>>(p, v.text_rows);
    if (cudaGetLastError() != cudaSuccess) return CLEAR_ERR_CUDA;
  }
  return CLEAR_OK;
}

clear_status_t run_fwd_varlen(const VarlenPlan& v, const void* q, const void* k, const void* v_ptr, void* o,
                              float* lse, void* workspace, cudaStream_t s) {
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  const Geom& g = v.shared;
  // Token-axis (linear) maps over the whole batch: a problem of one grid row of tok_total tokens.
  const Geom gl = make_geom(1, g.heads, 0, 1, (int)g.tok_total, g.d, 1, kCircle);
  const TensorStrides ts = contiguous_strides(gl);
  const TensorStrides st4[4] = {ts, ts, ts, ts};
  QKVMaps maps;
  if (!make_fwd_maps(&maps, q, k, v_ptr, st4, gl, false)) return CLEAR_ERR_CUDA;
  // Staged part of the workspace: geometries, per-item image maps, pair bounds.
  const size_t n = v.items.size();
  std::vector<unsigned char> host(v.staged, 0);
  std::memcpy(host.data(), v.items.data(), sizeof(Geom) * n);
  CUtensorMap* hm = reinterpret_cast<CUtensorMap*>(host.data() + v.maps_off);
  const void* bases[3] = {q, k, v_ptr};
  const int img_rows[3] = {kQH, kFKH, kFKH};
  const int lin_rows[3] = {kTile, kFChunk, kFChunk};
  for (size_t i = 0; i < n; ++i) {
    const Geom& gi = v.items[i];
    for (int t = 0; t < 3; ++t) {
      CUtensorMap lin_unused;
      const char* base = static_cast<const char*>(bases[t]) + (size_t)gi.t0 * g.d * 2;
      if (!make_fwd_tensor_maps(&lin_unused, &hm[3 * i + t], base, ts, gi, lin_rows[t], img_rows[t], false))
        return CLEAR_ERR_CUDA;
    }
  }
  std::memcpy(host.data() + v.bound_off, v.wbound.data(), sizeof(long long) * v.wbound.size());
  if (cudaMemcpyAsync(workspace, host.data(), host.size(), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  return g.d == 128 ? launch_fwd_varlen<128>(v, maps, o, lse, workspace, num_sms, s)
                    : launch_fwd_varlen<64>(v, maps, o, lse, workspace, num_sms, s);
}

}  // namespace

// ------------------------------------------------------------------------------------------------
// C ABI
// ------------------------------------------------------------------------------------------------
extern "C" {

int clear_attn_version(void) { return kVersion; }

const char* clear_status_string(clear_status_t s) {
  switch (s) {
    case CLEAR_OK: return "CLEAR_OK";
    case CLEAR_ERR_INVALID_ARG: return "CLEAR_ERR_INVALID_ARG";
    case CLEAR_ERR_UNSUPPORTED: return "CLEAR_ERR_UNSUPPORTED";
    case CLEAR_ERR_WORKSPACE: return "CLEAR_ERR_WORKSPACE";
    case CLEAR_ERR_CUDA: return "CLEAR_ERR_CUDA";
    case CLEAR_ERR_DEVICE_TIMEOUT: return "CLEAR_ERR_DEVICE_TIMEOUT";
  }
  return "CLEAR_ERR_UNKNOWN";
}

size_t clear_attn_fwd_workspace_size(const clear_attn_params_t* params, clear_status_t* status) {
  const Checked c = check_params(params);
  if (status) *status = c.st;
  if (c.st != CLEAR_OK) return 0;
  return fwd_workspace_layout(c.g).total;
}

size_t clear_attn_bwd_workspace_size(const clear_attn_params_t* params, clear_status_t* status) {
  const Checked c = check_params(params);
  const clear_status_t st = (c.st == CLEAR_OK && c.g.window == kShifted) ? CLEAR_ERR_UNSUPPORTED : c.st;
  if (status) *status = st;
  if (st != CLEAR_OK) return 0;
  return bwd_workspace_layout(c.g).total;
}

clear_status_t clear_attn_fwd(const clear_attn_params_t* params, const void* q, const void* k,
                              const void* v, void* o, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CLEAR_ERR_INVALID_ARG;
  const size_t need = fwd_workspace_layout(c.g).total;
  if (need > 0 && (workspace_bytes < need || !aligned16(workspace))) return CLEAR_ERR_WORKSPACE;
  const TensorStrides cs = contiguous_strides(c.g);
  const TensorStrides st4[4] = {cs, cs, cs, cs};
  return run_fwd(c.g, st4, q, k, v, o, lse, workspace, static_cast<cudaStream_t>(stream));
}

clear_status_t clear_attn_fwd_strided(const clear_attn_params_t* params, const clear_attn_strides_t* strides,
                                      const void* q, const void* k, const void* v, void* o, float* lse,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (!strides || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CLEAR_ERR_INVALID_ARG;
  const TensorStrides st4[4] = {{strides->q[0], strides->q[1], strides->q[2]},
                                {strides->k[0], strides->k[1], strides->k[2]},
                                {strides->v[0], strides->v[1], strides->v[2]},
                                {strides->o[0], strides->o[1], strides->o[2]}};
  for (const TensorStrides& t : st4)
    if (!strides_ok(t)) return CLEAR_ERR_UNSUPPORTED;
  const size_t need = fwd_workspace_layout(c.g).total;
  if (need > 0 && (workspace_bytes < need || !aligned16(workspace))) return CLEAR_ERR_WORKSPACE;
  return run_fwd(c.g, st4, q, k, v, o, lse, workspace, static_cast<cudaStream_t>(stream));
}

size_t clear_attn_fwd_stripe_workspace_size(const clear_attn_params_t* params, const clear_attn_stripe_t* stripe,
                                            clear_status_t* status) {
  const Checked c = check_stripe(params, stripe);
  if (status) *status = c.st;
  if (c.st != CLEAR_OK) return 0;
  return fwd_workspace_layout(c.g).total;
}

clear_status_t clear_attn_fwd_stripe(const clear_attn_params_t* params, const clear_attn_stripe_t* stripe,
                                     const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  const Checked c = check_stripe(params, stripe);
  if (c.st != CLEAR_OK) return c.st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CLEAR_ERR_INVALID_ARG;
  const size_t need = fwd_workspace_layout(c.g).total;
  if (need > 0 && (workspace_bytes < need || !aligned16(workspace))) return CLEAR_ERR_WORKSPACE;
  const TensorStrides cs = contiguous_strides(c.g);
  const TensorStrides st4[4] = {cs, cs, cs, cs};
  return run_fwd(c.g, st4, q, k, v, o, lse, workspace, static_cast<cudaStream_t>(stream));
}

clear_status_t clear_attn_fwd_fp8(const clear_attn_params_t* params, const void* q8, const void* k8, const void* v,
                                  const float* qk_descale, void* o, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (params->d != 128) return CLEAR_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !qk_descale ||
      (reinterpret_cast<uintptr_t>(qk_descale) & 3u) != 0)
    return CLEAR_ERR_INVALID_ARG;
  const size_t need = fwd_workspace_layout(c.g).total;
  if (need > 0 && (workspace_bytes < need || !aligned16(workspace))) return CLEAR_ERR_WORKSPACE;
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  return launch_fwd_f8(c.g, q8, k8, v, qk_descale, o, lse, workspace, num_sms, static_cast<cudaStream_t>(stream));
}

size_t clear_attn_fwd_rope_workspace_size(const clear_attn_params_t* params, clear_status_t* status) {
  const Checked c = check_params(params);
  if (status) *status = c.st;
  if (c.st != CLEAR_OK) return 0;
  return rope_workspace_bytes(c.g);
}

clear_status_t clear_attn_fwd_rope(const clear_attn_params_t* params, const clear_attn_rope_t* rope, const void* q,
                                   const void* k, const void* v, void* o, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (!rope_ok(rope)) return CLEAR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CLEAR_ERR_INVALID_ARG;
  if (workspace_bytes < rope_workspace_bytes(c.g) || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return CLEAR_ERR_WORKSPACE;
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const RopeWorkspace wl = rope_workspace_layout(c.g);
  char* base = static_cast<char*>(workspace);
  const clear_status_t rs = launch_rope(c.g, *rope, false, q, k, base + wl.q_off, base + wl.k_off, base + wl.tab_off,
                                        num_sms, s);
  if (rs != CLEAR_OK) return rs;
  const TensorStrides cs = contiguous_strides(c.g);
  const TensorStrides st4[4] = {cs, cs, cs, cs};
  return run_fwd(c.g, st4, base + wl.q_off, base + wl.k_off, v, o, lse, workspace, s);
}

size_t clear_attn_rope_workspace_size(const clear_attn_params_t* params, clear_status_t* status) {
  const Checked c = check_params(params);
  if (status) *status = c.st;
  if (c.st != CLEAR_OK) return 0;
  return align256(rope_table_shape(c.g).bytes);
}

clear_status_t clear_attn_rope(const clear_attn_params_t* params, const clear_attn_rope_t* rope, int inverse,
                               const void* q, const void* k, void* q_out, void* k_out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (!rope_ok(rope) || (inverse != 0 && inverse != 1)) return CLEAR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out)) return CLEAR_ERR_INVALID_ARG;
  if (workspace_bytes < align256(rope_table_shape(c.g).bytes) || !workspace ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return CLEAR_ERR_WORKSPACE;
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  return launch_rope(c.g, *rope, inverse != 0, q, k, q_out, k_out, workspace, num_sms, static_cast<cudaStream_t>(stream));
}

size_t clear_attn_fwd_varlen_workspace_size(const clear_attn_params_t* params, int n_items, const int* item_shapes,
                                            clear_status_t* status) {
  VarlenPlan v;
  const clear_status_t st = plan_varlen(params, n_items, item_shapes, &v);
  if (status) *status = st;
  return st == CLEAR_OK ? v.total : 0;
}

clear_status_t clear_attn_fwd_varlen(const clear_attn_params_t* params, int n_items, const int* item_shapes,
                                     const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  VarlenPlan plan;
  const clear_status_t st = plan_varlen(params, n_items, item_shapes, &plan);
  if (st != CLEAR_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CLEAR_ERR_INVALID_ARG;
  if (workspace_bytes < plan.total || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return CLEAR_ERR_WORKSPACE;
  return run_fwd_varlen(plan, q, k, v, o, lse, workspace, static_cast<cudaStream_t>(stream));
}

clear_status_t clear_attn_text_merge(const clear_attn_params_t* params, int n_parts, int mode, const void* o_parts,
                                     const float* lse_parts, void* o, float* lse, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (n_parts < 1 || n_parts > 4096 || (mode != 0 && mode != 1) || c.g.n_text == 0) return CLEAR_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(o) || !aligned16(lse)) return CLEAR_ERR_INVALID_ARG;
  const long long rows = (long long)c.g.BH * c.g.n_text;
  if (rows * n_parts >= (1ll << 31)) return CLEAR_ERR_INVALID_ARG;
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  const int wpb = 8;
  const unsigned blocks = (unsigned)((rows + wpb - 1) / wpb);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* op = static_cast<const __nv_bfloat16*>(o_parts);
  __nv_bfloat16* oo = static_cast<__nv_bfloat16*>(o);
  if (c.g.d == 128)
    clear_text_merge_kernel<128><<<blocks, wpb * 32, 0, s>>>((int)rows, n_parts, mode, op, lse_parts, oo, lse);
  else
    clear_text_merge_kernel<64><<<blocks, wpb * 32, 0, s>>>((int)rows, n_parts, mode, op, lse_parts, oo, lse);
  return cudaGetLastError() == cudaSuccess ? CLEAR_OK : CLEAR_ERR_CUDA;
}

clear_status_t clear_attn_fwd_noalloc(const clear_attn_params_t* params, const void* q, const void* k,
                                      const void* v, void* o, float* lse, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return CLEAR_ERR_INVALID_ARG;
  Geom g = c.g;
  clear_status_t st = noalloc_geom(&g);
  if (st != CLEAR_OK) return st;
  int num_sms = 0;
  st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != CLEAR_OK) return st;
  const TensorStrides cs = contiguous_strides(g);
  const TensorStrides st4[4] = {cs, cs, cs, cs};
  return run_fwd(g, st4, q, k, v, o, lse, scratch, static_cast<cudaStream_t>(stream));
}

size_t clear_attn_fwd_host_workspace_size(const clear_attn_params_t* params, clear_status_t* status) {
  const Checked c = check_params(params);
  HostPlan hp;
  clear_status_t st = c.st;
  if (st == CLEAR_OK && !host_plan(params, c.g, &hp)) st = CLEAR_ERR_INVALID_ARG;
  if (status) *status = st;
  return st == CLEAR_OK ? hp.total : 0;
}

clear_status_t clear_attn_fwd_host(const clear_attn_params_t* params, const void* q_host, const void* k_host,
                                   const void* v_host, void* o_host, float* lse_host, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (!aligned16(q_host) || !aligned16(k_host) || !aligned16(v_host) || !aligned16(o_host) ||
      !aligned16(lse_host))
    return CLEAR_ERR_INVALID_ARG;
  HostPlan hp;
  if (!host_plan(params, c.g, &hp)) return CLEAR_ERR_INVALID_ARG;
  if (workspace_bytes < hp.total || !aligned16(workspace)) return CLEAR_ERR_WORKSPACE;
  int num_sms = 0;
  clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  const size_t tens = hp.slice_bytes * hp.slices, lse_bytes = hp.slice_lse_bytes * hp.slices;
  if (!page_locked(q_host, tens) || !page_locked(k_host, tens) || !page_locked(v_host, tens) ||
      !page_locked(o_host, tens) || !page_locked(lse_host, lse_bytes))
    return CLEAR_ERR_INVALID_ARG;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  st = copy_streams(&h2d, &d2h);
  if (st != CLEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);

  // Events: [0] entry on the caller's stream, [1] all returns copied, then per group "inputs in"
  // and "outputs ready".
  const long long n_ev = 2 + 2 * hp.n_groups;
  cudaEvent_t* ev = new (std::nothrow) cudaEvent_t[n_ev];
  if (!ev) return CLEAR_ERR_CUDA;
  long long made = 0;
  for (; made < n_ev; ++made)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) break;
  bool ok = made == n_ev;
  auto cu = [&ok](cudaError_t e) { if (e != cudaSuccess) ok = false; return ok; };
  // Copies start after the work already queued on the caller's stream (an earlier call may still
  // read the device buffers this one overwrites).
  if (ok && cu(cudaEventRecord(ev[0], s)) && cu(cudaStreamWaitEvent(h2d, ev[0], 0)))
    cu(cudaStreamWaitEvent(d2h, ev[0], 0));
  for (long long gi = 0; ok && gi < hp.n_groups; ++gi) {
    const long long s0 = gi * hp.group;
    const long long n = (hp.slices - s0 < hp.group) ? hp.slices - s0 : hp.group;
    const size_t off = hp.slice_bytes * s0, bytes = hp.slice_bytes * n;
    const size_t loff = hp.slice_lse_bytes * s0, lbytes = hp.slice_lse_bytes * n;
    cudaEvent_t in = ev[2 + 2 * gi], out = ev[3 + 2 * gi];
    char *dq = ws + hp.q_off + off, *dk = ws + hp.k_off + off, *dv = ws + hp.v_off + off;
    char *dout = ws + hp.o_off + off, *dlse = ws + hp.lse_off + hp.lse_group_bytes * gi;
    const cudaMemcpyKind up = cudaMemcpyHostToDevice, down = cudaMemcpyDeviceToHost;
    if (!(cu(cudaMemcpyAsync(dq, static_cast<const char*>(q_host) + off, bytes, up, h2d)) &&
          cu(cudaMemcpyAsync(dk, static_cast<const char*>(k_host) + off, bytes, up, h2d)) &&
          cu(cudaMemcpyAsync(dv, static_cast<const char*>(v_host) + off, bytes, up, h2d)) &&
          cu(cudaEventRecord(in, h2d)) && cu(cudaStreamWaitEvent(s, in, 0))))
      break;
    const clear_attn_params_t gp = group_params(params, n);
    st = clear_attn_fwd(&gp, dq, dk, dv, dout, reinterpret_cast<float*>(dlse), ws + hp.fws_off, hp.fws_bytes, stream);
    if (st != CLEAR_OK) {
      ok = false;
      break;
    }
    if (!(cu(cudaEventRecord(out, s)) && cu(cudaStreamWaitEvent(d2h, out, 0)) &&
          cu(cudaMemcpyAsync(static_cast<char*>(o_host) + off, dout, bytes, down, d2h)) &&
          cu(cudaMemcpyAsync(reinterpret_cast<char*>(lse_host) + loff, dlse, lbytes, down, d2h))))
      break;
  }
  // Work queued on the caller's stream from here on runs after every return copy.
  if (made == n_ev) {
    if (cudaEventRecord(ev[1], d2h) != cudaSuccess || cudaStreamWaitEvent(s, ev[1], 0) != cudaSuccess) ok = false;
  }
  for (long long i = 0; i < made; ++i) cudaEventDestroy(ev[i]);  // released once their work completes
  delete[] ev;
  if (st != CLEAR_OK) return st;
  return ok ? CLEAR_OK : CLEAR_ERR_CUDA;
}

clear_status_t clear_attn_bwd(const clear_attn_params_t* params, const void* q, const void* k,
                              const void* v, const void* o, const float* lse, const void* dO,
                              void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                              void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  // The shifted window's mask is not symmetric, which the KV-stationary dK/dV kernel relies on.
  if (c.g.window == kShifted) return CLEAR_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return CLEAR_ERR_INVALID_ARG;
  const BwdWorkspace wl = bwd_workspace_layout(c.g);
  if (workspace_bytes < wl.total || !aligned16(workspace)) return CLEAR_ERR_WORKSPACE;
  int num_sms = 0;
  clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  QKVMaps maps;
  if (!make_qkv_maps(&maps, q, k, v, c.g)) return CLEAR_ERR_CUDA;
  CUtensorMap do_lin, do_img;
  if (!make_linear_map(&do_lin, dO, c.g) || !make_image_map(&do_img, dO, c.g)) return CLEAR_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BwdArgs a{};
  a.g = c.g;
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.dO = static_cast<const __nv_bfloat16*>(dO);
  a.lse = lse;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.ws = static_cast<char*>(workspace);
  a.wl = wl;
  return c.g.d == 128 ? launch_bwd<128>(a, maps.q_lin, maps.q_img, maps.k_lin, maps.k_img, maps.v_lin,
                                        maps.v_img, do_lin, do_img, num_sms, s)
                      : launch_bwd<64>(a, maps.q_lin, maps.q_img, maps.k_lin, maps.k_img, maps.v_lin,
                                       maps.v_img, do_lin, do_img, num_sms, s);
}

// Backward through the rotary embedding: [backward workspace][table][rotated q][rotated k].
struct BwdRopeWorkspace {
  size_t tab_off, q_off, k_off, total;
};

BwdRopeWorkspace bwd_rope_workspace_layout(const Geom& g) {
  BwdRopeWorkspace w;
  const size_t qk = (size_t)g.BH * g.T * g.d * sizeof(__nv_bfloat16);
  w.tab_off = align256(bwd_workspace_layout(g).total);
  w.q_off = w.tab_off + align256(rope_table_shape(g).bytes);
  w.k_off = w.q_off + align256(qk);
  w.total = w.k_off + align256(qk);
  return w;
}

size_t clear_attn_bwd_rope_workspace_size(const clear_attn_params_t* params, clear_status_t* status) {
  const Checked c = check_params(params);
  if (status) *status = c.st;
  if (c.st != CLEAR_OK) return 0;
  return bwd_rope_workspace_layout(c.g).total;
}

clear_status_t clear_attn_bwd_rope(const clear_attn_params_t* params, const clear_attn_rope_t* rope, const void* q,
                                   const void* k, const void* v, const void* o, const float* lse, const void* dO,
                                   void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (c.g.window == kShifted) return CLEAR_ERR_UNSUPPORTED;
  if (!rope_ok(rope)) return CLEAR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return CLEAR_ERR_INVALID_ARG;
  const BwdRopeWorkspace wl = bwd_rope_workspace_layout(c.g);
  if (workspace_bytes < wl.total || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return CLEAR_ERR_WORKSPACE;
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  // q, k rotated as the forward saw them; the backward on the rotated tensors; then dQ, dK carried
  // back through the rotation by its transpose, in place.
  clear_status_t rs = launch_rope(c.g, *rope, false, q, k, base + wl.q_off, base + wl.k_off, base + wl.tab_off,
                                  num_sms, s);
  if (rs != CLEAR_OK) return rs;
  rs = clear_attn_bwd(params, base + wl.q_off, base + wl.k_off, v, o, lse, dO, dq, dk, dv, workspace, wl.tab_off,
                      stream);
  if (rs != CLEAR_OK) return rs;
  return launch_rope(c.g, *rope, true, dq, dk, dq, dk, base + wl.tab_off, num_sms, s);
}

static thread_local int t_last_diag[8] = {0, 0, 0, 0, 0, 0, 0, 0};

clear_status_t clear_attn_check(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CLEAR_ERR_CUDA;
  int err = 0;
  if (cudaMemcpyFromSymbol(&err, clear::g_clear_device_error, sizeof(int)) != cudaSuccess)
    return CLEAR_ERR_CUDA;
  if (err != 0) {
    if (cudaMemcpyFromSymbol(t_last_diag, clear::g_clear_device_diag, sizeof(t_last_diag)) != cudaSuccess)
      return CLEAR_ERR_CUDA;
    const int zero = 0;
    cudaMemcpyToSymbol(clear::g_clear_device_error, &zero, sizeof(int));
    return CLEAR_ERR_DEVICE_TIMEOUT;
  }
  return CLEAR_OK;
}

void clear_attn_device_diag(int* out8) {
  if (!out8) return;
  for (int i = 0; i < 8; ++i) out8[i] = t_last_diag[i];
}

clear_status_t clear_attn_selftest_expiry(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 5000) return CLEAR_ERR_INVALID_ARG;
  int num_sms = 0;
  const clear_status_t st = check_device(&num_sms);
  if (st != CLEAR_OK) return st;
  clear_selftest_expiry_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_ms * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? CLEAR_OK : CLEAR_ERR_CUDA;
}

clear_status_t clear_sched_forward_shape(const clear_attn_params_t* params, long long* n_text_items,
                                         long long* n_image_items, int* splits,
                                         int* chunks_per_split) {
  return clear_sched_stripe_forward_shape(params, nullptr, n_text_items, n_image_items, splits, chunks_per_split);
}

clear_status_t clear_sched_stripe_forward_shape(const clear_attn_params_t* params, const clear_attn_stripe_t* stripe,
                                                long long* n_text_items, long long* n_image_items, int* splits,
                                                int* chunks_per_split) {
  const Checked c = stripe ? check_stripe(params, stripe) : check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (n_text_items) *n_text_items = c.g.n_txt_pairs;
  if (n_image_items) *n_image_items = c.g.n_img_pairs;
  if (splits) *splits = c.g.fS;
  if (chunks_per_split) *chunks_per_split = c.g.fcps;
  return CLEAR_OK;
}

clear_status_t clear_sched_item_tiles(const clear_attn_params_t* params, long long item, int* q_info,
                                      int* tiles, int max_tiles, int* n_tiles) {
  return clear_sched_stripe_item_tiles(params, nullptr, item, q_info, tiles, max_tiles, n_tiles);
}

clear_status_t clear_sched_stripe_item_tiles(const clear_attn_params_t* params, const clear_attn_stripe_t* stripe,
                                             long long item, int* q_info, int* tiles, int max_tiles, int* n_tiles) {
  const Checked c = stripe ? check_stripe(params, stripe) : check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  if (item < 0 || item >= c.g.n_txt_pairs + c.g.n_img_pairs || max_tiles < 0) return CLEAR_ERR_INVALID_ARG;
  const PairItem it = decode_pair(c.g, item);
  if (q_info) {
    q_info[0] = it.is_text;
    q_info[1] = it.bh;
    q_info[2] = it.q0;
    q_info[3] = it.x0;
    q_info[4] = it.validB;
  }
  PairKeyIter ki;
  ki.init(c.g, it);
  KeyTile t;
  int n = 0;
  while (ki.next(&t)) {
    if (tiles && n < max_tiles) {
      tiles[4 * n + 0] = t.kind;
      tiles[4 * n + 1] = t.a;
      tiles[4 * n + 2] = t.b;
      tiles[4 * n + 3] = t.flags;
    }
    ++n;
  }
  if (n_tiles) *n_tiles = n;
  return CLEAR_OK;
}

clear_status_t clear_sched_pair_counts(const clear_attn_params_t* params, long long* useful_pairs,
                                       long long* executed_pairs) {
  const Checked c = check_params(params);
  if (c.st != CLEAR_OK) return c.st;
  const Geom& g = c.g;
  // Kept pairs: text rows see all T keys, image rows see all text keys plus their window (clipped,
  // or for the shifted window exactly (2r-1)^2 keys).
  long long win = 0;
  if (g.window == kShifted) win = (long long)g.H * g.W * (2 * g.r - 1) * (2 * g.r - 1);
  for (int dy = -(g.r - 1); dy <= g.r - 1 && g.window != kShifted; ++dy) {
    const int w = half_width(g.r, dy < 0 ? -dy : dy, g.window);
    if (w < 0) continue;
    const long long rows = g.H - (dy < 0 ? -dy : dy);
    if (rows <= 0) continue;
    for (int dx = -w; dx <= w; ++dx) {
      const long long cols = g.W - (dx < 0 ? -dx : dx);
      if (cols > 0) win += rows * cols;
    }
  }
  const long long N = (long long)g.H * g.W;
  const long long per_head = (long long)g.n_text * g.T + N * g.n_text + win;
  if (useful_pairs) *useful_pairs = per_head * g.BH;
  if (executed_pairs) {
    // Tile products actually issued by the forward: each half of a pair multiplies the union key
    // tiles it needs (image blocks of one (b, h), then the text tile pairs over all splits).
    long long tiles = 0;
    for (int blk = 0; blk < g.nQ2; ++blk) {
      const PairItem it = decode_pair(g, g.n_txt_pairs + blk);
      int nu, na, nb;
      count_pair_tiles(g, it, nullptr, 0, &nu, &na, &nb);
      tiles += na + nb;
    }
    for (long long w = 0; w < (long long)g.nTq2 * g.fS; ++w) {
      const PairItem it = decode_pair(g, w);
      int nu, na, nb;
      count_pair_tiles(g, it, nullptr, 0, &nu, &na, &nb);
      tiles += na + nb;
    }
    *executed_pairs = tiles * (long long)kTile * kFChunk * g.BH;
  }
  return CLEAR_OK;
}

}  // extern "C"
