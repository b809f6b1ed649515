// Device helpers shared by the MoBA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moba.h"

#define MOBA_DEV __device__ __forceinline__

namespace moba {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- problem description passed by value to kernels -----------------------
struct Dims {
  int batch, N, hq, hkv, d, B, topk, n, G;
  int chunk;        // tokens per attention pass
  int nchunks;
  int t_lo, t_hi;   // token window [t_lo, t_hi) of the gate kernels (t_lo a multiple of 128)
  float scale_log2; // softmax scale * log2(e)
};

// ---- conversions -------------------------------------------------------------
MOBA_DEV float to_f32(float x) { return x; }
MOBA_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> MOBA_DEV T from_f32(float x);
template <> MOBA_DEV float from_f32<float>(float x) { return x; }
template <> MOBA_DEV __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

MOBA_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

// 16-byte vector of inputs widened to fp32
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int kN = 8;
  static MOBA_DEV void load(const __nv_bfloat16* p, float* out) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
};
template <> struct Vec16<float> {
  static constexpr int kN = 4;
  static MOBA_DEV void load(const float* p, float* out) {
    float4 u = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = u.x; out[1] = u.y; out[2] = u.z; out[3] = u.w;
  }
};

// ---- warp reductions ---------------------------------------------------------
MOBA_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
MOBA_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- async copies ------------------------------------------------------------
MOBA_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
MOBA_DEV void cp_async16(uint32_t dst, const void* src, bool pred) {
  // zero-fills the 16 bytes when pred is false (src-size 0)
  int sz = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
MOBA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> MOBA_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// slot of block j in a sorted selection list (entries < j that are valid)
MOBA_DEV int slot_of(const int32_t* sel_row, int topk, int j) {
  int s = 0;
  for (int i = 0; i < topk; ++i) {
    int e = sel_row[i];
    s += (e >= 0 && e < j) ? 1 : 0;
  }
  return s;
}

}  // namespace moba
