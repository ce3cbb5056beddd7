// Shared device helpers of the sm_100a gated block-sparse attention library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sas.h"

namespace sas {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 8 consecutive elements (16-byte aligned for bf16, 32-byte for fp32) as floats.
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* out);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* out) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* out) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

// Sequence holding packed token tg: largest b with cu[b] <= tg.
__device__ __forceinline__ int seq_of(const int32_t* __restrict__ cu, int batch, int tg) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= tg) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Monotone map fp32 -> uint32 (larger float, larger key; -0 < +0 is harmless here).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace sas

// ---- host side ------------------------------------------------------------------------------
namespace sas {
void set_error(const char* fmt, ...);
sas_status launch_status(const char* what, int launches);
void count_launches(int n);
// Return the status of `expr` from the calling function unless it is SAS_OK.
#define SAS_TRY(expr)              \
  do {                             \
    sas_status s_ = (expr);        \
    if (s_ != SAS_OK) return s_;   \
  } while (0)

}  // namespace sas

#define SAS_CHECK_ARG(cond, ...)                      \
  do {                                                \
    if (!(cond)) {                                    \
      sas::set_error(__VA_ARGS__);                    \
      return SAS_ERR_INVALID_ARG;                     \
    }                                                 \
  } while (0)
