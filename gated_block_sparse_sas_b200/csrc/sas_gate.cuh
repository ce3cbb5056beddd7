// Device helpers shared by the gate kernels (sas_gate.cu, sas_gate_select.cu): the gate's
// RMSNorm + rotary epilogue of a projected row, and the exact per-row Top-K of one warp.
// Model card "tencent/Simple-Attention-Sparsification", table "Checkpoint configuration":
// Q/K normalisation, gate RoPE, Training Top-K.
#pragma once

#include "sas_common.cuh"

namespace sas {

// ---------------------------------------------------------------------------------------
// Shared epilogue: RMSNorm over h (x / sqrt(mean x^2 + eps) * w), then rotate-half rotary
// at position pos using the fp32 tables (built in double on the host). One warp per row.
// ---------------------------------------------------------------------------------------
template <int H>
__device__ __forceinline__ void norm_rope_row(const float* x, const float* __restrict__ w, float eps,
                                              const float* __restrict__ rc, const float* __restrict__ rs,
                                              int pos, float* dst, int lane) {
  float ss = 0.f;
  for (int e = lane; e < H; e += 32) ss += x[e] * x[e];
  ss = warp_sum(ss);
  const float rn = sqrtf(ss / (float)H + eps);
  const float* c = rc + (size_t)pos * (H / 2);
  const float* s = rs + (size_t)pos * (H / 2);
  for (int e = lane; e < H / 2; e += 32) {
    const float a = x[e] / rn * w[e];
    const float b = x[e + H / 2] / rn * w[e + H / 2];
    dst[e] = a * c[e] - b * s[e];
    dst[e + H / 2] = b * c[e] + a * s[e];
  }
}

// Nearest tf32 value of a finite x (rounded, low 13 mantissa bits cleared): the hi part of the
// split x = hi + lo used by the tensor-core historical scores.
__device__ __forceinline__ float tf32_hi(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// One row with c > K historical candidates held as NPL keys per lane (c <= 32 NPL).
template <int NPL>
__device__ __forceinline__ void topk_row(const float* __restrict__ srow, float l, int c, int K,
                                         int lane, int32_t* __restrict__ irow,
                                         float* __restrict__ grow) {
  uint32_t key[NPL];
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int j = r * 32 + lane;
    key[r] = (j < c) ? order_key(srow[j]) : 0u;
  }
  uint32_t thr = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = thr | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int r = 0; r < NPL; ++r) cnt += (key[r] >= cand) ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= K) thr = cand;
  }
  int gt = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) gt += (key[r] > thr) ? 1 : 0;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need_eq = K - gt;
  const unsigned below = (1u << lane) - 1u;
  int out = 0, eq_seen = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const bool is_gt = key[r] > thr, is_eq = key[r] == thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eqm & below);
    const bool sel = is_gt || (is_eq && eq_rank < need_eq);
    const unsigned selm = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int pos = out + __popc(selm & below);
      const int j = r * 32 + lane;
      irow[pos] = j;
      grow[pos] = srow[j] - l;
    }
    out += __popc(selm);
    eq_seen += __popc(eqm);
  }
}

}  // namespace sas
