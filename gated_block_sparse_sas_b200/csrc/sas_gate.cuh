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

// Inverse of order_key: the float whose key is k (bit for bit).
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The same row selection as topk_row (exact K-th largest key, ties to the lower block index,
// ascending emission), with the threshold found by a radix select: four rounds over the 8-bit
// digits of the order-preserving keys, each a histogram in the warp's own 256 shared counters
// (`hist`) over the keys that share the digits chosen so far. Padding keys are 0, below every
// real key, and c > K, so the K-th largest is a real key. Once at most 32 keys share the digits
// chosen so far (usually after two rounds), they are ranked directly in the warp.
template <int NPL>
__device__ __forceinline__ void topk_row_radix(const float* __restrict__ srow, float l, int c, int K,
                                               int lane, int* hist, int32_t* __restrict__ irow,
                                               float* __restrict__ grow) {
  uint32_t key[NPL];
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int j = r * 32 + lane;
    key[r] = (j < c) ? order_key(srow[j]) : 0u;
  }
  uint32_t thr = 0, pmask = 0;
  int need = K;   // rank wanted among the keys that share the digits chosen so far
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) hist[i * 32 + lane] = 0;
    __syncwarp();
#pragma unroll
    for (int r = 0; r < NPL; ++r)
      if ((key[r] & pmask) == thr) atomicAdd(&hist[(key[r] >> shift) & 255u], 1);
    __syncwarp();
    // lane owns digits 8 lane .. 8 lane + 7: the digit where the count of keys with a larger or
    // equal digit first reaches `need`
    int hv[8], loc = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      hv[k] = hist[8 * lane + k];
      loc += hv[k];
    }
    int incl = loc;   // keys in this lane's digits and all larger ones
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += v;
    }
    int acc = incl - loc, found = -1, rest = 0, fcnt = 0;
#pragma unroll
    for (int k = 7; k >= 0; --k) {
      if (found < 0 && acc < need && acc + hv[k] >= need) {
        found = 8 * lane + k;
        rest = need - acc;
        fcnt = hv[k];
      }
      acc += hv[k];
    }
    const unsigned who = __ballot_sync(0xffffffffu, found >= 0);   // exactly one lane
    const int src = who ? __ffs(who) - 1 : 0;
    const int dsel = __shfl_sync(0xffffffffu, found, src);
    need = __shfl_sync(0xffffffffu, rest, src);
    const int ncand = __shfl_sync(0xffffffffu, fcnt, src);   // keys sharing the new prefix
    thr |= (uint32_t)dsel << shift;
    pmask |= 255u << shift;
    __syncwarp();   // every lane has read the counters before they are reused
    if (shift > 0 && ncand <= 32) {
      // few candidates left: gather them (one per lane) and take the need-th largest by
      // ranking them against each other, instead of more histogram rounds
      uint32_t* cand = reinterpret_cast<uint32_t*>(hist);
      int at = 0;
#pragma unroll
      for (int r = 0; r < NPL; ++r) {
        const bool m = (key[r] & pmask) == thr;
        const unsigned bal = __ballot_sync(0xffffffffu, m);
        if (m) cand[at + __popc(bal & ((1u << lane) - 1u))] = key[r];
        at += __popc(bal);
      }
      __syncwarp();
      const uint32_t x = lane < ncand ? cand[lane] : 0u;
      int gt = 0, eq = 0;
      for (int i = 0; i < ncand; ++i) {
        const uint32_t y = cand[i];
        gt += y > x ? 1 : 0;
        eq += y == x ? 1 : 0;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, lane < ncand && gt < need && need <= gt + eq);
      const int hs = hit ? __ffs(hit) - 1 : 0;
      thr = __shfl_sync(0xffffffffu, x, hs);
      need -= __shfl_sync(0xffffffffu, gt, hs);
      __syncwarp();
      break;
    }
  }
  const int need_eq = need;   // keys equal to thr to take, lowest block indices first
  const unsigned below = (1u << lane) - 1u;
  int out = 0, eq_seen = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const bool is_gt = key[r] > thr, is_eq = key[r] == thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eqm & below);
    const bool sel = is_gt || (is_eq && eq_rank < need_eq);
    const unsigned selm = __ballot_sync(0xffffffffu, sel);
    if (sel) {   // the score comes back from its key, exactly (no reload)
      const int pos = out + __popc(selm & below);
      irow[pos] = r * 32 + lane;
      grow[pos] = key_float(key[r]) - l;
    }
    out += __popc(selm);
    eq_seen += __popc(eqm);
  }
}

}  // namespace sas
