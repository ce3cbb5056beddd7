// The decode gate's per-row selection (A7), shared by the three-launch decode and the fused
// persistent decode: given the row's scores s[0..c] in shared memory (s[c] the current block),
// the logsumexp over j <= c, the exact Top-K of the historical blocks j < c (ties to the lower
// block index, ids ascending) and the current block in the last slot, with log-gates s - lse.
// Model card "tencent/Simple-Attention-Sparsification": Top-K historical blocks plus the current
// block; paper abstract: the current block is always retained.
#pragma once

#include <math.h>

#include "sas_common.cuh"

namespace sas {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < kDecWarps; ++w) r += red[w];
  return r;
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int w = 0; w < kDecWarps; ++w) r = fmaxf(r, red[w]);
  return r;
}

// Shared-memory scratch of decode_select_row: red [kDecWarps] floats, cnt_red [2 kDecWarps],
// misc [4] and hist [256] ints.
struct DecSelScratch {
  float* red;
  int* cnt_red;
  int* misc;
  int* hist;
};

// All kDecThreads threads of the block call this with the same arguments. Row `orow` of the
// selection receives K + 1 slots: the Top-K historical blocks ascending (all of 0..c when
// c <= K, then -1 padding with log-gate 0), the current block c in slot K. sel_logg holds the
// attention's bias (0 when `ungated`), logg_out (optional) the log-gates themselves.
// NPT * kDecThreads >= c.
template <int NPT>
__device__ void decode_select_row(const float* s, int c, int K, int ungated, size_t orow,
                                  int32_t* sel_idx, float* sel_logg, int32_t* idx_out,
                                  float* logg_out, const DecSelScratch& w) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float mx = -INFINITY;
  for (int j = tid; j <= c; j += kDecThreads) mx = fmaxf(mx, s[j]);
  mx = block_reduce_max(mx, w.red);
  float se = 0.f;
  for (int j = tid; j <= c; j += kDecThreads) se += expf(s[j] - mx);
  se = block_reduce_sum(se, w.red);
  const float lse = mx + logf(se);
  if (c <= K) {
    for (int sl = tid; sl <= K; sl += kDecThreads) {
      const int jj = sl <= c ? sl : -1;
      const float lg = sl <= c ? s[sl] - lse : 0.f;
      sel_idx[orow + sl] = jj;
      sel_logg[orow + sl] = ungated ? 0.f : lg;   // the attention's bias
      if (idx_out) idx_out[orow + sl] = jj;
      if (logg_out) logg_out[orow + sl] = lg;
    }
    return;
  }
  // exact K-th largest of s[0..c-1] over order-preserving keys, by a radix select: up to four
  // rounds of an 8-bit digit histogram; `need` is the wanted rank among the keys that share the
  // digits chosen so far (padding keys are 0, below every real key, and c > K); once at most 32
  // keys share them, warp 0 ranks those directly
  uint32_t key[NPT];
#pragma unroll
  for (int r = 0; r < NPT; ++r) {
    const int j = tid + r * kDecThreads;
    key[r] = (j < c) ? order_key(s[j]) : 0u;
  }
  uint32_t thr = 0, pmask = 0;
  int need = K;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kDecThreads) w.hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < NPT; ++r) {   // one shared atomic per distinct digit in the warp
      const bool in = (key[r] & pmask) == thr;
      const int bin = in ? (int)((key[r] >> shift) & 255u) : 256;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&w.hist[bin], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {   // lane owns digits 8 lane .. 8 lane + 7; find the digit where the
                       // count of keys with a larger-or-equal digit first reaches `need`
      int hv[8], loc = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        hv[k] = w.hist[8 * lane + k];
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
      const int nrest = __shfl_sync(0xffffffffu, rest, src);
      const int ncand = __shfl_sync(0xffffffffu, fcnt, src);
      if (lane == 0) {
        w.misc[0] = ncand;   // keys sharing the new prefix
        w.misc[1] = dsel;
        w.misc[2] = nrest;
        w.misc[3] = 0;       // gather cursor of the direct finish
      }
    }
    __syncthreads();
    thr |= (uint32_t)w.misc[1] << shift;
    pmask |= 255u << shift;
    need = w.misc[2];
    const int ncand = w.misc[0];
    if (shift > 0 && ncand <= 32) {
      // few candidates left: gather them and let warp 0 rank them against each other (the
      // need-th largest), instead of more histogram rounds
      uint32_t* cand = reinterpret_cast<uint32_t*>(w.hist);
#pragma unroll
      for (int r = 0; r < NPT; ++r)
        if ((key[r] & pmask) == thr) cand[atomicAdd(&w.misc[3], 1)] = key[r];
      __syncthreads();
      if (warp == 0) {
        const uint32_t x = lane < ncand ? cand[lane] : 0u;
        int gt = 0, eq = 0;
        for (int i = 0; i < ncand; ++i) {
          const uint32_t y = cand[i];
          gt += y > x ? 1 : 0;
          eq += y == x ? 1 : 0;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, lane < ncand && gt < need && need <= gt + eq);
        const int hs = hit ? __ffs(hit) - 1 : 0;
        const uint32_t xs = __shfl_sync(0xffffffffu, x, hs);
        const int gs = __shfl_sync(0xffffffffu, gt, hs);
        if (lane == 0) {
          w.misc[1] = (int)xs;
          w.misc[2] = need - gs;
        }
      }
      __syncthreads();
      thr = (uint32_t)w.misc[1];
      need = w.misc[2];
      break;
    }
  }
  const int need_eq = need;   // keys equal to thr to take, lowest block indices first
  // ordered emission: warp w takes a contiguous range of blocks; a first pass counts its keys
  // above and equal to thr, a second writes its selected blocks at their global positions
  const int per = (c + kDecWarps - 1) / kDecWarps;
  const int wj0 = min(c, warp * per), wj1 = min(c, wj0 + per);
  const unsigned below = (1u << lane) - 1u;
  int n_gt = 0, n_eq = 0;
  for (int j0 = wj0; j0 < wj1; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t kk = j < wj1 ? order_key(s[j]) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, j < wj1 && kk > thr));
    n_eq += __popc(__ballot_sync(0xffffffffu, j < wj1 && kk == thr));
  }
  if (lane == 0) {
    w.cnt_red[warp] = n_gt;
    w.cnt_red[kDecWarps + warp] = n_eq;
  }
  __syncthreads();
  int gt_before = 0, eq_seen = 0;
  for (int v = 0; v < warp; ++v) {
    gt_before += w.cnt_red[v];
    eq_seen += w.cnt_red[kDecWarps + v];
  }
  int out = gt_before + min(eq_seen, need_eq);
  for (int j0 = wj0; j0 < wj1; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < wj1;
    const uint32_t kk = valid ? order_key(s[j]) : 0u;
    const bool is_gt = valid && kk > thr, is_eq = valid && kk == thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eqm & below);
    const bool sel = is_gt || (is_eq && eq_rank < need_eq);
    const unsigned selm = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int pos = out + __popc(selm & below);
      const float lg = s[j] - lse;
      sel_idx[orow + pos] = j;
      sel_logg[orow + pos] = ungated ? 0.f : lg;
      if (idx_out) idx_out[orow + pos] = j;
      if (logg_out) logg_out[orow + pos] = lg;
    }
    out += __popc(selm);
    eq_seen += __popc(eqm);
  }
  if (tid == 0) {
    const float lg = s[c] - lse;
    sel_idx[orow + K] = c;
    sel_logg[orow + K] = ungated ? 0.f : lg;
    if (idx_out) idx_out[orow + K] = c;
    if (logg_out) logg_out[orow + K] = lg;
  }
}

// The row of a sequence with nothing to select (invalid length, a bad page id): every slot
// -1 with log-gate 0.
__device__ __forceinline__ void decode_select_empty(int K, size_t orow, int32_t* sel_idx,
                                                    float* sel_logg, int32_t* idx_out,
                                                    float* logg_out) {
  for (int sl = threadIdx.x; sl <= K; sl += blockDim.x) {
    sel_idx[orow + sl] = -1;
    sel_logg[orow + sl] = 0.f;
    if (idx_out) idx_out[orow + sl] = -1;
    if (logg_out) logg_out[orow + sl] = 0.f;
  }
}

}  // namespace sas
