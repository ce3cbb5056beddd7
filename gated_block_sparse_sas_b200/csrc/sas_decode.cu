// Sparse decode step (A7). Model card "tencent/Simple-Attention-Sparsification": the
// released setup decodes with a 2,048-token budget (1,024 / 4,096 also usable), i.e.
// Top-K historical blocks plus the current block; Chinese guide, caveat 3: the budget
// caps the tokens each query attends to, not the KV cache.
//
// Three launches: (1) gate + Top-K per (sequence, kv head) -> selection in workspace;
// (2) split-K gated attention over the selected blocks -> per-split (m, l, acc);
// (3) merge of the splits -> O. The attention only ever reads the selected blocks.
#include <math.h>

#include <type_traits>

#include "sas_common.cuh"
#include "sas_decode_select.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {

// ---------------------------------------------------------------------------------------
// (1) gate: q~ (Qproj over the G concatenated pre-rotary heads, RMSNorm, rotary at L-1),
// current-block key from the running pool state (max, min, sum/n; Kproj, RMSNorm, rotary
// at c*B), scores against the cached block keys, logsumexp over j <= c, Top-K over j < c.
// ---------------------------------------------------------------------------------------
template <typename T, int H, int NPT>
__global__ void __launch_bounds__(kDecThreads) decode_gate_kernel(
    const T* __restrict__ q_nope, const __nv_bfloat16* __restrict__ gkc,
    const float* __restrict__ cur_pool, const T* __restrict__ wq, const float* __restrict__ qnorm_w,
    const T* __restrict__ wk, const float* __restrict__ knorm_w, const int32_t* __restrict__ seqlens,
    const float* __restrict__ rc, const float* __restrict__ rs, int Hq, int Hkv, int Hs, int d, int B, int K,
    int NBmax, int capacity, float eps, int ungated, int32_t* __restrict__ sel_idx,
    float* __restrict__ sel_logg, int32_t* __restrict__ idx_out, float* __restrict__ logg_out,
    const int32_t* __restrict__ pt, int num_pages, int* __restrict__ err) {
  extern __shared__ float smem[];
  const int G = Hq / Hs, GD = G * d, C = 3 * d;   // G: query heads of the gate head
  float* qcat = smem;                  // [GD]
  float* P = qcat + GD;                // [C]
  float* xq = P + C;                   // [H]
  float* xk = xq + H;                  // [H]
  float* s = xk + H;                   // [NBmax + 1]
  float* red = s + NBmax + 1;          // [kDecWarps]
  int* cnt_red = reinterpret_cast<int*>(red + kDecWarps);  // [2][kDecWarps]
  int* misc = cnt_red + 2 * kDecWarps;                      // [4]
  int* hist = misc + 4;                                     // [256] radix histogram
  int* pages = hist + 256;                                  // [NBmax] paged caches: page of block j

  // gate head sh (a KV head, or a query head with one gate per query head); its block keys,
  // pool state and Kproj are KV head kv's
  const int sh = blockIdx.x, b = blockIdx.y;
  const int kv = sh / (Hs / Hkv);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = seqlens[b];
  const int t = L - 1, c = t / B, n = L - c * B;
  const size_t orow = ((size_t)b * Hs + sh) * (K + 1);
  bool empty = L < 1 || L > capacity;   // invalid length: empty selection, the merge writes 0
  if (!empty && pt != nullptr) {   // paged caches: the pages of blocks 0..c, range-checked
    int bad = 0;
    for (int j = tid; j <= c; j += kDecThreads) {
      const int pg = pt[(size_t)b * NBmax + j];
      bad |= (pg < 0 || pg >= num_pages) ? 1 : 0;
      pages[j] = pg;
    }
    if (__syncthreads_or(bad)) {   // a page id out of range: report it, read nothing
      if (tid == 0) atomicCAS(err, 0, 62);
      empty = true;
    }
  }
  if (empty) {
    decode_select_empty(K, orow, sel_idx, sel_logg, idx_out, logg_out);
    return;
  }

  if (tid == 0 && c > 0 && pt == nullptr) {   // start streaming this row's cached block keys into L2 now: the
    // projections below take a while and the scores read these rows only afterwards
    const char* src = reinterpret_cast<const char*>(gkc + ((size_t)b * Hkv + kv) * (size_t)NBmax * H);
    const size_t bytes = (size_t)c * H * 2;   // a multiple of 16 (H >= 32)
    for (size_t o = 0; o < bytes; o += 65536) {
      const uint32_t n = (uint32_t)min((size_t)65536, bytes - o);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src + o), "r"(n) : "memory");
    }
  }
  for (int e = tid; e < GD; e += kDecThreads)
    qcat[e] = to_f(q_nope[((size_t)b * Hq + (size_t)sh * G) * d + e]);
  for (int e = tid; e < C; e += kDecThreads) {
    const int part = e / d, ch = e - part * d;
    const float x = cur_pool[(((size_t)b * Hkv + kv) * 3 + part) * d + ch];
    P[e] = (part == 2) ? x / (float)n : x;
  }
  __syncthreads();
  // projections: warp-coalesced weight rows (lanes across the input, 16-byte loads), eight
  // output channels per warp step with all their loads issued before any arithmetic
  if constexpr (!std::is_same<T, __nv_bfloat16>::value) {   // fp32 weights: one row per step
    for (int job = warp; job < 2 * H; job += kDecWarps) {
      const bool isq = job < H;
      const int i = isq ? job : job - H;
      const T* w = isq ? wq + ((size_t)sh * H + i) * GD : wk + ((size_t)kv * H + i) * C;
      const float* x = isq ? qcat : P;
      const int n_in = isq ? GD : C;
      float acc = 0.f;
      for (int e0 = lane * 8; e0 < n_in; e0 += 256) {
        float w8[8];
        load8<T>(w + e0, w8);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = fmaf(w8[u], x[e0 + u], acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) (isq ? xq : xk)[i] = acc;
    }
  } else {
    constexpr int R = 8;
    for (int job0 = warp * R; job0 < 2 * H; job0 += kDecWarps * R) {
      const bool isq = job0 < H;   // H is a multiple of 8: a step never mixes q and k rows
      const int i0 = isq ? job0 : job0 - H;
      const T* w = isq ? wq + ((size_t)sh * H + i0) * GD : wk + ((size_t)kv * H + i0) * C;
      const int n_in = isq ? GD : C;
      const float* x = isq ? qcat : P;
      const int nv = n_in / 8;   // 16-byte vectors per row
      float acc[R];
#pragma unroll
      for (int u = 0; u < R; ++u) acc[u] = 0.f;
      for (int v0 = 0; v0 < nv; v0 += 64) {   // two vectors per lane per row in flight
        uint4 raw[R][2];
#pragma unroll
        for (int u = 0; u < R; ++u)
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int v = v0 + h2 * 32 + lane;
            raw[u][h2] = v < nv ? __ldg(reinterpret_cast<const uint4*>(w + (size_t)u * n_in) + v)
                                : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int v = v0 + h2 * 32 + lane;
          if (v < nv) {
            const float4 xa = *reinterpret_cast<const float4*>(x + v * 8);
            const float4 xb = *reinterpret_cast<const float4*>(x + v * 8 + 4);
#pragma unroll
            for (int u = 0; u < R; ++u) {
              float f[8];
              const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&raw[u][h2]);
#pragma unroll
              for (int q2 = 0; q2 < 4; ++q2) {
                const float2 ff = __bfloat1622float2(hh[q2]);
                f[2 * q2] = ff.x;
                f[2 * q2 + 1] = ff.y;
              }
              acc[u] = fmaf(f[0], xa.x, acc[u]); acc[u] = fmaf(f[1], xa.y, acc[u]);
              acc[u] = fmaf(f[2], xa.z, acc[u]); acc[u] = fmaf(f[3], xa.w, acc[u]);
              acc[u] = fmaf(f[4], xb.x, acc[u]); acc[u] = fmaf(f[5], xb.y, acc[u]);
              acc[u] = fmaf(f[6], xb.z, acc[u]); acc[u] = fmaf(f[7], xb.w, acc[u]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const float r = warp_sum(acc[u]);
        if (lane == 0) (isq ? xq : xk)[i0 + u] = r;
      }
    }
  }
  __syncthreads();
  if (warp == 0 || warp == 1) {
    float* x = warp == 0 ? xq : xk;
    const float* w = warp == 0 ? qnorm_w : knorm_w;
    const int pos = warp == 0 ? t : c * B;
    float ss = 0.f;
    for (int e = lane; e < H; e += 32) ss += x[e] * x[e];
    ss = warp_sum(ss);
    const float rn = sqrtf(ss / (float)H + eps);
    float lo[H / 64 > 0 ? H / 64 : 1], hi[H / 64 > 0 ? H / 64 : 1];
    int u = 0;
    for (int e = lane; e < H / 2; e += 32, ++u) {
      const float a = x[e] / rn * w[e], bb = x[e + H / 2] / rn * w[e + H / 2];
      const float cs = rc[(size_t)pos * (H / 2) + e], sn = rs[(size_t)pos * (H / 2) + e];
      lo[u] = a * cs - bb * sn;
      hi[u] = bb * cs + a * sn;
    }
    __syncwarp();
    u = 0;
    for (int e = lane; e < H / 2; e += 32, ++u) { x[e] = lo[u]; x[e + H / 2] = hi[u]; }
  }
  __syncthreads();
  const float sqrt_h = sqrtf((float)H);
  // historical scores: H/8 lanes per cached key row (16 bytes each, so a row is one
  // coalesced segment), 32*8/H rows per warp instruction, 8 rows in flight per lane group
  {
    constexpr int LPR = H / 8, RPW = 32 / LPR, UNR = 8;
    const int sub = lane % LPR, rsub = lane / LPR;
    float qv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) qv[u] = xq[sub * 8 + u];
    const __nv_bfloat16* base = gkc + ((size_t)b * Hkv + kv) * (size_t)NBmax * H + sub * 8;
    for (int j0 = warp * RPW * UNR; j0 < c; j0 += kDecWarps * RPW * UNR) {   // warp-uniform
      uint4 raw[UNR];
#pragma unroll
      for (int it = 0; it < UNR; ++it) {
        const int j = j0 + it * RPW + rsub;
        const __nv_bfloat16* row =
            pt != nullptr ? gkc + ((size_t)pages[j < c ? j : 0] * Hkv + kv) * H + sub * 8
                          : base + (size_t)j * H;
        raw[it] = (j < c) ? __ldg(reinterpret_cast<const uint4*>(row)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int it = 0; it < UNR; ++it) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[it]);
        float acc = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) {
          const float2 f = __bfloat1622float2(h2[w2]);
          acc = fmaf(qv[2 * w2], f.x, acc);
          acc = fmaf(qv[2 * w2 + 1], f.y, acc);
        }
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const int j = j0 + it * RPW + rsub;
        if (sub == 0 && j < c) s[j] = acc / sqrt_h;
      }
    }
    if (warp == 0) {
      float dot = 0.f;
      for (int e = lane; e < H; e += 32) dot += xq[e] * xk[e];
      dot = warp_sum(dot);
      if (lane == 0) s[c] = dot / sqrt_h;
    }
  }
  __syncthreads();
  decode_select_row<NPT>(s, c, K, ungated, orow, sel_idx, sel_logg, idx_out, logg_out,
                         DecSelScratch{red, cnt_red, misc, hist});
}

// ---------------------------------------------------------------------------------------
// (2) split-K attention over the selected blocks. CTA = (kv, sequence, split); each warp
// streams every 8th key of the CTA's blocks (one 2*d-byte row of K and of V per key, lane
// slices of d/32 channels) and keeps an online softmax for the G heads.
// ---------------------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
    const int32_t* __restrict__ seqlens, const int32_t* __restrict__ sel_idx,
    const float* __restrict__ sel_logg, int Hkv, int R, int capacity, int B, int K, int nsplit,
    float scale_log2, float* __restrict__ part_ml, float* __restrict__ part_acc) {
  // Hkv counts gate heads here; gate head kv reads the keys/values of KV head kv / R
  constexpr int E = D / 32;
  __shared__ float sm_m[kDecWarps][G], sm_l[kDecWarps][G];
  __shared__ float sm_acc[kDecWarps][G][D];
  const int kv = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = min(seqlens[b], capacity);
  const int Hq = Hkv * G;
  const int slots = K + 1;
  const int per = (slots + nsplit - 1) / nsplit;
  const int sl0 = split * per, sl1 = min(slots, sl0 + per);
  const size_t srow = ((size_t)b * Hkv + kv) * (K + 1);
  float qr[G][E], acc[G][E], m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qr[g][e] = to_f(q[((size_t)b * Hq + kv * G + g) * D + lane * E + e]);
      acc[g][e] = 0.f;
    }
    m[g] = -INFINITY;
    l[g] = 0.f;
  }
  const T* kbase = kc + ((size_t)b * (Hkv / R) + kv / R) * (size_t)capacity * D + lane * E;
  const T* vbase = vc + ((size_t)b * (Hkv / R) + kv / R) * (size_t)capacity * D + lane * E;
  for (int sl = sl0; sl < sl1; ++sl) {
    const int j = sel_idx[srow + sl];
    if (j < 0) continue;
    const float bias = sel_logg[srow + sl] * kLog2e;
    const int i0 = j * B, i1 = min(i0 + B, L);
    for (int i = i0 + warp; i < i1; i += kDecWarps) {
      float kk[E], vv[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        kk[e] = to_f(kbase[(size_t)i * D + e]);
        vv[e] = to_f(vbase[(size_t)i * D + e]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float p = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) p = fmaf(qr[g][e], kk[e], p);
        p = warp_sum(p) * scale_log2 + bias;
        const float mn = fmaxf(m[g], p);
        const float a = exp2f(m[g] - mn), pe = exp2f(p - mn);
        l[g] = l[g] * a + pe;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] = fmaf(acc[g][e], a, pe * vv[e]);
        m[g] = mn;
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (lane == 0) { sm_m[warp][g] = m[g]; sm_l[warp][g] = l[g]; }
#pragma unroll
    for (int e = 0; e < E; ++e) sm_acc[warp][g][lane * E + e] = acc[g][e];
  }
  __syncthreads();
  const size_t prow = (((size_t)b * Hkv + kv) * nsplit + split) * G;
  for (int e = threadIdx.x; e < G * D; e += kDecThreads) {
    const int g = e / D, ch = e - g * D;
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_m[w][g]);
    float ls = 0.f, as = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float f = exp2f(sm_m[w][g] - M);
        ls += sm_l[w][g] * f;
        as += sm_acc[w][g][ch] * f;
      }
    }
    part_acc[(prow + g) * D + ch] = as;
    if (ch == 0) {
      part_ml[(prow + g) * 2] = M;
      part_ml[(prow + g) * 2 + 1] = ls;
    }
  }
}

// ---------------------------------------------------------------------------------------
// (2') the same split-K attention for bf16, head_dim 128: each kept block's K and V rows
// (contiguous, up to 16 KB each) are streamed into a 3-stage shared-memory ring by bulk
// asynchronous copies issued by one thread, so many kilobytes per SM are in flight; all 256
// threads then work from shared memory: scores (a warp per key, lanes across head_dim),
// per-head online softmax (a warp per head), P.V (a thread per (head, 2 channels)).
// ---------------------------------------------------------------------------------------
constexpr int kAttStages = 3;
constexpr int kAttRow = 128 * 2;                  // bytes of one bf16 K or V row (d = 128)
constexpr int kAttBlk = 64 * kAttRow;             // one block of K (or V): 16 KB
constexpr int kAttStage = 2 * kAttBlk;

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

template <int G>
__global__ void __launch_bounds__(kDecThreads, 2) decode_attn_bulk_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
    const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ seqlens,
    const int32_t* __restrict__ sel_idx, const float* __restrict__ sel_logg, int Hkv, int R,
    int capacity, int B, int K, int nsplit, float scale_log2, float* __restrict__ part_ml,
    float* __restrict__ part_acc, int* __restrict__ err) {
  // Hkv counts gate heads here; gate head kv reads the keys/values of KV head kv / R
  using namespace sm100;
  constexpr int D = 128;
  constexpr int NP = (G * 64 + kDecThreads - 1) / kDecThreads;   // (head, 2-channel) pairs per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                           ~static_cast<uintptr_t>(127));
  float* q_sm = reinterpret_cast<float*>(sm + kAttStages * kAttStage);   // [G][128]
  float* s_sm = q_sm + G * D;                                            // [G][64]
  float* st_sm = s_sm + G * 64;                                          // [3][8]: m, l, alpha
  int* blk_j = reinterpret_cast<int*>(st_sm + 3 * 8);                    // [128] kept blocks
  float* blk_b = reinterpret_cast<float*>(blk_j + 128);                  // their log-gates (log2)
  uint64_t* full = reinterpret_cast<uint64_t*>(blk_b + 128);             // [kAttStages], 8-aligned
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kAttStages);
  int* nblk_s = reinterpret_cast<int*>(full + kAttStages) + 1;

  const int kv = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = min(seqlens[b], capacity);
  const int Hq = Hkv * G;
  const int slots = K + 1;
  const int per = (slots + nsplit - 1) / nsplit;
  const int sl0 = split * per, sl1 = min(slots, sl0 + per);
  const size_t srow = ((size_t)b * Hkv + kv) * (K + 1);
  if (warp == 0) {   // this split's kept blocks, in slot order (at most 128 slots)
    int n = 0;
    for (int sl0w = sl0; sl0w < sl1; sl0w += 32) {
      const int sl = sl0w + lane;
      int j = -1;
      float lg = 0.f;
      if (sl < sl1) {
        j = sel_idx[srow + sl];
        lg = sel_logg[srow + sl];
      }
      const bool keep = j >= 0 && j * B < L;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int pos = n + __popc(m & ((1u << lane) - 1u));
        blk_j[pos] = j;
        blk_b[pos] = lg * kLog2e;
      }
      n += __popc(m);
    }
    if (lane == 0) {
      *nblk_s = n;
      for (int s = 0; s < kAttStages; ++s) mbar_init(full + s, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
  }
  for (int e = tid; e < G * D; e += kDecThreads)
    q_sm[e] = __bfloat162float(q[((size_t)b * Hq + kv * G) * D + e]);
  if (tid < G) {
    st_sm[tid] = -INFINITY;
    st_sm[8 + tid] = 0.f;
  }
  __syncthreads();
  const int nblk = *nblk_s;
  const __nv_bfloat16* kbase = kc + ((size_t)b * (Hkv / R) + kv / R) * (size_t)capacity * D;
  const __nv_bfloat16* vbase = vc + ((size_t)b * (Hkv / R) + kv / R) * (size_t)capacity * D;
  auto issue = [&](int n) {   // thread 0: copy block n's K and V rows into stage n % kAttStages
    const int st = n % kAttStages;
    const int i0 = blk_j[n] * B;
    const int nk = min(B, L - i0);
    const uint32_t bytes = (uint32_t)nk * kAttRow;
    const uint32_t dst = smem_u32(sm + st * kAttStage);
    mbar_arrive_expect_tx(full + st, 2 * bytes);
    bulk_g2s(dst, kbase + (size_t)i0 * D, bytes, full + st);
    bulk_g2s(dst + kAttBlk, vbase + (size_t)i0 * D, bytes, full + st);
  };
  int issued = 0;   // thread 0 only
  if (tid == 0)
    for (; issued < min(nblk, kAttStages); ++issued) issue(issued);

  float acc[NP][2];
#pragma unroll
  for (int u = 0; u < NP; ++u) acc[u][0] = acc[u][1] = 0.f;
  bool ok = true;
  for (int n = 0; n < nblk; ++n) {
    const int st = n % kAttStages;
    const int i0 = blk_j[n] * B;
    const int nk = min(B, L - i0);
    const float bias = blk_b[n];
    if (ok && !mbar_wait(full + st, (n / kAttStages) & 1, abort_flag)) {
      *abort_flag = 1;
      atomicCAS(err, 0, 41);
      ok = false;
    }
    ok = __all_sync(0xffffffffu, ok);   // warp-uniform for the warp reductions below
    const uint8_t* kst = sm + st * kAttStage;
    const uint8_t* vst = kst + kAttBlk;
    // scores: 8 lanes per key (16 channels each), 4 keys per warp step, 8 keys per warp
    {
      const int sub = lane & 7, kq = lane >> 3;
#pragma unroll 1
      for (int step = 0; step < 2; ++step) {
        const int k = warp * 8 + step * 4 + kq;
        float kf[16];
        const bool live = ok && k < nk;
        if (live) {
          const uint4 a0 = *reinterpret_cast<const uint4*>(kst + k * kAttRow + sub * 32);
          const uint4 a1 = *reinterpret_cast<const uint4*>(kst + k * kAttRow + sub * 32 + 16);
          const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&a0);
          const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&a1);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 f0 = __bfloat1622float2(h0[u]), f1 = __bfloat1622float2(h1[u]);
            kf[2 * u] = f0.x; kf[2 * u + 1] = f0.y; kf[8 + 2 * u] = f1.x; kf[8 + 2 * u + 1] = f1.y;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) kf[u] = 0.f;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float* qh = q_sm + h * D + sub * 16;
          float dot = 0.f;
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            const float4 qq = *reinterpret_cast<const float4*>(qh + u);
            dot = fmaf(qq.x, kf[u], dot);
            dot = fmaf(qq.y, kf[u + 1], dot);
            dot = fmaf(qq.z, kf[u + 2], dot);
            dot = fmaf(qq.w, kf[u + 3], dot);
          }
          dot += __shfl_xor_sync(0xffffffffu, dot, 1);
          dot += __shfl_xor_sync(0xffffffffu, dot, 2);
          dot += __shfl_xor_sync(0xffffffffu, dot, 4);
          if (sub == 0) s_sm[h * 64 + k] = live ? fmaf(dot, scale_log2, bias) : -INFINITY;
        }
      }
    }
    __syncthreads();
    // online softmax per head (warp h)
    if (warp < G) {
      const float s0v = s_sm[warp * 64 + lane], s1v = s_sm[warp * 64 + 32 + lane];
      const float mx = warp_max(fmaxf(s0v, s1v));
      const float m_old = st_sm[warp];
      const float m_new = fmaxf(m_old, mx);
      const float ref = (m_new == -INFINITY) ? 0.f : m_new;
      const float p0 = exp2f(s0v - ref), p1 = exp2f(s1v - ref);
      s_sm[warp * 64 + lane] = p0;
      s_sm[warp * 64 + 32 + lane] = p1;
      const float ps = warp_sum(p0 + p1);
      if (lane == 0) {
        const float alpha = (m_old == -INFINITY) ? 0.f : exp2f(m_old - ref);
        st_sm[warp] = m_new;
        st_sm[8 + warp] = st_sm[8 + warp] * alpha + ps;
        st_sm[16 + warp] = alpha;
      }
    }
    __syncthreads();
    // P.V: thread owns (head, channel pair) o = tid + 256 u
#pragma unroll
    for (int u = 0; u < NP; ++u) {
      const int o = tid + u * kDecThreads;
      if (o < G * 64) {
        const int h = o >> 6, d2 = (o & 63) * 2;
        const float alpha = st_sm[16 + h];
        float a0 = acc[u][0] * alpha, a1 = acc[u][1] * alpha;
        const float* ph = s_sm + h * 64;
        float b0 = 0.f, b1 = 0.f;   // second chain for instruction-level parallelism
        int k = 0;
        for (; k + 8 <= nk; k += 8) {
#pragma unroll
          for (int kk = 0; kk < 8; kk += 2) {
            const float2 v0 = __bfloat1622float2(
                *reinterpret_cast<const __nv_bfloat162*>(vst + (k + kk) * kAttRow + d2 * 2));
            const float2 v1 = __bfloat1622float2(
                *reinterpret_cast<const __nv_bfloat162*>(vst + (k + kk + 1) * kAttRow + d2 * 2));
            a0 = fmaf(ph[k + kk], v0.x, a0);
            a1 = fmaf(ph[k + kk], v0.y, a1);
            b0 = fmaf(ph[k + kk + 1], v1.x, b0);
            b1 = fmaf(ph[k + kk + 1], v1.y, b1);
          }
        }
        for (; k < nk; ++k) {
          const float2 v = __bfloat1622float2(
              *reinterpret_cast<const __nv_bfloat162*>(vst + k * kAttRow + d2 * 2));
          a0 = fmaf(ph[k], v.x, a0);
          a1 = fmaf(ph[k], v.y, a1);
        }
        acc[u][0] = a0 + b0;
        acc[u][1] = a1 + b1;
      }
    }
    __syncthreads();   // stage and score buffer free again
    if (tid == 0 && ok && issued < nblk) issue(issued++);
  }
  // no bulk copy may still be in flight at exit (normal path: every one was consumed)
  if (tid == 0)
    for (int m = max(0, issued - kAttStages); m < issued; ++m)
      mbar_wait_drain(full + m % kAttStages, (m / kAttStages) & 1);
  const size_t prow = (((size_t)b * Hkv + kv) * nsplit + split) * G;
#pragma unroll
  for (int u = 0; u < NP; ++u) {
    const int o = tid + u * kDecThreads;
    if (o < G * 64) {
      const int h = o >> 6, d2 = (o & 63) * 2;
      part_acc[(prow + h) * D + d2] = acc[u][0];
      part_acc[(prow + h) * D + d2 + 1] = acc[u][1];
    }
  }
  if (tid < G) {
    part_ml[(prow + tid) * 2] = st_sm[tid];
    part_ml[(prow + tid) * 2 + 1] = st_sm[8 + tid];
  }
}

// (3) merge the splits (log2-domain maxima) and normalise.
template <typename T, int D, int G>
__global__ void decode_merge_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_acc,
                                    int Hkv, int nsplit, T* __restrict__ o) {
  const int kv = blockIdx.x, b = blockIdx.y;
  const int Hq = Hkv * G;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int g = e / D, ch = e - g * D;
    float M = -INFINITY;
    for (int sp = 0; sp < nsplit; ++sp)
      M = fmaxf(M, part_ml[((((size_t)b * Hkv + kv) * nsplit + sp) * G + g) * 2]);
    float ls = 0.f, as = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) {
      const size_t pr = (((size_t)b * Hkv + kv) * nsplit + sp) * G + g;
      const float mm = part_ml[pr * 2];
      if (mm == -INFINITY) continue;
      const float f = exp2f(mm - M);
      ls += part_ml[pr * 2 + 1] * f;
      as += part_acc[pr * D + ch] * f;
    }
    // a head outside the fixed reference's range (error 61: ls overflowed) is written as 0
    o[((size_t)b * Hq + kv * G + g) * D + ch] =
        from_f<T>(ls > 0.f && isfinite(ls) ? as / ls : 0.f);
  }
}

// ---------------------------------------------------------------------------------------
int decode_nsplit(const sas_decode_problem& p) {
  const int pairs = p.batch * gate_heads(p);
  int ns = (4 * 148 + pairs - 1) / pairs;   // about 4 CTAs per SM, each a long stream
  if (ns < 1) ns = 1;
  if (ns > p.topk + 1) ns = p.topk + 1;
  return ns;
}

size_t decode_workspace_bytes(const sas_decode_problem& p) {
  const int G = p.num_q_heads / gate_heads(p);
  const size_t pairs = (size_t)p.batch * gate_heads(p);
  const size_t ns = decode_nsplit(p);
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t three = 256 /* error word */ + al(pairs * (p.topk + 1) * 4) * 2 +
                       al(pairs * ns * G * 2 * 4) + al(pairs * ns * G * p.head_dim * 4);
  // either path may run (the choice is process-wide and may change between calls)
  if (!decode_fused_supported(p)) return three;
  const size_t fused = decode_fused_workspace_bytes(p);
  return fused > three ? fused : three;
}

namespace {
bool g_decode_fused = true;
}
bool decode_fused_enabled() { return g_decode_fused; }

template <int G>
static size_t decode_bulk_smem() {
  return (size_t)kAttStages * kAttStage + (size_t)G * 128 * 4 + (size_t)G * 64 * 4 + 3 * 8 * 4 +
         2 * 128 * 4 + kAttStages * 8 + 16 + 128;
}

template <typename T, int D, int G>
static void decode_attn_launch(const sas_decode_problem& p, const void* q, const void* kc,
                               const void* vc, int32_t* sel_idx, float* sel_logg, float* part_ml,
                               float* part_acc, int* err, void* o, int ns,
                               const DecodePaging& pg, cudaStream_t st) {
  const int Hs = gate_heads(p), R = Hs / p.num_kv_heads;   // G: query heads per gate head
  dim3 grid(Hs, p.batch, ns);
  if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
    if (decode_attn_tc_supported(p)) {   // tensor-core path (sas_decode_tc.cu)
      launch_decode_attn_tc(p, q, kc, vc, sel_idx, sel_logg, part_ml, part_acc, err, ns, pg, st);
      decode_merge_kernel<T, D, G><<<dim3(Hs, p.batch), 256, 0, st>>>(part_ml, part_acc, Hs, ns,
                                                                     (T*)o);
      return;
    }
    if (p.block <= 64) {   // bulk-copy streaming path
      const size_t smem = decode_bulk_smem<G>();
      cudaFuncSetAttribute(decode_attn_bulk_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      decode_attn_bulk_kernel<G><<<grid, kDecThreads, smem, st>>>(
          (const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, p.seqlens,
          sel_idx, sel_logg, Hs, R, p.capacity, p.block, p.topk, ns,
          kLog2e / sqrtf((float)D), part_ml, part_acc, err);
      decode_merge_kernel<T, D, G><<<dim3(Hs, p.batch), 256, 0, st>>>(part_ml, part_acc, Hs, ns,
                                                                     (T*)o);
      return;
    }
  }
  decode_attn_kernel<T, D, G><<<grid, kDecThreads, 0, st>>>(
      (const T*)q, (const T*)kc, (const T*)vc, p.seqlens, sel_idx, sel_logg, Hs, R,
      p.capacity, p.block, p.topk, ns, kLog2e / sqrtf((float)D), part_ml, part_acc);
  decode_merge_kernel<T, D, G><<<dim3(Hs, p.batch), 256, 0, st>>>(part_ml, part_acc, Hs, ns,
                                                                 (T*)o);
}

template <typename T>
static void decode_gate_launch(const sas_decode_problem& p, const void* q_nope, const void* gkc,
                               const float* cur_pool, const void* wq, const float* qnorm_w,
                               const void* wk, const float* knorm_w, int32_t* sel_idx,
                               float* sel_logg, int32_t* idx_out, float* logg_out,
                               const DecodePaging& pg, int* err, cudaStream_t st) {
  const int NBmax = (p.capacity + p.block - 1) / p.block;
  const int G = p.num_q_heads / gate_heads(p);
  const size_t smem = (size_t)(G * p.head_dim + 3 * p.head_dim + 2 * p.gate_hidden + NBmax + 1 +
                               3 * kDecWarps + 4 + 256 + NBmax) * sizeof(float);
  dim3 grid(gate_heads(p), p.batch);
#define SAS_DG(H, NPT)                                                                           \
  {                                                                                              \
    cudaFuncSetAttribute(decode_gate_kernel<T, H, NPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                         (int)smem);                                                             \
    decode_gate_kernel<T, H, NPT><<<grid, kDecThreads, smem, st>>>(                              \
        (const T*)q_nope, (const __nv_bfloat16*)gkc, cur_pool, (const T*)wq, qnorm_w, (const T*)wk, \
        knorm_w, p.seqlens, p.gate_rope_cos, p.gate_rope_sin, p.num_q_heads, p.num_kv_heads,      \
        gate_heads(p),                                                                           \
        p.head_dim, p.block, p.topk, NBmax, p.capacity, p.rms_eps, p.ungated, sel_idx, sel_logg, \
        idx_out, logg_out, pg.pt, pg.num_pages, err);                                           \
  }
#define SAS_DG_H(NPT)                              \
  switch (p.gate_hidden) {                         \
    case 32: SAS_DG(32, NPT); break;               \
    case 64: SAS_DG(64, NPT); break;               \
    default: SAS_DG(128, NPT); break;              \
  }
  if (NBmax <= 256) { SAS_DG_H(1) }
  else if (NBmax <= 1024) { SAS_DG_H(4) }
  else if (NBmax <= 2048) { SAS_DG_H(8) }
  else { SAS_DG_H(16) }
#undef SAS_DG_H
#undef SAS_DG
}

sas_status launch_decode(const sas_decode_problem& p, const void* q, const void* q_nope,
                         const void* k_cache, const void* v_cache, const void* gkc,
                         const float* cur_pool, const void* wq, const float* qnorm_w,
                         const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                         float* logg_out, void* ws, const DecodePaging& pg, cudaStream_t st) {
  if (decode_fused_enabled() && decode_fused_supported(p)) {
    SAS_TRY(launch_decode_fused(p, q, q_nope, k_cache, v_cache, gkc, cur_pool, wq, qnorm_w, wk,
                                knorm_w, o, idx_out, logg_out, ws, pg, st));
    return launch_status("decode (fused)", 1);
  }
  const int G = p.num_q_heads / gate_heads(p);   // query heads per gate head
  const size_t pairs = (size_t)p.batch * gate_heads(p);
  const int ns = decode_nsplit(p);
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* w = (char*)ws;
  // word 0: this call's error code (0 = none), cleared first so it never reports an earlier call
  int* err = (int*)w;
  if (cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess) {
    set_error("decode: clearing the error word failed");
    return SAS_ERR_CUDA;
  }
  w += 256;
  int32_t* sel_idx = (int32_t*)w;
  w += al(pairs * (p.topk + 1) * 4);
  float* sel_logg = (float*)w;
  w += al(pairs * (p.topk + 1) * 4);
  float* part_ml = (float*)w;
  w += al(pairs * ns * G * 2 * 4);
  float* part_acc = (float*)w;
  w += al(pairs * ns * G * p.head_dim * 4);
  if (p.dtype == SAS_BF16)
    decode_gate_launch<__nv_bfloat16>(p, q_nope, gkc, cur_pool, wq, qnorm_w, wk, knorm_w, sel_idx,
                                      sel_logg, idx_out, logg_out, pg, err, st);
  else
    decode_gate_launch<float>(p, q_nope, gkc, cur_pool, wq, qnorm_w, wk, knorm_w, sel_idx, sel_logg,
                              idx_out, logg_out, pg, err, st);
  sas_status s = launch_status("decode gate", 1);
  if (s != SAS_OK) return s;
#define SAS_DA(T, D, G)                                                                      \
  decode_attn_launch<T, D, G>(p, q, k_cache, v_cache, sel_idx, sel_logg, part_ml, part_acc, err, \
                              o, ns, pg, st)
#define SAS_DA_G(T, D)                   \
  switch (G) {                           \
    case 1: SAS_DA(T, D, 1); break;      \
    case 2: SAS_DA(T, D, 2); break;      \
    case 4: SAS_DA(T, D, 4); break;      \
    case 5: SAS_DA(T, D, 5); break;      \
    default: SAS_DA(T, D, 8); break;     \
  }
  if (p.dtype == SAS_BF16) {
    if (p.head_dim == 64) { SAS_DA_G(__nv_bfloat16, 64) } else { SAS_DA_G(__nv_bfloat16, 128) }
  } else {
    if (p.head_dim == 64) { SAS_DA_G(float, 64) } else { SAS_DA_G(float, 128) }
  }
#undef SAS_DA_G
#undef SAS_DA
  return launch_status("decode attention", 2);
}

}  // namespace sas

extern "C" sas_status sas_decode_set_fused(int enable) {
  sas::g_decode_fused = enable != 0;
  return SAS_OK;
}
