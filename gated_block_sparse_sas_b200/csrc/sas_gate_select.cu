// A3 + A4 fused: gate scores and Top-K selection in one kernel, so the score matrix
// s[T, Hkv, NBmax] never reaches global memory. Model card "tencent/Simple-Attention-
// Sparsification", table "Checkpoint configuration" (Qproj, max + min + average pooling, Q/K
// normalisation, gate RoPE, Top-K 31 historical blocks); paper abstract (softmax gates over
// the history plus the always-retained current block; Top-K keeps the computation sparse).
//
// CTA = (TQ-token tile of one sequence, gate head), 512 threads (one CTA per SM: the score
// rows fill most of the shared memory, so the CTA brings its own warps to hide latency):
//   1. q~_t: the tensor-core query projection of each token (sas_gate_tc.cu), RMSNorm with
//      its weight, rotary at t; kept transposed in shared memory.
//   2. the current block's key from the tensor-core projection of its visible prefix,
//      RMSNorm, rotary at c_t*B; s_cur[t] = q~_t . k~cur_t / sqrt(h).
//   3. s[t][j] = q~_t . k~_j / sqrt(h) for the historical blocks j < c_t, in fp32 on CUDA
//      cores over chunks of the cached block keys, into a shared-memory row per token
//      (s_cur at j = c_t). The products and their order are those of sas_gate_scores, so
//      the scores, and the selection, are bit-identical to the unfused path.
//   4. one warp per token row: logsumexp over j <= c_t, exact Top-K of the historical
//      scores (bitwise search for the K-th largest key, ties to the lower index, the same
//      routine as sas_topk), the current block last, -1 padding; idx and log-gates out.
// TQ = 64 tokens for NBmax <= 512 (rows of 512 scores), 32 tokens for NBmax <= 1024.
#include <math.h>

#include "sas_common.cuh"
#include "sas_gate.cuh"
#include "sas_kernels.h"

namespace sas {
namespace gsel {

constexpr int kThreads = 512;
constexpr int kH = 128;   // gate hidden size of the fused path
constexpr int kRT = 2;    // tokens per thread in the score GEMM (x 4 blocks)

template <int TQ>
struct Cfg {
  static constexpr int NTY = TQ / kRT;         // groups of kRT tokens
  static constexpr int NTX = kThreads / NTY;   // groups of 4 blocks
  static constexpr int CHUNK = NTX * 4;        // cached block keys staged per step
  static constexpr int QS = TQ + 4;            // row stride of the transposed q~ tile
  static constexpr int BS = CHUNK + 4;         // row stride of the transposed key chunk
  static constexpr int X = TQ * (kH + 1);      // staging of projected rows
  static constexpr int RB = (kH * BS > X ? kH * BS : X);
  static constexpr int FIXED = kH * QS + RB + TQ;   // floats before the score rows
};

// score row stride: a multiple of 4 floats (16-byte rows), shifted by 4 banks per row
inline int score_stride(int NBmax) { return ((NBmax + 3) / 4) * 4 + 4; }

template <int TQ>
size_t smem_bytes(int NBmax) {
  return ((size_t)Cfg<TQ>::FIXED + (size_t)TQ * score_stride(NBmax)) * sizeof(float);
}

template <int TQ>
__global__ void __launch_bounds__(kThreads, 1) gate_select_kernel(
    const float* __restrict__ qproj, const float* __restrict__ kproj,
    const float* __restrict__ gkeys, const float* __restrict__ qnorm_w,
    const float* __restrict__ knorm_w, const int32_t* __restrict__ cu,
    const float* __restrict__ rc, const float* __restrict__ rs, int Hkv, int Hs, int B, int NBmax,
    int SS, int K, float eps, int32_t* __restrict__ idx, float* __restrict__ logg,
    float* __restrict__ lse_out) {
  using C = Cfg<TQ>;
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  float* Qt = smem;                   // [H][QS]   q~ transposed
  float* R = Qt + kH * C::QS;         // staging rows / transposed key chunk
  float* scur = R + C::RB;            // [TQ]
  float* S = scur + TQ;               // [TQ][SS]  score rows

  // gate head sh (a KV head, or a query head with one gate per query head); its block keys
  // and current-block key are KV head kv's
  const int tile = blockIdx.x, b = blockIdx.y, sh = blockIdx.z;
  const int kv = sh / (Hs / Hkv);
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int t0 = tile * TQ;
  if (t0 >= L) return;
  const int nt = min(TQ, L - t0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float sqrt_h = sqrtf((float)kH);

  // ---- 1: q~ ----
  {
    float* X = R;   // [TQ][H+1]
    for (int e = tid; e < TQ * kH; e += kThreads) {
      const int t = e / kH, c = e - t * kH;
      X[t * (kH + 1) + c] = (t < nt) ? qproj[((size_t)(s0 + t0 + t) * Hs + sh) * kH + c] : 0.f;
    }
    __syncthreads();
    for (int t = warp; t < TQ; t += kThreads / 32) {
      if (t < nt)
        norm_rope_row<kH>(X + t * (kH + 1), qnorm_w, eps, rc, rs, t0 + t, X + t * (kH + 1), lane);
      __syncwarp();
      for (int e = lane; e < kH; e += 32) Qt[e * C::QS + t] = (t < nt) ? X[t * (kH + 1) + e] : 0.f;
    }
    __syncthreads();
  }
  // ---- 2: current block's key and score ----
  {
    float* X = R;
    for (int e = tid; e < TQ * kH; e += kThreads) {
      const int t = e / kH, c = e - t * kH;
      X[t * (kH + 1) + c] = (t < nt) ? kproj[((size_t)(s0 + t0 + t) * Hkv + kv) * kH + c] : 0.f;
    }
    __syncthreads();
    for (int t = warp; t < TQ; t += kThreads / 32) {
      if (t < nt) {
        const int cb = ((t0 + t) / B) * B;
        norm_rope_row<kH>(X + t * (kH + 1), knorm_w, eps, rc, rs, cb, X + t * (kH + 1), lane);
        __syncwarp();
        float dot = 0.f;
        for (int e = lane; e < kH; e += 32) dot += Qt[e * C::QS + t] * X[t * (kH + 1) + e];
        dot = warp_sum(dot);
        if (lane == 0) scur[t] = dot / sqrt_h;
      }
    }
    __syncthreads();
  }
  // ---- 3: historical scores into the shared score rows ----
  {
    const int ty = tid / C::NTX, tx = tid - ty * C::NTX;
    float* Bs = R;    // [H][BS]
    const int cmax = (t0 + nt - 1) / B;   // current block of the tile's last token
    for (int j0 = 0; j0 < cmax; j0 += C::CHUNK) {
      for (int e = tid; e < C::CHUNK * kH; e += kThreads) {
        const int jj = e / kH, i = e - jj * kH;
        const int j = j0 + jj;
        Bs[i * C::BS + jj] = (j < cmax) ? gkeys[(((size_t)b * NBmax + j) * Hkv + kv) * kH + i] : 0.f;
      }
      __syncthreads();
      float acc[kRT][4];
#pragma unroll
      for (int a = 0; a < kRT; ++a)
#pragma unroll
        for (int o = 0; o < 4; ++o) acc[a][o] = 0.f;
#pragma unroll 8
      for (int k = 0; k < kH; ++k) {
        const float2 a = *reinterpret_cast<const float2*>(Qt + k * C::QS + ty * kRT);
        const float4 bb = *reinterpret_cast<const float4*>(Bs + k * C::BS + tx * 4);
        const float av[kRT] = {a.x, a.y};
        const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
        for (int aa = 0; aa < kRT; ++aa)
#pragma unroll
          for (int o = 0; o < 4; ++o) acc[aa][o] = fmaf(av[aa], bv[o], acc[aa][o]);
      }
#pragma unroll
      for (int aa = 0; aa < kRT; ++aa) {
        const int t = ty * kRT + aa;
        const int ct = (t0 + t) / B;
        float* srow = S + (size_t)t * SS;
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const int j = j0 + tx * 4 + o;
          if (t < nt && j < ct) srow[j] = acc[aa][o] / sqrt_h;
        }
      }
      __syncthreads();
    }
    for (int t = tid; t < nt; t += kThreads) S[(size_t)t * SS + (t0 + t) / B] = scur[t];
    __syncthreads();
  }
  // ---- 4: logsumexp and Top-K, one warp per token row ----
  for (int t = warp; t < nt; t += kThreads / 32) {
    const int c = (t0 + t) / B;
    const float* srow = S + (size_t)t * SS;
    float m = -INFINITY;
    for (int j = lane; j <= c; j += 32) m = fmaxf(m, srow[j]);
    m = warp_max(m);
    float l = 0.f;
    for (int j = lane; j <= c; j += 32) l += expf(srow[j] - m);
    l = warp_sum(l);
    const float lse = m + logf(l);
    const size_t row = (size_t)(s0 + t0 + t) * Hs + sh;
    int32_t* irow = idx + row * (K + 1);
    float* grow = logg + row * (K + 1);
    if (lse_out != nullptr && lane == 0) lse_out[row] = lse;
    if (c <= K) {
      for (int s = lane; s <= K; s += 32) {
        if (s <= c) { irow[s] = s; grow[s] = srow[s] - lse; }
        else { irow[s] = -1; grow[s] = 0.f; }
      }
      continue;
    }
    if (c <= 64) topk_row<2>(srow, lse, c, K, lane, irow, grow);
    else if (c <= 128) topk_row<4>(srow, lse, c, K, lane, irow, grow);
    else if (c <= 256) topk_row<8>(srow, lse, c, K, lane, irow, grow);
    else if (TQ == 64 || c <= 512) topk_row<16>(srow, lse, c, K, lane, irow, grow);
    else topk_row<32>(srow, lse, c, K, lane, irow, grow);
    if (lane == 0) {
      irow[K] = c;
      grow[K] = srow[c] - lse;
    }
  }
}

}  // namespace gsel

static size_t al256s(size_t x) { return (x + 255) & ~(size_t)255; }

bool gate_select_fused(const sas_problem& p) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  return gate_tc_supported(p) && NBmax <= 1024;
}

size_t gate_select_workspace_bytes(const sas_problem& p) {
  if (gate_select_fused(p)) return gate_tc_workspace_bytes(p);
  // other shapes: sas_gate_scores' own workspace, then the scores and their logsumexp
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const size_t rows = (size_t)p.total_tokens * gate_heads(p);
  return al256s(gate_scores_workspace_bytes(p)) + al256s(rows * NBmax * 4) + al256s(rows * 4);
}

sas_status launch_gate_select(const sas_problem& p, const void* q_nope, const void* k_nope,
                              const float* gkeys, const void* wq, const float* qnorm_w,
                              const void* wk, const float* knorm_w, int32_t* idx, float* logg,
                              float* lse, void* workspace, cudaStream_t st) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  if (!gate_select_fused(p)) {
    const size_t rows = (size_t)p.total_tokens * gate_heads(p);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* scores = reinterpret_cast<float*>(ws + al256s(gate_scores_workspace_bytes(p)));
    float* slse = lse != nullptr
                      ? lse
                      : reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(scores) +
                                                 al256s(rows * NBmax * 4));
    SAS_TRY(launch_gate_scores(p, q_nope, k_nope, gkeys, wq, qnorm_w, wk, knorm_w, scores, slse,
                               workspace, st));
    return launch_topk(p, scores, slse, idx, logg, st);
  }
  float *qproj = nullptr, *kproj = nullptr;
  SAS_TRY(launch_gate_proj_tc(p, q_nope, k_nope, wq, wk, workspace, &qproj, &kproj, st));
  const int SS = gsel::score_stride(NBmax);
#define SAS_GSEL(TQ)                                                                         \
  {                                                                                          \
    const size_t smem = gsel::smem_bytes<TQ>(NBmax);                                          \
    cudaFuncSetAttribute(gsel::gate_select_kernel<TQ>,                                        \
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);             \
    const dim3 grid((p.max_seqlen + TQ - 1) / TQ, p.batch, gate_heads(p));                   \
    gsel::gate_select_kernel<TQ><<<grid, gsel::kThreads, smem, st>>>(                         \
        qproj, kproj, gkeys, qnorm_w, knorm_w, p.cu_seqlens, p.gate_rope_cos, p.gate_rope_sin, \
        p.num_kv_heads, gate_heads(p), p.block, NBmax, SS, p.topk, p.rms_eps, idx, logg, lse);\
  }
  if (NBmax <= 512) SAS_GSEL(64)
  else SAS_GSEL(32)
#undef SAS_GSEL
  return launch_status("gate_select (fused scores + Top-K)", 4);
}

}  // namespace sas
