// Gate router kernels: key-block pooling (A1), gate block keys (A2), gate scores (A3)
// and Top-K selection (A4). Model card "tencent/Simple-Attention-Sparsification",
// table "Checkpoint configuration" (block 64, Top-K 31, gate hidden 128, Qproj,
// max + min + average pooling, Q/K normalization, gate RoPE); paper abstract (softmax
// gates over history plus the always-retained current block).
//
// All gate arithmetic is fp32 on CUDA cores: the selection must match the exact one
// bit for bit except at near-ties, so no reduced-precision tensor-core math here.
#include <math.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_gate.cuh"
#include "sas_kernels.h"

namespace sas {

// ---------------------------------------------------------------------------------------
// A1: pooled[b, j, kv, :] = (max | min | mean) of k_nope over the tokens of block j.
// One CTA per (block, sequence); threads stride over the (kv, channel) pairs, so each
// token row is read once, coalesced.
// ---------------------------------------------------------------------------------------
template <typename T>
__global__ void pool_keys_kernel(const T* __restrict__ k_nope, const int32_t* __restrict__ cu,
                                 int Hkv, int d, int B, int NBmax, float* __restrict__ pooled) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int HD = Hkv * d;
  float* out = pooled + ((size_t)b * NBmax + j) * (size_t)HD * 3;
  const int t0 = j * B;
  if (t0 >= L) {
    for (int e = threadIdx.x; e < 3 * HD; e += blockDim.x) out[e] = 0.f;
    return;
  }
  const int n = min(B, L - t0);
  const T* src = k_nope + (size_t)(s0 + t0) * HD;
  for (int e = threadIdx.x; e < HD; e += blockDim.x) {
    float mx = -INFINITY, mn = INFINITY, sm = 0.f;
    for (int i = 0; i < n; ++i) {
      const float x = to_f(src[(size_t)i * HD + e]);
      mx = fmaxf(mx, x);
      mn = fminf(mn, x);
      sm += x;
    }
    const int kv = e / d, c = e - kv * d;
    float* o = out + (size_t)kv * 3 * d;
    o[c] = mx;
    o[d + c] = mn;
    o[2 * d + c] = sm / (float)n;
  }
}

sas_status launch_pool_keys(const sas_problem& p, const void* k_nope, float* pooled,
                            cudaStream_t st) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  dim3 grid(NBmax, p.batch);
  if (p.dtype == SAS_BF16)
    pool_keys_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)k_nope, p.cu_seqlens,
                                           p.num_kv_heads, p.head_dim, p.block, NBmax, pooled);
  else
    pool_keys_kernel<<<grid, 256, 0, st>>>((const float*)k_nope, p.cu_seqlens, p.num_kv_heads,
                                           p.head_dim, p.block, NBmax, pooled);
  return launch_status("pool_keys", 1);
}

// ---------------------------------------------------------------------------------------
// A2: k~ = rope(RMSNorm(Wk . pooled), pos = j*B). CTA = (kv head, 16 consecutive (b, j)
// rows); thread i computes output channel i for all 16 rows, so each Wk row is read once
// per CTA.
// ---------------------------------------------------------------------------------------
constexpr int kGkRows = 16;

template <typename T, int H>
__global__ void __launch_bounds__(H) gate_keys_kernel(
    const float* __restrict__ pooled, const T* __restrict__ wk, const float* __restrict__ knorm_w,
    const int32_t* __restrict__ cu, const float* __restrict__ rc, const float* __restrict__ rs,
    int batch, int NBmax, int Hkv, int d, int B, float eps, float* __restrict__ gkeys) {
  extern __shared__ float smem[];
  const int C = 3 * d;
  float* P = smem;                      // [kGkRows][C]
  float* X = smem + kGkRows * C;        // [kGkRows][H]
  const int kv = blockIdx.y;
  const int first = blockIdx.x * kGkRows;
  const int nrows = batch * NBmax;
  for (int e = threadIdx.x; e < kGkRows * C; e += blockDim.x) {
    const int r = e / C, c = e - r * C, fj = first + r;
    P[e] = (fj < nrows) ? pooled[((size_t)fj * Hkv + kv) * C + c] : 0.f;
  }
  __syncthreads();
  const int i = threadIdx.x;
  float acc[kGkRows];
#pragma unroll
  for (int r = 0; r < kGkRows; ++r) acc[r] = 0.f;
  const T* w = wk + ((size_t)kv * H + i) * C;
  for (int c0 = 0; c0 < C; c0 += 8) {
    float wv[8];
    load8<T>(w + c0, wv);
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int r = 0; r < kGkRows; ++r) acc[r] = fmaf(wv[u], P[r * C + c0 + u], acc[r]);
  }
#pragma unroll
  for (int r = 0; r < kGkRows; ++r) X[r * H + i] = acc[r];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < kGkRows; r += H / 32) {
    const int fj = first + r;
    if (fj >= nrows) continue;
    const int b = fj / NBmax, j = fj - b * NBmax;
    const int L = cu[b + 1] - cu[b];
    float* dst = gkeys + ((size_t)fj * Hkv + kv) * H;
    if (j * B >= L) {
      for (int e = lane; e < H; e += 32) dst[e] = 0.f;
      continue;
    }
    norm_rope_row<H>(X + r * H, knorm_w, eps, rc, rs, j * B, dst, lane);
  }
}

template <typename T>
static sas_status gate_keys_dispatch(const sas_problem& p, const float* pooled, const void* wk,
                                     const float* knorm_w, float* gkeys, cudaStream_t st) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  dim3 grid((p.batch * NBmax + kGkRows - 1) / kGkRows, p.num_kv_heads);
  const size_t smem = (size_t)kGkRows * (3 * p.head_dim + p.gate_hidden) * sizeof(float);
#define SAS_GK(H)                                                                           \
  gate_keys_kernel<T, H><<<grid, H, smem, st>>>(pooled, (const T*)wk, knorm_w, p.cu_seqlens, \
                                                p.gate_rope_cos, p.gate_rope_sin, p.batch,  \
                                                NBmax, p.num_kv_heads, p.head_dim, p.block, \
                                                p.rms_eps, gkeys)
  switch (p.gate_hidden) {
    case 32: SAS_GK(32); break;
    case 64: SAS_GK(64); break;
    default: SAS_GK(128); break;
  }
#undef SAS_GK
  return launch_status("gate_keys", 1);
}

sas_status launch_gate_keys(const sas_problem& p, const float* pooled, const void* wk,
                            const float* knorm_w, float* gkeys, cudaStream_t st) {
  return p.dtype == SAS_BF16 ? gate_keys_dispatch<__nv_bfloat16>(p, pooled, wk, knorm_w, gkeys, st)
                             : gate_keys_dispatch<float>(p, pooled, wk, knorm_w, gkeys, st);
}

// ---------------------------------------------------------------------------------------
// A3: gate scores. CTA = (64-token tile of one sequence, kv head), 256 threads.
//   phase 1: qhat[64][H] = qcat[64][G*d] . Wq^T   (register-tiled SIMT GEMM, fp32)
//            -> RMSNorm, rotary at t -> q~ (kept transposed in smem)
//   phase 2: prefix pooling of the current block for every token (running max/min/sum
//            scan), khat_cur[64][H] = Pprefix[64][3d] . Wk^T -> RMSNorm, rotary at c_t*B
//            -> s_cur[t] = q~_t . k~cur_t / sqrt(H)
//   phase 3: s[t][j] = q~_t . k~_j / sqrt(H) over 64-block chunks of the cached block keys,
//            written for j < c_t (s_cur at j = c_t, -inf past it), with an online
//            logsumexp per token.
// Tiles start at multiples of 64 tokens within a sequence, so with B | 64 every block
// that a tile's tokens sit in starts inside the tile.
// ---------------------------------------------------------------------------------------
constexpr int kTQ = 64;         // tokens per tile
constexpr int kGsThreads = 256;
constexpr int kKC = 32;         // reduction chunk of the query projection
constexpr int kAP = kTQ + 4;    // padded row of transposed A tiles

template <int H, bool PROJ = false>
struct GsSmem {
  // floats
  static constexpr int QT = H * kAP;                  // q~ transposed [H][kAP]
  static constexpr int X = kTQ * (H + 1);             // row staging [64][H+1]
  static constexpr int P1 = kKC * kAP + kKC * (H + 4);  // phase-1 A/B chunks
  static constexpr int KT = kTQ * 129;                // token keys [64][d+1] (d <= 128)
  static constexpr int P2 = 64 * kAP + 64 * (H + 4);  // phase-2 A/B chunks
  static constexpr int P3 = H * kAP;                  // block-key chunk [H][kAP]
  static constexpr int R1 = (P1 > X ? P1 : X);
  static constexpr int R2a = KT + P2;
  static constexpr int R2 = (R2a > X + KT ? R2a : X + KT);
  static constexpr int RMAX0 = PROJ ? X : (R1 > R2 ? R1 : R2);   // PROJ: only row staging
  static constexpr int RMAX = (RMAX0 > P3 ? RMAX0 : P3);
  static constexpr int TOTAL = QT + RMAX + kTQ;       // + s_cur[64]
};

// PROJ: the two projections come precomputed (tensor-core GEMMs, sas_gate_tc.cu) as
// qproj [T, Hs, H] / kproj [T, Hkv, H] fp32, so phases 1 and 2 only load, normalise and
// rotate them.
template <typename T, int H, bool PROJ>
__global__ void __launch_bounds__(kGsThreads) gate_scores_kernel(
    const T* __restrict__ q_nope, const T* __restrict__ k_nope, const float* __restrict__ gkeys,
    const T* __restrict__ wq, const float* __restrict__ qnorm_w, const T* __restrict__ wk,
    const float* __restrict__ knorm_w, const int32_t* __restrict__ cu,
    const float* __restrict__ rc, const float* __restrict__ rs, int Hq, int Hkv, int Hs, int d,
    int B, int NBmax, float eps, const float* __restrict__ qproj, const float* __restrict__ kproj,
    float* __restrict__ scores, float* __restrict__ lse) {
  extern __shared__ float smem[];
  using S = GsSmem<H, PROJ>;
  constexpr int NO = H / 16;   // outputs per thread in the 64 x H GEMMs
  float* Qt = smem;            // [H][kAP]
  float* R = smem + S::QT;     // phase-dependent region
  float* scur = R + S::RMAX;   // [64]

  // gate head sh: its Gs query heads feed the query projection; its keys are KV head kv's
  const int tile = blockIdx.x, b = blockIdx.y, sh = blockIdx.z;
  const int kv = sh / (Hs / Hkv);
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int t0 = tile * kTQ;
  if (t0 >= L) return;
  const int nt = min(kTQ, L - t0);
  const int G = Hq / Hs, GD = G * d;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int warp = tid >> 5, lane = tid & 31;

  // ---------------- phase 1: query projection ----------------
  if constexpr (PROJ) {
    float* X = R;  // [64][H+1]
    for (int e = tid; e < kTQ * H; e += kGsThreads) {
      const int t = e / H, c = e - t * H;
      X[t * (H + 1) + c] = (t < nt) ? qproj[((size_t)(s0 + t0 + t) * Hs + sh) * H + c] : 0.f;
    }
    __syncthreads();
    for (int t = warp; t < kTQ; t += kGsThreads / 32) {
      if (t < nt) {
        norm_rope_row<H>(X + t * (H + 1), qnorm_w, eps, rc, rs, t0 + t, X + t * (H + 1), lane);
      }
      __syncwarp();
      for (int e = lane; e < H; e += 32) Qt[e * kAP + t] = (t < nt) ? X[t * (H + 1) + e] : 0.f;
    }
    __syncthreads();
  } else {
    float acc[4][NO];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int o = 0; o < NO; ++o) acc[a][o] = 0.f;
    float* As = R;                    // [kKC][kAP]
    float* Bs = R + kKC * kAP;        // [kKC][H+4]
    for (int k0 = 0; k0 < GD; k0 += kKC) {
      {  // A: 64 tokens x 32 -> 256 threads x 8
        const int t = tid >> 2, part = tid & 3;
        float v[8];
        if (t < nt) {
          load8<T>(q_nope + ((size_t)(s0 + t0 + t) * Hq + (size_t)sh * G) * d + k0 + part * 8, v);
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) As[(part * 8 + u) * kAP + t] = v[u];
      }
      for (int e = tid; e < H * (kKC / 8); e += kGsThreads) {  // B: H x 32
        const int i = e / (kKC / 8), part = e - i * (kKC / 8);
        float v[8];
        load8<T>(wq + ((size_t)sh * H + i) * GD + k0 + part * 8, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) Bs[(part * 8 + u) * (H + 4) + i] = v[u];
      }
      __syncthreads();
#pragma unroll 8
      for (int k = 0; k < kKC; ++k) {
        const float4 a = *reinterpret_cast<const float4*>(As + k * kAP + ty * 4);
        float bv[NO];
#pragma unroll
        for (int o = 0; o < NO; ++o) bv[o] = Bs[k * (H + 4) + tx * NO + o];
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int aa = 0; aa < 4; ++aa)
#pragma unroll
          for (int o = 0; o < NO; ++o) acc[aa][o] = fmaf(av[aa], bv[o], acc[aa][o]);
      }
      __syncthreads();
    }
    float* X = R;  // [64][H+1]
#pragma unroll
    for (int aa = 0; aa < 4; ++aa)
#pragma unroll
      for (int o = 0; o < NO; ++o) X[(ty * 4 + aa) * (H + 1) + tx * NO + o] = acc[aa][o];
    __syncthreads();
    for (int t = warp; t < kTQ; t += kGsThreads / 32) {
      if (t < nt) {
        norm_rope_row<H>(X + t * (H + 1), qnorm_w, eps, rc, rs, t0 + t, X + t * (H + 1), lane);
      }
      __syncwarp();
      for (int e = lane; e < H; e += 32) Qt[e * kAP + t] = (t < nt) ? X[t * (H + 1) + e] : 0.f;
    }
    __syncthreads();
  }

  // ---------------- phase 2: current-block keys ----------------
  if constexpr (PROJ) {
    float* X = R;  // [64][H+1]
    for (int e = tid; e < kTQ * H; e += kGsThreads) {
      const int t = e / H, c = e - t * H;
      X[t * (H + 1) + c] = (t < nt) ? kproj[((size_t)(s0 + t0 + t) * Hkv + kv) * H + c] : 0.f;
    }
    __syncthreads();
    for (int t = warp; t < kTQ; t += kGsThreads / 32) {
      if (t < nt) {
        const int cb = ((t0 + t) / B) * B;
        norm_rope_row<H>(X + t * (H + 1), knorm_w, eps, rc, rs, cb, X + t * (H + 1), lane);
        __syncwarp();
        float dot = 0.f;
        for (int e = lane; e < H; e += 32) dot += Qt[e * kAP + t] * X[t * (H + 1) + e];
        dot = warp_sum(dot);
        if (lane == 0) scur[t] = dot / sqrtf((float)H);
      }
    }
    __syncthreads();
  } else {
    float* KT = R;                       // [64][d+1] token keys of this kv head (fp32)
    float* As = R + S::KT;               // [64 pooled channels][kAP]
    float* Bs = As + 64 * kAP;           // [64][H+4]
    for (int e = tid; e < kTQ * d; e += kGsThreads) {
      const int t = e / d, c = e - t * d;
      KT[t * 129 + c] = (t < nt) ? to_f(k_nope[((size_t)(s0 + t0 + t) * Hkv + kv) * d + c]) : 0.f;
    }
    float acc[4][NO];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int o = 0; o < NO; ++o) acc[a][o] = 0.f;
    __syncthreads();
    const int C = 3 * d;
    for (int c0 = 0; c0 < C; c0 += 64) {
      const int part = c0 / d, e0 = c0 - part * d;   // 0 max, 1 min, 2 mean
      if (tid < 64) {
        const int c = e0 + tid;
        float run = 0.f;
        for (int t = 0; t < kTQ; ++t) {
          const int r = t % B;   // in-block index (tile starts on a block boundary)
          const float x = KT[t * 129 + c];
          if (r == 0) run = x;
          else if (part == 0) run = fmaxf(run, x);
          else if (part == 1) run = fminf(run, x);
          else run += x;
          As[tid * kAP + t] = (part == 2) ? run / (float)(r + 1) : run;
        }
      } else {
        for (int e = tid - 64; e < H * 8; e += kGsThreads - 64) {  // Wk chunk: H x 64
          const int i = e >> 3, pp = e & 7;
          float v[8];
          load8<T>(wk + ((size_t)kv * H + i) * C + c0 + pp * 8, v);
#pragma unroll
          for (int u = 0; u < 8; ++u) Bs[(pp * 8 + u) * (H + 4) + i] = v[u];
        }
      }
      __syncthreads();
#pragma unroll 8
      for (int k = 0; k < 64; ++k) {
        const float4 a = *reinterpret_cast<const float4*>(As + k * kAP + ty * 4);
        float bv[NO];
#pragma unroll
        for (int o = 0; o < NO; ++o) bv[o] = Bs[k * (H + 4) + tx * NO + o];
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int aa = 0; aa < 4; ++aa)
#pragma unroll
          for (int o = 0; o < NO; ++o) acc[aa][o] = fmaf(av[aa], bv[o], acc[aa][o]);
      }
      __syncthreads();
    }
    float* X = R + S::KT;  // [64][H+1], over the finished GEMM chunks
#pragma unroll
    for (int aa = 0; aa < 4; ++aa)
#pragma unroll
      for (int o = 0; o < NO; ++o) X[(ty * 4 + aa) * (H + 1) + tx * NO + o] = acc[aa][o];
    __syncthreads();
    for (int t = warp; t < kTQ; t += kGsThreads / 32) {
      if (t < nt) {
        const int cb = ((t0 + t) / B) * B;
        norm_rope_row<H>(X + t * (H + 1), knorm_w, eps, rc, rs, cb, X + t * (H + 1), lane);
        __syncwarp();
        float dot = 0.f;
        for (int e = lane; e < H; e += 32) dot += Qt[e * kAP + t] * X[t * (H + 1) + e];
        dot = warp_sum(dot);
        if (lane == 0) scur[t] = dot / sqrtf((float)H);
      }
    }
    __syncthreads();
  }

  // ---------------- phase 3: historical scores + logsumexp ----------------
  {
    float* Bs = R;  // [H][kAP] block keys of a 64-block chunk, transposed
    const int cmax = (t0 + nt - 1) / B;  // current block of the last token
    float m[4], l[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) { m[a] = -INFINITY; l[a] = 0.f; }
    const float sqrt_h = sqrtf((float)H);
    for (int j0 = 0; j0 < NBmax; j0 += 64) {
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int o = 0; o < 4; ++o) acc[a][o] = 0.f;
      const bool need = j0 < cmax;
      if (need) {
        for (int e = tid; e < 64 * H; e += kGsThreads) {
          const int jj = e / H, i = e - jj * H;
          const int j = j0 + jj;
          Bs[i * kAP + jj] = (j < cmax) ? gkeys[(((size_t)b * NBmax + j) * Hkv + kv) * H + i] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < H; ++k) {
          const float4 a = *reinterpret_cast<const float4*>(Qt + k * kAP + ty * 4);
          const float4 bb = *reinterpret_cast<const float4*>(Bs + k * kAP + tx * 4);
          const float av[4] = {a.x, a.y, a.z, a.w};
          const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
          for (int aa = 0; aa < 4; ++aa)
#pragma unroll
            for (int o = 0; o < 4; ++o) acc[aa][o] = fmaf(av[aa], bv[o], acc[aa][o]);
        }
        __syncthreads();
      }
#pragma unroll
      for (int aa = 0; aa < 4; ++aa) {
        const int t = ty * 4 + aa;
        if (t >= nt) continue;
        const int ct = (t0 + t) / B;
        float* srow = scores + ((size_t)(s0 + t0 + t) * Hs + sh) * NBmax;
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const int j = j0 + tx * 4 + o;
          if (j >= NBmax) continue;
          float v;
          if (j < ct) v = acc[aa][o] / sqrt_h;
          else if (j == ct) v = scur[t];
          else v = -INFINITY;
          srow[j] = v;
          if (j <= ct) {
            if (v > m[aa]) { l[aa] = l[aa] * expf(m[aa] - v) + 1.f; m[aa] = v; }
            else l[aa] += expf(v - m[aa]);
          }
        }
      }
    }
    // merge (m, l) over the 16 threads of a token row (contiguous lanes tx = 0..15)
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      float mm = m[aa], ll = l[aa];
#pragma unroll
      for (int off = 8; off; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mm, off);
        const float l2 = __shfl_xor_sync(0xffffffffu, ll, off);
        const float M = fmaxf(mm, m2);
        if (M == -INFINITY) { ll = 0.f; }
        else ll = ll * expf(mm - M) + l2 * expf(m2 - M);
        mm = M;
      }
      const int t = ty * 4 + aa;
      if (tx == 0 && t < nt) lse[(size_t)(s0 + t0 + t) * Hs + sh] = mm + logf(ll);
    }
  }
}

template <typename T>
static sas_status gate_scores_dispatch(const sas_problem& p, const void* q_nope, const void* k_nope,
                                       const float* gkeys, const void* wq, const float* qnorm_w,
                                       const void* wk, const float* knorm_w, float* scores,
                                       float* lse, void* workspace, cudaStream_t st) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const int Hs = gate_heads(p);
  dim3 grid((p.max_seqlen + kTQ - 1) / kTQ, p.batch, Hs);
  if (gate_hist_tc_supported(p)) {   // projections, then the historical scores on the tensor cores
    float *qproj = nullptr, *kproj = nullptr;
    SAS_TRY(launch_gate_proj_tc(p, q_nope, k_nope, wq, wk, workspace, &qproj, &kproj, st));
    char* extra = (char*)workspace + gate_tc_workspace_bytes(p);
    const size_t qbytes = ((size_t)p.total_tokens * Hs * 128 * 4 + 255) & ~(size_t)255;
    float* qhi = (float*)extra;
    float* qlo = (float*)(extra + qbytes);
    void* key_ws = extra + 2 * qbytes;
    SAS_TRY(launch_gate_hist_tc(p, gkeys, qproj, kproj, qnorm_w, knorm_w, qhi, qlo, key_ws, scores,
                                lse, (int*)workspace, st));
    return launch_status("gate_scores (tensor-core projections and historical scores)", 6);
  }
  if (gate_tc_supported(p)) {   // projections on the tensor cores, then norms, rotary, scores
    float *qproj = nullptr, *kproj = nullptr;
    SAS_TRY(launch_gate_proj_tc(p, q_nope, k_nope, wq, wk, workspace, &qproj, &kproj, st));
    const size_t smem = (size_t)GsSmem<128, true>::TOTAL * sizeof(float);
    static std::once_flag once;
    std::call_once(once, [smem] {
      cudaFuncSetAttribute(gate_scores_kernel<T, 128, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    gate_scores_kernel<T, 128, true><<<grid, kGsThreads, smem, st>>>(
        (const T*)q_nope, (const T*)k_nope, gkeys, (const T*)wq, qnorm_w, (const T*)wk, knorm_w,
        p.cu_seqlens, p.gate_rope_cos, p.gate_rope_sin, p.num_q_heads, p.num_kv_heads, Hs,
        p.head_dim, p.block, NBmax, p.rms_eps, qproj, kproj, scores, lse);
    return launch_status("gate_scores (tensor-core projections)", 4);
  }
#define SAS_GS(H)                                                                             \
  {                                                                                           \
    const size_t smem = (size_t)GsSmem<H>::TOTAL * sizeof(float);                             \
    cudaFuncSetAttribute(gate_scores_kernel<T, H, false>,                                     \
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);              \
    gate_scores_kernel<T, H, false><<<grid, kGsThreads, smem, st>>>(                          \
        (const T*)q_nope, (const T*)k_nope, gkeys, (const T*)wq, qnorm_w, (const T*)wk,        \
        knorm_w, p.cu_seqlens, p.gate_rope_cos, p.gate_rope_sin, p.num_q_heads,               \
        p.num_kv_heads, Hs, p.head_dim, p.block, NBmax, p.rms_eps, nullptr, nullptr, scores,   \
        lse);                                                                                  \
  }
  switch (p.gate_hidden) {
    case 32: SAS_GS(32); break;
    case 64: SAS_GS(64); break;
    default: SAS_GS(128); break;
  }
#undef SAS_GS
  return launch_status("gate_scores", 1);
}

size_t gate_scores_workspace_bytes(const sas_problem& p) {
  if (gate_hist_tc_supported(p)) {   // + q~ hi, lo and the key splits
    const size_t qbytes = ((size_t)p.total_tokens * gate_heads(p) * 128 * 4 + 255) & ~(size_t)255;
    return gate_tc_workspace_bytes(p) + 2 * qbytes + gate_hist_tc_workspace_bytes(p);
  }
  return gate_tc_supported(p) ? gate_tc_workspace_bytes(p) : 256;
}

sas_status launch_gate_scores(const sas_problem& p, const void* q_nope, const void* k_nope,
                              const float* gkeys, const void* wq, const float* qnorm_w,
                              const void* wk, const float* knorm_w, float* scores, float* lse,
                              void* workspace, cudaStream_t st) {
  if (p.dtype == SAS_BF16)
    return gate_scores_dispatch<__nv_bfloat16>(p, q_nope, k_nope, gkeys, wq, qnorm_w, wk, knorm_w,
                                               scores, lse, workspace, st);
  return gate_scores_dispatch<float>(p, q_nope, k_nope, gkeys, wq, qnorm_w, wk, knorm_w, scores,
                                     lse, workspace, st);
}

// ---------------------------------------------------------------------------------------
// A4: Top-K. One warp per (token, kv) row. The K-th largest score is found exactly by a
// radix select over order-preserving uint32 keys held in registers (four 8-bit digit rounds,
// warp-private shared counters); then the row is emitted in ascending block order with
// ballots: every key above the threshold, plus the lowest-index ties at the threshold until K
// are kept.
// ---------------------------------------------------------------------------------------
// The key count per lane follows the row's own candidate count c_t (warp-uniform), so the
// work of a row scales with its visible blocks, not with the longest sequence. MAXNPL bounds
// the instantiated sizes (and so the registers) by the problem's NBmax.
constexpr int kTopkThreads = 256;

template <int MAXNPL>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, const float* __restrict__ lse,
                            const int32_t* __restrict__ cu, int batch, int T, int Hkv, int NBmax,
                            int B, int K, int32_t* __restrict__ idx, float* __restrict__ logg) {
  __shared__ int hist_s[kTopkThreads / 32][256];   // per-warp radix counters
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  int* hist = hist_s[threadIdx.x >> 5];
  if (row >= T * Hkv) return;
  const int tg = row / Hkv;
  const int b = seq_of(cu, batch, tg);
  const int t = tg - cu[b];
  const int c = t / B;
  const float* srow = scores + (size_t)row * NBmax;
  const float l = lse[row];
  int32_t* irow = idx + (size_t)row * (K + 1);
  float* grow = logg + (size_t)row * (K + 1);
  if (c <= K) {
    for (int s = lane; s <= K; s += 32) {
      if (s <= c) { irow[s] = s; grow[s] = srow[s] - l; }
      else { irow[s] = -1; grow[s] = 0.f; }
    }
    return;
  }
  if (MAXNPL <= 2 || c <= 64) topk_row_radix<2>(srow, l, c, K, lane, hist, irow, grow);
  else if (MAXNPL <= 4 || c <= 128) topk_row_radix<(MAXNPL < 4 ? MAXNPL : 4)>(srow, l, c, K, lane, hist, irow, grow);
  else if (MAXNPL <= 8 || c <= 256) topk_row_radix<(MAXNPL < 8 ? MAXNPL : 8)>(srow, l, c, K, lane, hist, irow, grow);
  else if (MAXNPL <= 16 || c <= 512) topk_row_radix<(MAXNPL < 16 ? MAXNPL : 16)>(srow, l, c, K, lane, hist, irow, grow);
  else if (MAXNPL <= 32 || c <= 1024) topk_row_radix<(MAXNPL < 32 ? MAXNPL : 32)>(srow, l, c, K, lane, hist, irow, grow);
  else topk_row_radix<MAXNPL>(srow, l, c, K, lane, hist, irow, grow);
  if (lane == 0) {
    irow[K] = c;
    grow[K] = srow[c] - l;
  }
}

sas_status launch_topk(const sas_problem& p, const float* scores, const float* lse, int32_t* idx,
                       float* logg, cudaStream_t st) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const int rows = p.total_tokens * gate_heads(p);
  const int threads = kTopkThreads;
  const int grid = (int)(((size_t)rows * 32 + threads - 1) / threads);
#define SAS_TK(N)                                                                              \
  topk_kernel<N><<<grid, threads, 0, st>>>(scores, lse, p.cu_seqlens, p.batch, p.total_tokens,  \
                                           gate_heads(p), NBmax, p.block, p.topk, idx, logg)
  if (NBmax <= 64) SAS_TK(2);
  else if (NBmax <= 256) SAS_TK(8);
  else if (NBmax <= 512) SAS_TK(16);
  else if (NBmax <= 1024) SAS_TK(32);
  else SAS_TK(64);
#undef SAS_TK
  return launch_status("topk", 1);
}

}  // namespace sas
