// CUDA-core gated sparse attention, forward (A5) and backward (A6).
//
// These kernels serve the shapes the tensor-core path does not take (fp32 inputs,
// head_dim 64) and give a second, independent GPU implementation. One warp owns one
// (token, gate head) row: the G query heads of the gate head share the row's selection
// (README (b): per-query Top-K blocks with a continuous gate; abstract: the gate enters
// the attention softmax in log form), each lane holds d/32 channels of every head. A gate
// head is a KV head (one gate per KV group: Hs = Hkv, R = 1) or a query head (one gate per
// query head: Hs = Hq, G = 1 here, R = Hq / Hkv); its keys and values are those of KV head
// s / R.
#include <math.h>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {

template <typename T, int E>
__device__ __forceinline__ void load_vec(const T* p, float* out) {
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = to_f(p[e]);
}

template <typename T, int E>
__device__ __forceinline__ void store_vec(T* p, const float* v) {
#pragma unroll
  for (int e = 0; e < E; ++e) p[e] = from_f<T>(v[e]);
}

// ---------------------------------------------------------------------------------------
// forward: online softmax over the keys of the row's selected blocks, in slot order.
// ---------------------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void __launch_bounds__(128) attn_fwd_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const int32_t* __restrict__ idx, const float* __restrict__ logg, const int32_t* __restrict__ cu,
    int batch, int T_total, int Hkv, int R, int B, int K, float scale_log2, T* __restrict__ o,
    float* __restrict__ lse) {
  constexpr int E = D / 32;
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T_total * Hkv) return;
  const int tg = row / Hkv, kv = row - tg * Hkv;   // kv: gate head; its K/V head is kv / R
  const int b = seq_of(cu, batch, tg);
  const int s0 = cu[b], t = tg - s0;
  const int Hq = Hkv * G;
  const int Hk = Hkv / R, kh = kv / R;
  float qr[G][E], acc[G][E], m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    load_vec<T, E>(q + ((size_t)tg * Hq + kv * G + g) * D + lane * E, qr[g]);
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[g][e] = 0.f;
  }
  const int32_t* ir = idx + (size_t)row * (K + 1);
  const float* gr = logg + (size_t)row * (K + 1);
  for (int s = 0; s <= K; ++s) {
    const int j = ir[s];
    if (j < 0) break;
    const float bias = gr[s] * kLog2e;
    const int i0 = j * B, i1 = min(i0 + B, t + 1);
    for (int i = i0; i < i1; ++i) {
      float kk[E], vv[E];
      const size_t off = ((size_t)(s0 + i) * Hk + kh) * D + lane * E;
      load_vec<T, E>(k + off, kk);
      load_vec<T, E>(v + off, vv);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float p = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) p = fmaf(qr[g][e], kk[e], p);
        p = warp_sum(p) * scale_log2 + bias;
        const float mn = fmaxf(m[g], p);
        const float a = exp2f(m[g] - mn);
        const float pe = exp2f(p - mn);
        l[g] = l[g] * a + pe;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] = fmaf(acc[g][e], a, pe * vv[e]);
        m[g] = mn;
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float out[E];
    const float inv = 1.f / l[g];
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = acc[g][e] * inv;
    store_vec<T, E>(o + ((size_t)tg * Hq + kv * G + g) * D + lane * E, out);
    if (lane == 0) lse[(size_t)tg * Hq + kv * G + g] = (m[g] + log2f(l[g])) * kLn2;
  }
}

// ---------------------------------------------------------------------------------------
// backward, pass 0: Drow[t, hq] = dO . O
// ---------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void attn_bwd_rowdot_kernel(const T* __restrict__ o, const T* __restrict__ dout, int rows,
                                       float* __restrict__ drow) {
  constexpr int E = D / 32;
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float a[E], b[E];
  load_vec<T, E>(o + (size_t)row * D + lane * E, a);
  load_vec<T, E>(dout + (size_t)row * D + lane * E, b);
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) s = fmaf(a[e], b[e], s);
  s = warp_sum(s);
  if (lane == 0) drow[row] = s;
}

// ---------------------------------------------------------------------------------------
// backward, pass 1 (query-major): dQ and dlogg of one (token, kv) row.
// dS = P (dP - D); dQ = scale * sum_i dS_i k_i; dlogg[slot] = sum over heads and the
// slot's keys of dS.
// ---------------------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void __launch_bounds__(128) attn_bwd_dq_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ drow,
    const int32_t* __restrict__ idx, const float* __restrict__ logg, const int32_t* __restrict__ cu,
    int batch, int T_total, int Hkv, int R, int B, int K, float scale, T* __restrict__ dq,
    float* __restrict__ dlogg) {
  constexpr int E = D / 32;
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T_total * Hkv) return;
  const int tg = row / Hkv, kv = row - tg * Hkv;   // kv: gate head; its K/V head is kv / R
  const int b = seq_of(cu, batch, tg);
  const int s0 = cu[b], t = tg - s0;
  const int Hq = Hkv * G;
  const int Hk = Hkv / R, kh = kv / R;
  const float scale_log2 = scale * kLog2e;
  float qr[G][E], dor[G][E], acc[G][E], l2[G], dd[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const size_t r = (size_t)tg * Hq + kv * G + g;
    load_vec<T, E>(q + r * D + lane * E, qr[g]);
    load_vec<T, E>(dout + r * D + lane * E, dor[g]);
    l2[g] = lse[r] * kLog2e;
    dd[g] = drow[r];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[g][e] = 0.f;
  }
  const int32_t* ir = idx + (size_t)row * (K + 1);
  const float* gr = logg + (size_t)row * (K + 1);
  float* dl = dlogg + (size_t)row * (K + 1);
  for (int s = 0; s <= K; ++s) {
    const int j = ir[s];
    if (j < 0) {
      if (lane == 0) dl[s] = 0.f;
      continue;
    }
    const float bias = gr[s] * kLog2e;
    const int i0 = j * B, i1 = min(i0 + B, t + 1);
    float dsum = 0.f;
    for (int i = i0; i < i1; ++i) {
      float kk[E], vv[E];
      const size_t off = ((size_t)(s0 + i) * Hk + kh) * D + lane * E;
      load_vec<T, E>(k + off, kk);
      load_vec<T, E>(v + off, vv);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float sc = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          sc = fmaf(qr[g][e], kk[e], sc);
          dp = fmaf(dor[g][e], vv[e], dp);
        }
        sc = warp_sum(sc);
        dp = warp_sum(dp);
        const float p = exp2f(sc * scale_log2 + bias - l2[g]);
        const float ds = p * (dp - dd[g]);
        dsum += ds;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[g][e] = fmaf(ds, kk[e], acc[g][e]);
      }
    }
    if (lane == 0) dl[s] = dsum;
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float out[E];
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = acc[g][e] * scale;
    store_vec<T, E>(dq + ((size_t)tg * Hq + kv * G + g) * D + lane * E, out);
  }
}

// ---------------------------------------------------------------------------------------
// backward, pass 2 (key-major): dK, dV of one KV block. The CTA scans the rows of its
// sequence (in token order, so the sums are deterministic) for the ones that selected
// this block, then each warp accumulates dK/dV of its own keys over those rows.
// ---------------------------------------------------------------------------------------
constexpr int kDkvThreads = 256;
constexpr int kDkvWarps = kDkvThreads / 32;
constexpr int kDkvChunk = 256;   // tokens scanned per round

template <typename T, int D, int G, int KPW>
__global__ void __launch_bounds__(kDkvThreads) attn_bwd_dkdv_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ drow,
    const int32_t* __restrict__ idx, const float* __restrict__ logg, const int32_t* __restrict__ cu,
    int Hkv, int R, int B, int K, float scale, T* __restrict__ dk, T* __restrict__ dv) {
  // Hkv here counts gate heads; the CTA's KV head kh is read by gate heads kh*R .. kh*R+R-1
  constexpr int E = D / 32;
  __shared__ int list_t[kDkvChunk];
  __shared__ int list_s[kDkvChunk];
  __shared__ int warp_cnt[kDkvWarps];
  __shared__ int n_list;
  const int j = blockIdx.x, b = blockIdx.y, kh = blockIdx.z;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int i0 = j * B;
  if (i0 >= L) return;
  const int nkeys = min(B, L - i0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = Hkv * G;
  const int Hk = Hkv / R;
  const float scale_log2 = scale * kLog2e;

  // this warp's keys: local key index kk = warp + r * kDkvWarps
  float kr[KPW][E], vr[KPW][E], dkr[KPW][E], dvr[KPW][E];
#pragma unroll
  for (int r = 0; r < KPW; ++r) {
    const int kl = warp + r * kDkvWarps;
#pragma unroll
    for (int e = 0; e < E; ++e) { kr[r][e] = vr[r][e] = dkr[r][e] = dvr[r][e] = 0.f; }
    if (kl < nkeys) {
      const size_t off = ((size_t)(s0 + i0 + kl) * Hk + kh) * D + lane * E;
      load_vec<T, E>(k + off, kr[r]);
      load_vec<T, E>(v + off, vr[r]);
    }
  }

  for (int kv = kh * R; kv < kh * R + R; ++kv)   // the gate heads reading this KV head
  for (int c0 = i0; c0 < L; c0 += kDkvChunk) {
    // ---- ordered compaction of the rows in [c0, c0 + chunk) that selected block j ----
    const int t = c0 + threadIdx.x;
    int slot = -1;
    if (t < L) {
      const int32_t* ir = idx + ((size_t)(s0 + t) * Hkv + kv) * (K + 1);
      for (int s = 0; s <= K; ++s) {
        const int jj = ir[s];
        if (jj == j) { slot = s; break; }
        if (jj < 0 || jj > j) break;   // ascending: block j cannot follow
      }
    }
    const unsigned m = __ballot_sync(0xffffffffu, slot >= 0);
    if (lane == 0) warp_cnt[warp] = __popc(m);
    __syncthreads();
    if (threadIdx.x == 0) {
      int run = 0;
      for (int w = 0; w < kDkvWarps; ++w) { const int c = warp_cnt[w]; warp_cnt[w] = run; run += c; }
      n_list = run;
    }
    __syncthreads();
    if (slot >= 0) {
      const int pos = warp_cnt[warp] + __popc(m & ((1u << lane) - 1u));
      list_t[pos] = t;
      list_s[pos] = slot;
    }
    __syncthreads();
    const int n = n_list;
    // ---- accumulate ----
    for (int u = 0; u < n; ++u) {
      const int tt = list_t[u];
      const size_t rrow = (size_t)(s0 + tt) * Hkv + kv;
      const float bias = logg[rrow * (K + 1) + list_s[u]] * kLog2e;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const size_t qrow = (size_t)(s0 + tt) * Hq + kv * G + g;
        float qg[E], dg[E];
        load_vec<T, E>(q + qrow * D + lane * E, qg);
        load_vec<T, E>(dout + qrow * D + lane * E, dg);
        const float l2 = lse[qrow] * kLog2e;
        const float dd = drow[qrow];
#pragma unroll
        for (int r = 0; r < KPW; ++r) {
          const int kl = warp + r * kDkvWarps;
          if (kl >= nkeys || i0 + kl > tt) continue;   // warp-uniform
          float sc = 0.f, dp = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            sc = fmaf(qg[e], kr[r][e], sc);
            dp = fmaf(dg[e], vr[r][e], dp);
          }
          sc = warp_sum(sc);
          dp = warp_sum(dp);
          const float p = exp2f(sc * scale_log2 + bias - l2);
          const float ds = p * (dp - dd);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            dkr[r][e] = fmaf(ds, qg[e], dkr[r][e]);
            dvr[r][e] = fmaf(p, dg[e], dvr[r][e]);
          }
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < KPW; ++r) {
    const int kl = warp + r * kDkvWarps;
    if (kl >= nkeys) continue;
    const size_t off = ((size_t)(s0 + i0 + kl) * Hk + kh) * D + lane * E;
    float a[E];
#pragma unroll
    for (int e = 0; e < E; ++e) a[e] = dkr[r][e] * scale;
    store_vec<T, E>(dk + off, a);
    store_vec<T, E>(dv + off, dvr[r]);
  }
}

// ---------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------
template <typename T, int D, int G>
static void fwd_simt_launch(const sas_problem& p, const void* q, const void* k, const void* v,
                            const int32_t* idx, const float* logg, void* o, float* lse,
                            cudaStream_t st) {
  const int Hs = gate_heads(p), R = Hs / p.num_kv_heads;
  const int rows = p.total_tokens * Hs;
  const int grid = (int)(((size_t)rows * 32 + 127) / 128);
  const float scale_log2 = kLog2e / sqrtf((float)D);
  attn_fwd_simt_kernel<T, D, G><<<grid, 128, 0, st>>>(
      (const T*)q, (const T*)k, (const T*)v, idx, logg, p.cu_seqlens, p.batch, p.total_tokens,
      Hs, R, p.block, p.topk, scale_log2, (T*)o, lse);
}

template <typename T, int D, int G>
static void bwd_simt_launch(const sas_problem& p, const void* q, const void* k, const void* v,
                            const void* o, const void* dout, const float* lse, const int32_t* idx,
                            const float* logg, void* dq, void* dk, void* dv, float* dlogg,
                            float* drow, cudaStream_t st) {
  const int rows_q = p.total_tokens * p.num_q_heads;
  attn_bwd_rowdot_kernel<T, D><<<(int)(((size_t)rows_q * 32 + 255) / 256), 256, 0, st>>>(
      (const T*)o, (const T*)dout, rows_q, drow);
  const int Hs = gate_heads(p), R = Hs / p.num_kv_heads;
  const int rows = p.total_tokens * Hs;
  const float scale = 1.0f / sqrtf((float)D);
  attn_bwd_dq_simt_kernel<T, D, G><<<(int)(((size_t)rows * 32 + 127) / 128), 128, 0, st>>>(
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, drow, idx, logg, p.cu_seqlens,
      p.batch, p.total_tokens, Hs, R, p.block, p.topk, scale, (T*)dq, dlogg);
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  dim3 grid(NBmax, p.batch, p.num_kv_heads);
#define SAS_DKV(KPW)                                                                          \
  attn_bwd_dkdv_simt_kernel<T, D, G, KPW><<<grid, kDkvThreads, 0, st>>>(                       \
      (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, drow, idx, logg,              \
      p.cu_seqlens, Hs, R, p.block, p.topk, scale, (T*)dk, (T*)dv)
  if (p.block <= 16) SAS_DKV(2);
  else if (p.block <= 32) SAS_DKV(4);
  else if (p.block <= 64) SAS_DKV(8);
  else SAS_DKV(16);
#undef SAS_DKV
}

#define SAS_FOR_G(MACRO, T, D)           \
  switch (p.num_q_heads / gate_heads(p)) { \
    case 1: MACRO(T, D, 1); break;       \
    case 2: MACRO(T, D, 2); break;       \
    case 4: MACRO(T, D, 4); break;       \
    case 5: MACRO(T, D, 5); break;       \
    default: MACRO(T, D, 8); break;      \
  }

sas_status launch_rowdot(const sas_problem& p, const void* o, const void* dout, float* drow,
                         cudaStream_t st) {
  const int rows_q = p.total_tokens * p.num_q_heads;
  const int grid = (int)(((size_t)rows_q * 32 + 255) / 256);
#define SAS_RD(T, D) attn_bwd_rowdot_kernel<T, D><<<grid, 256, 0, st>>>((const T*)o, (const T*)dout, rows_q, drow)
  if (p.dtype == SAS_BF16) {
    if (p.head_dim == 64) SAS_RD(__nv_bfloat16, 64); else SAS_RD(__nv_bfloat16, 128);
  } else {
    if (p.head_dim == 64) SAS_RD(float, 64); else SAS_RD(float, 128);
  }
#undef SAS_RD
  return launch_status("attn_bwd row dot", 1);
}

sas_status launch_attn_fwd_simt(const sas_problem& p, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* logg, void* o, float* lse,
                                cudaStream_t st) {
#define SAS_F(T, D, G) fwd_simt_launch<T, D, G>(p, q, k, v, idx, logg, o, lse, st)
  if (p.dtype == SAS_BF16) {
    if (p.head_dim == 64) { SAS_FOR_G(SAS_F, __nv_bfloat16, 64) } else { SAS_FOR_G(SAS_F, __nv_bfloat16, 128) }
  } else {
    if (p.head_dim == 64) { SAS_FOR_G(SAS_F, float, 64) } else { SAS_FOR_G(SAS_F, float, 128) }
  }
#undef SAS_F
  return launch_status("attn_fwd (cuda cores)", 1);
}

sas_status launch_attn_bwd_simt(const sas_problem& p, const void* q, const void* k, const void* v,
                                const void* o, const void* dout, const float* lse,
                                const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                                float* dlogg, float* drow, cudaStream_t st) {
#define SAS_B(T, D, G) \
  bwd_simt_launch<T, D, G>(p, q, k, v, o, dout, lse, idx, logg, dq, dk, dv, dlogg, drow, st)
  if (p.dtype == SAS_BF16) {
    if (p.head_dim == 64) { SAS_FOR_G(SAS_B, __nv_bfloat16, 64) } else { SAS_FOR_G(SAS_B, __nv_bfloat16, 128) }
  } else {
    if (p.head_dim == 64) { SAS_FOR_G(SAS_B, float, 64) } else { SAS_FOR_G(SAS_B, float, 128) }
  }
#undef SAS_B
  return launch_status("attn_bwd (cuda cores)", 3);
}

}  // namespace sas
