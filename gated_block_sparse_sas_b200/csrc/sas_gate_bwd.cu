// Router backward: gradients of the gate parameters (Wq, Wk and the two RMSNorm weights)
// through the log-gates of the kept blocks, with the selection held fixed. The project
// README (intro item (b)) and the paper abstract make the selector trainable end to end
// from the language-model loss; this is that gradient for one layer's gate.
//
// Forward being differentiated (per token t, kv head; h = 128):
//   xq_t = Wq . concat_g q_nope[t, kv*G+g],  q~_t = rope_t(RMSNorm(xq_t) * qnorm_w)
//   xk_j = Wk . P_j (pooled block j),        k~_j = rope_{jB}(RMSNorm(xk_j) * knorm_w)
//   xc_t = Wk . P_cur(t) (block c_t's prefix up to t), k~c_t = rope_{c_t B}(...)
//   s[t, j] = q~_t . k~_j / sqrt(h),  log g = s - logsumexp over visible blocks
// Given dlogg[t, kv, slot]: dL/ds[t, j] = dlogg on the kept slots. The logsumexp term
// (- softmax_j * sum of the row's dlogg) is zero: the attention is unchanged when every
// log-gate of a row moves by one constant, so the row sums of the dlogg it returns are zero.
//
// Passes (fp32 throughout; h = 128, bf16 inputs):
//   0. xq, xc for every (t, kv): the tensor-core projections of the forward gate.
//   1. block keys: xk_j and k~_j per (sequence, block, kv), one warp per row.
//   2. rows: per (t, kv) one warp: q~, k~c; dq~ = sum_slots ds k~_j; dk~_j += ds q~ (L2
//      reductions into a per-block buffer); dk~c = ds_c q~; both back through the rotary and
//      the RMSNorm -> dxq, dxc and the norm-weight gradients.
//   3. block keys backward: dk~_j -> dxk_j and the knorm_w gradient.
//   4. weight gradients as sums of outer products over rows, register-tiled 64 x 64 tiles:
//      dWq += dxq (x) q_nope group, dWk += dxk (x) P_j + dxc (x) P_cur(t) (the prefix pools
//      rebuilt per block by a running max / min / sum).
#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using sm100::red_add_v4;

namespace gbw {
constexpr int H = 128;           // gate hidden of the supported configuration
constexpr int kRowThreads = 256;
constexpr int kTile = 64;        // outer-product tile (rows of W x columns of W)
constexpr int kKs = 16;          // rows per step of the outer-product kernel
}  // namespace gbw

// One row of h = 128 values per warp: lane holds e = lane + 32 u (u = 0..3); the rotary
// pairs (e, e + 64) are (u = 0, 2) and (u = 1, 3) of the same lane.
__device__ __forceinline__ void gbw_norm_rope_fwd(const float x[4], const float* __restrict__ w,
                                                  const float* __restrict__ rc,
                                                  const float* __restrict__ rs, int pos, float eps,
                                                  int lane, float out[4], float u[4], float& r) {
  float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
  ss = warp_sum(ss);
  r = sqrtf(ss / (float)gbw::H + eps);
#pragma unroll
  for (int k = 0; k < 4; ++k) u[k] = x[k] / r;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int e = lane + 32 * p;
    const float a = u[p] * w[e], b = u[p + 2] * w[e + 64];
    const float c = rc[(size_t)pos * 64 + e], s = rs[(size_t)pos * 64 + e];
    out[p] = a * c - b * s;
    out[p + 2] = b * c + a * s;
  }
}

// Backward of gbw_norm_rope_fwd: dout = dL/d(rotated output) -> dx; dw += dL/dw.
__device__ __forceinline__ void gbw_norm_rope_bwd(const float x[4], const float u[4], float r,
                                                  const float* __restrict__ w,
                                                  const float* __restrict__ rc,
                                                  const float* __restrict__ rs, int pos, int lane,
                                                  const float dout[4], float dx[4], float dw[4]) {
  float dy[4];
#pragma unroll
  for (int p = 0; p < 2; ++p) {   // the rotation's transpose: rotation by -angle
    const int e = lane + 32 * p;
    const float c = rc[(size_t)pos * 64 + e], s = rs[(size_t)pos * 64 + e];
    dy[p] = dout[p] * c + dout[p + 2] * s;
    dy[p + 2] = dout[p + 2] * c - dout[p] * s;
  }
  float du[4], dot = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float wk = w[lane + 32 * k];
    dw[k] += dy[k] * u[k];
    du[k] = dy[k] * wk;
    dot += du[k] * x[k];
  }
  dot = warp_sum(dot);
  const float r3 = r * r * r * (float)gbw::H;
#pragma unroll
  for (int k = 0; k < 4; ++k) dx[k] = du[k] / r - x[k] * dot / r3;
}

// The same two steps with lane holding 4 consecutive values e = 4 lane + k (so a row moves
// as one 16-byte vector per lane); the rotary partner of e (e +- 64) sits in lane ^ 16.
__device__ __forceinline__ void gbw_norm_rope_fwd_v(const float x[4], const float* __restrict__ w,
                                                    const float* __restrict__ rc,
                                                    const float* __restrict__ rs, int pos,
                                                    float eps, int lane, float out[4], float u[4],
                                                    float& r) {
  float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
  ss = warp_sum(ss);
  r = sqrtf(ss / (float)gbw::H + eps);
  const bool lo = lane < 16;
  const int e0 = 4 * lane, t0 = lo ? e0 : e0 - 64;   // rotary table index of e0
  float y[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    u[k] = x[k] / r;
    y[k] = u[k] * w[e0 + k];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float yp = __shfl_xor_sync(0xffffffffu, y[k], 16);
    const float c = rc[(size_t)pos * 64 + t0 + k], s = rs[(size_t)pos * 64 + t0 + k];
    out[k] = lo ? y[k] * c - yp * s : y[k] * c + yp * s;
  }
}

__device__ __forceinline__ void gbw_norm_rope_bwd_v(const float x[4], const float u[4], float r,
                                                    const float* __restrict__ w,
                                                    const float* __restrict__ rc,
                                                    const float* __restrict__ rs, int pos,
                                                    int lane, const float dout[4], float dx[4],
                                                    float dw[4]) {
  const bool lo = lane < 16;
  const int e0 = 4 * lane, t0 = lo ? e0 : e0 - 64;
  float du[4], dot = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {   // the rotation's transpose: rotation by -angle
    const float dp = __shfl_xor_sync(0xffffffffu, dout[k], 16);
    const float c = rc[(size_t)pos * 64 + t0 + k], s = rs[(size_t)pos * 64 + t0 + k];
    const float dy = lo ? dout[k] * c + dp * s : dout[k] * c - dp * s;
    dw[k] += dy * u[k];
    du[k] = dy * w[e0 + k];
    dot += du[k] * x[k];
  }
  dot = warp_sum(dot);
  const float r3 = r * r * r * (float)gbw::H;
#pragma unroll
  for (int k = 0; k < 4; ++k) dx[k] = du[k] / r - x[k] * dot / r3;
}

// Sum the CTA's per-lane norm-weight gradients (4 per lane and warp) into dw[128].
__device__ __forceinline__ void gbw_cta_add_dw(const float acc[4], float* red, float* __restrict__ dw,
                                               bool vec_layout) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k)
    red[warp * gbw::H + (vec_layout ? 4 * lane + k : lane + 32 * k)] = acc[k];
  __syncthreads();
  for (int e = threadIdx.x; e < gbw::H; e += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += red[w * gbw::H + e];
    atomicAdd(dw + e, s);
  }
}

// (1) block keys: xk = Wk . P_j and k~_j, one warp per (sequence, block, kv); zeros past a
// sequence's end.
__global__ void __launch_bounds__(gbw::kRowThreads) gbw_block_fwd_kernel(
    const float* __restrict__ pooled, const __nv_bfloat16* __restrict__ wk,
    const float* __restrict__ knorm_w, const int32_t* __restrict__ cu, const float* __restrict__ rc,
    const float* __restrict__ rs, int batch, int NBmax, int Hkv, int d, int B, float eps,
    float* __restrict__ xk_out, float* __restrict__ kt_out) {
  const int lane = threadIdx.x & 31;
  const int C = 3 * d;   // <= 384: 12 inputs per lane
  const size_t nrows = (size_t)batch * NBmax * Hkv;
  for (size_t row = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; row < nrows;
       row += (gridDim.x * (size_t)blockDim.x) >> 5) {
    const int kv = (int)(row % Hkv);
    const size_t bj = row / Hkv;
    const int b = (int)(bj / NBmax), j = (int)(bj % NBmax);
    const int L = cu[b + 1] - cu[b];
    float* xo = xk_out + row * gbw::H;
    float* ko = kt_out + row * gbw::H;
    if (j * B >= L) {
#pragma unroll
      for (int k = 0; k < 4; ++k) xo[lane + 32 * k] = ko[lane + 32 * k] = 0.f;
      continue;
    }
    float pv[12];
    const float* P = pooled + row * C;
#pragma unroll
    for (int m = 0; m < 12; ++m) pv[m] = (lane + 32 * m < C) ? P[lane + 32 * m] : 0.f;
    const __nv_bfloat16* W = wk + (size_t)kv * gbw::H * C;
    float x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[u] = 0.f;
#pragma unroll 1
      for (int ii = 0; ii < 32; ++ii) {
        const __nv_bfloat16* wr = W + (size_t)(32 * u + ii) * C;
        float part = 0.f;
#pragma unroll
        for (int m = 0; m < 12; ++m)
          if (lane + 32 * m < C) part = fmaf(__bfloat162float(wr[lane + 32 * m]), pv[m], part);
        part = warp_sum(part);
        if (lane == ii) x[u] = part;
      }
    }
    float out[4], uu[4], r;
    gbw_norm_rope_fwd(x, knorm_w, rc, rs, j * B, eps, lane, out, uu, r);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      xo[lane + 32 * k] = x[k];
      ko[lane + 32 * k] = out[k];
    }
  }
}

// (2) rows: one warp per (token, kv head).
__global__ void __launch_bounds__(gbw::kRowThreads) gbw_row_kernel(
    const float* __restrict__ xq_all, const float* __restrict__ xc_all,
    const float* __restrict__ kt_hist, const int32_t* __restrict__ idx,
    const float* __restrict__ dlogg, const float* __restrict__ qnorm_w,
    const float* __restrict__ knorm_w, const int32_t* __restrict__ cu, const float* __restrict__ rc,
    const float* __restrict__ rs, int batch, int T, int NBmax, int Hkv, int B, int K1, float eps,
    float* __restrict__ dkt_hist, float* __restrict__ dxq_out, float* __restrict__ dxc_out,
    float* __restrict__ dqnorm_w, float* __restrict__ dknorm_w) {
  __shared__ float red[(gbw::kRowThreads / 32) * gbw::H];
  const int lane = threadIdx.x & 31;
  const float inv_sqrt_h = 1.f / sqrtf((float)gbw::H);
  float dwq[4] = {0.f, 0.f, 0.f, 0.f}, dwk[4] = {0.f, 0.f, 0.f, 0.f};
  const size_t nrows = (size_t)T * Hkv;
  for (size_t row = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; row < nrows;
       row += (gridDim.x * (size_t)blockDim.x) >> 5) {
    const int tg = (int)(row / Hkv), kv = (int)(row % Hkv);
    const int b = seq_of(cu, batch, tg);
    const int t = tg - cu[b], c = t / B;
    // lane holds e = 4 lane .. 4 lane + 3 of every row (16-byte vectors)
    const float4 xq4 = reinterpret_cast<const float4*>(xq_all + row * gbw::H)[lane];
    const float4 xc4 = reinterpret_cast<const float4*>(xc_all + row * gbw::H)[lane];
    const float xq[4] = {xq4.x, xq4.y, xq4.z, xq4.w}, xc[4] = {xc4.x, xc4.y, xc4.z, xc4.w};
    float qt[4], uq[4], rq, kc[4], uc[4], rcn;
    gbw_norm_rope_fwd_v(xq, qnorm_w, rc, rs, t, eps, lane, qt, uq, rq);
    gbw_norm_rope_fwd_v(xc, knorm_w, rc, rs, c * B, eps, lane, kc, uc, rcn);
    float dqt[4] = {0.f, 0.f, 0.f, 0.f}, dkc[4] = {0.f, 0.f, 0.f, 0.f};
    // slots 32 at a time: lane l reads slot base + l once; the kept keys of 4 slots are
    // loaded together before their arithmetic
    const size_t krow = (size_t)b * NBmax;
    for (int base = 0; base < K1; base += 32) {
      const int my = base + lane;
      const int jl = my < K1 ? idx[row * K1 + my] : -1;
      const float dsl = my < K1 ? dlogg[row * K1 + my] * inv_sqrt_h : 0.f;
      const int ns = min(32, K1 - base);
      for (int s0 = 0; s0 < ns; s0 += 4) {
        int jj[4];
        float dd[4];
        float4 kj[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          jj[u] = __shfl_sync(0xffffffffu, jl, (s0 + u) & 31);
          dd[u] = __shfl_sync(0xffffffffu, dsl, (s0 + u) & 31);
          if (s0 + u >= ns) jj[u] = -1;
          kj[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (jj[u] >= 0 && jj[u] != c)
            kj[u] = reinterpret_cast<const float4*>(
                kt_hist + ((krow + jj[u]) * Hkv + kv) * gbw::H)[lane];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {   // warp-uniform branches: every lane holds slot u
          if (jj[u] < 0) continue;
          const float ds = dd[u];
          if (jj[u] == c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              dqt[k] = fmaf(ds, kc[k], dqt[k]);
              dkc[k] = fmaf(ds, qt[k], dkc[k]);
            }
          } else {
            dqt[0] = fmaf(ds, kj[u].x, dqt[0]);
            dqt[1] = fmaf(ds, kj[u].y, dqt[1]);
            dqt[2] = fmaf(ds, kj[u].z, dqt[2]);
            dqt[3] = fmaf(ds, kj[u].w, dqt[3]);
            red_add_v4(dkt_hist + ((krow + jj[u]) * Hkv + kv) * gbw::H + 4 * lane,
                       make_float4(ds * qt[0], ds * qt[1], ds * qt[2], ds * qt[3]));
          }
        }
      }
    }
    float dx[4];
    gbw_norm_rope_bwd_v(xq, uq, rq, qnorm_w, rc, rs, t, lane, dqt, dx, dwq);
    reinterpret_cast<float4*>(dxq_out + row * gbw::H)[lane] = make_float4(dx[0], dx[1], dx[2], dx[3]);
    gbw_norm_rope_bwd_v(xc, uc, rcn, knorm_w, rc, rs, c * B, lane, dkc, dx, dwk);
    reinterpret_cast<float4*>(dxc_out + row * gbw::H)[lane] = make_float4(dx[0], dx[1], dx[2], dx[3]);
  }
  gbw_cta_add_dw(dwq, red, dqnorm_w, true);
  gbw_cta_add_dw(dwk, red, dknorm_w, true);
}

// (3) block keys backward: dk~_j -> dxk_j, knorm_w gradient.
__global__ void __launch_bounds__(gbw::kRowThreads) gbw_block_bwd_kernel(
    const float* __restrict__ xk_hist, const float* __restrict__ dkt_hist,
    const float* __restrict__ knorm_w, const int32_t* __restrict__ cu, const float* __restrict__ rc,
    const float* __restrict__ rs, int batch, int NBmax, int Hkv, int B, float eps,
    float* __restrict__ dxk_out, float* __restrict__ dknorm_w) {
  __shared__ float red[(gbw::kRowThreads / 32) * gbw::H];
  const int lane = threadIdx.x & 31;
  float dwk[4] = {0.f, 0.f, 0.f, 0.f};
  const size_t nrows = (size_t)batch * NBmax * Hkv;
  for (size_t row = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; row < nrows;
       row += (gridDim.x * (size_t)blockDim.x) >> 5) {
    const size_t bj = row / Hkv;
    const int b = (int)(bj / NBmax), j = (int)(bj % NBmax);
    float* xo = dxk_out + row * gbw::H;
    if (j * B >= cu[b + 1] - cu[b]) {
#pragma unroll
      for (int k = 0; k < 4; ++k) xo[lane + 32 * k] = 0.f;
      continue;
    }
    float x[4], g[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[k] = xk_hist[row * gbw::H + lane + 32 * k];
      g[k] = dkt_hist[row * gbw::H + lane + 32 * k];
    }
    float out[4], u[4], r, dx[4];
    gbw_norm_rope_fwd(x, knorm_w, rc, rs, j * B, eps, lane, out, u, r);
    gbw_norm_rope_bwd(x, u, r, knorm_w, rc, rs, j * B, lane, g, dx, dwk);
#pragma unroll
    for (int k = 0; k < 4; ++k) xo[lane + 32 * k] = dx[k];
  }
  gbw_cta_add_dw(dwk, red, dknorm_w, false);
}

// (4) dW[kv][i][c] += sum over rows of X[row][kv][i] * Y[row][kv][c], a 64 x 64 tile of dW per
// CTA (64 threads, 8 x 8 outputs each), rows split over gridDim.z / Hkv chunks, the partial
// tile added with fp32 atomics.
//   MODE 0: rows = tokens, X = dxq, Y = q_nope[t, kv*G .. kv*G+G-1, :] (C = G d)
//   MODE 1: rows = (sequence, block), X = dxk, Y = pooled (C = 3d)
//   MODE 2: rows = tokens taken block by block, X = dxc, Y = the block's prefix pool up to
//           the token (running max | min | sum / count, C = 3d)
template <int MODE>
__global__ void __launch_bounds__(64) gbw_outer_kernel(
    const float* __restrict__ X, const __nv_bfloat16* __restrict__ q_nope,
    const float* __restrict__ pooled, const __nv_bfloat16* __restrict__ k_nope,
    const int32_t* __restrict__ cu, int batch, int T, int Hq, int Hkv, int d, int B, int NBmax,
    int C, int nsplit, float* __restrict__ dW) {
  __shared__ float Xs[gbw::kKs][gbw::kTile];
  __shared__ float Ys[gbw::kKs][gbw::kTile];
  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  const int c0 = blockIdx.x * gbw::kTile, i0 = blockIdx.y * gbw::kTile;
  const int kv = blockIdx.z % Hkv, split = blockIdx.z / Hkv;
  const int G = Hq / Hkv;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) acc[a][bb] = 0.f;

  auto fma_step = [&](int nk) {
    __syncthreads();
    for (int k = 0; k < nk; ++k) {
      float xv[8], yv[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) xv[a] = Xs[k][ty + 8 * a];
#pragma unroll
      for (int bb = 0; bb < 8; ++bb) yv[bb] = Ys[k][tx + 8 * bb];
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int bb = 0; bb < 8; ++bb) acc[a][bb] = fmaf(xv[a], yv[bb], acc[a][bb]);
    }
    __syncthreads();
  };

  if constexpr (MODE == 0 || MODE == 1) {
    const int nrows = MODE == 0 ? T : batch * NBmax;
    const int per = (nrows + nsplit - 1) / nsplit;
    const int r0 = split * per, r1 = min(nrows, r0 + per);
    // the next step's 16 x 64 tiles are loaded into registers while this step computes
    constexpr int kPer = gbw::kKs * gbw::kTile / 64;   // elements of each tile per thread
    float xr[kPer], yr[kPer];
    auto load = [&](int rb) {
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        const int e = tid + 64 * q, k = e / gbw::kTile, col = e % gbw::kTile;
        const int r = rb + k;
        xr[q] = 0.f;
        yr[q] = 0.f;
        if (r < r1) {
          xr[q] = X[((size_t)r * Hkv + kv) * gbw::H + i0 + col];
          if constexpr (MODE == 0)
            yr[q] = __bfloat162float(q_nope[((size_t)r * Hq + (size_t)kv * G) * d + c0 + col]);
          else
            yr[q] = pooled[((size_t)r * Hkv + kv) * C + c0 + col];
        }
      }
    };
    if (r0 < r1) load(r0);
    for (int rb = r0; rb < r1; rb += gbw::kKs) {
      const int nk = min(gbw::kKs, r1 - rb);
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        const int e = tid + 64 * q;
        Xs[e / gbw::kTile][e % gbw::kTile] = xr[q];
        Ys[e / gbw::kTile][e % gbw::kTile] = yr[q];
      }
      if (rb + gbw::kKs < r1) load(rb + gbw::kKs);
      fma_step(nk);
    }
  } else {
    const int nblk = batch * NBmax;
    const int per = (nblk + nsplit - 1) / nsplit;
    const int q0 = split * per, q1 = min(nblk, q0 + per);
    // column owned by this thread in the prefix scan: c0 + tid -> (part, channel)
    const int col = c0 + tid, part = col / d, ch = col - part * d;
    for (int bj = q0; bj < q1; ++bj) {
      const int b = bj / NBmax, j = bj % NBmax;
      const int s0 = cu[b], L = cu[b + 1] - s0;
      if (j * B >= L) continue;   // uniform over the CTA
      const int n = min(B, L - j * B);
      float run = 0.f;
      for (int rb = 0; rb < n; rb += gbw::kKs) {
        const int nk = min(gbw::kKs, n - rb);
        float kvv[gbw::kKs];
#pragma unroll
        for (int k = 0; k < gbw::kKs; ++k)
          kvv[k] = k < nk ? __bfloat162float(
                                k_nope[((size_t)(s0 + j * B + rb + k) * Hkv + kv) * d + ch])
                          : 0.f;
#pragma unroll
        for (int k = 0; k < gbw::kKs; ++k) {
          if (k < nk) {
            const int cnt = rb + k + 1;
            const float v = kvv[k];
            if (cnt == 1) run = v;
            else if (part == 0) run = fmaxf(run, v);
            else if (part == 1) run = fminf(run, v);
            else run += v;
            Ys[k][tid] = part == 2 ? run / (float)cnt : run;
          } else {
            Ys[k][tid] = 0.f;
          }
        }
        for (int e = tid; e < gbw::kKs * gbw::kTile; e += 64) {
          const int k = e / gbw::kTile, cc = e % gbw::kTile;
          Xs[k][cc] = k < nk ? X[((size_t)(s0 + j * B + rb + k) * Hkv + kv) * gbw::H + i0 + cc] : 0.f;
        }
        fma_step(nk);
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int bb = 0; bb < 8; ++bb)
      atomicAdd(dW + ((size_t)kv * gbw::H + i0 + ty + 8 * a) * C + c0 + tx + 8 * bb, acc[a][bb]);
}

// ---------------------------------------------------------------------------------------
// (4') the two token-row outer products on the tensor cores. dW[kv] (+)= X^T Y summed over
// the token rows t, with X = dx[t, kv, :] (fp32, split into bf16 hi + lo parts: their sum
// carries 16 significant bits, so the products keep fp32-like accuracy) and Y the projection's
// bf16 input row (the G query heads for dWq; the prefix pools [max | min | mean hi | mid | lo]
// of the forward's tensor-core gate for dWk, whose three mean parts add into the same mean
// columns of dWk). CTA = (128 columns of W, kv head, split of the rows), 128 threads:
// warp 0 lane 0 loads 64-row chunks of X hi, X lo and Y by TMA into a 4-stage ring, warp 1
// lane 0 issues two MMAs per 16 rows (M = 128 W rows, N = 128 W columns; both operands
// MN-major: the rows of the chunk are the reduction dimension) into a TMEM accumulator, and
// all four warps add the 128 x 128 fp32 result into dW with vector atomics.
// ---------------------------------------------------------------------------------------
namespace gwt {
constexpr int kM = 128, kN = 128, kK = 64;   // W rows, W columns, token rows per stage
constexpr int kStages = 4;
constexpr int kBox = kK * 128;               // [64 rows][64 bf16]: 8 KB, 128B-swizzled
constexpr int kStage = 6 * kBox;             // X hi (2 halves), X lo (2 halves), Y (2 halves)
constexpr int kThreads = 128;
constexpr int OFF_BAR = kStages * kStage;
constexpr int OFF_MISC = OFF_BAR + (2 * kStages + 1) * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
}  // namespace gwt

struct WgradArgs {
  int T;             // token rows
  int rows_per;      // rows per split (a multiple of gwt::kK)
  int y_col0;        // Y column of W column 0 for kv head 0
  int y_col_kv;      // Y columns between kv heads
  float* dW;         // [Hkv][128][C]
  int C;             // W columns
  int mean_cols;     // > 0: W columns >= 2 * mean_cols fold onto [2 mean_cols, 3 mean_cols)
  int* err;
};

__global__ void __launch_bounds__(gwt::kThreads)
    gbw_wgrad_tc_kernel(const __grid_constant__ CUtensorMap tXh, const __grid_constant__ CUtensorMap tXl,
                        const __grid_constant__ CUtensorMap tY, const WgradArgs a) {
  using namespace gwt;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kN, kv = blockIdx.y, split = blockIdx.z;
  const int r0 = split * a.rows_per, r1 = min(a.T, r0 + a.rows_per);
  const int nk = r1 > r0 ? (r1 - r0 + kK - 1) / kK : 0;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {   // TMA producer: X hi, X lo (W rows 0-63, 64-127), Y (2 halves)
    prefetch_tmap(&tXh);
    prefetch_tmap(&tXl);
    prefetch_tmap(&tY);
    const int xc = kv * kM, yc = a.y_col0 + kv * a.y_col_kv + n0;
    int issued = 0;
    for (int ks = 0; ks < nk; ++ks) {
      const int st = ks % kStages;
      if (ks >= kStages && !mbar_wait(empty + st, ((ks / kStages) - 1) & 1, abort_flag)) {
        tc_fail(a.err, 94, abort_flag);
        break;
      }
      const int row = r0 + ks * kK;   // rows past T are filled with zeros by the TMA unit
      uint8_t* stg = sm + st * kStage;
      mbar_arrive_expect_tx(full + st, kStage);
      tma_load_2d(stg, &tXh, full + st, xc, row);
      tma_load_2d(stg + kBox, &tXh, full + st, xc + 64, row);
      tma_load_2d(stg + 2 * kBox, &tXl, full + st, xc, row);
      tma_load_2d(stg + 3 * kBox, &tXl, full + st, xc + 64, row);
      tma_load_2d(stg + 4 * kBox, &tY, full + st, yc, row);
      tma_load_2d(stg + 5 * kBox, &tY, full + st, yc + 64, row);
      issued = ks + 1;
    }
    for (int ks = max(0, issued - kStages); ks < issued; ++ks)
      mbar_wait_drain(full + ks % kStages, (ks / kStages) & 1);
  } else if (warp == 1 && lane == 0) {   // MMA issue
    // A = X^T (M = W rows, K = token rows), B = Y (N = W columns, K = token rows): both
    // MN-major in the chunk ([64 rows][64 elements] halves, 8 KB apart)
    constexpr uint32_t kId = idesc_bf16_f32(kM, kN, true, true);
    bool ok = true;
    for (int ks = 0; ks < nk; ++ks) {
      const int st = ks % kStages;
      if (!mbar_wait(full + st, (ks / kStages) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t base = smem_u32(sm + st * kStage);
#pragma unroll
      for (int kk = 0; kk < kK / 16; ++kk) {   // 16 token rows per MMA
        const uint64_t bdesc = sdesc_sw128(base + 4 * kBox + kk * 2048, kBox, 1024);
        mma_bf16_ss(tmem, sdesc_sw128(base + kk * 2048, kBox, 1024), bdesc, kId,
                    (ks > 0 || kk > 0) ? 1u : 0u);
        mma_bf16_ss(tmem, sdesc_sw128(base + 2 * kBox + kk * 2048, kBox, 1024), bdesc, kId, 1u);
      }
      tc_commit(empty + st);
    }
    if (!ok) tc_fail(a.err, 95, abort_flag);
    tc_commit(done);
    mbar_wait_drain(done, 0);
  }
  __syncwarp();
  // epilogue: thread r = TMEM lane r = W row r; 128 fp32 W columns
  const bool have = warp_wait(done, 0, abort_flag) && nk > 0;
  if (have) {
    tc_fence_after();
    int col = n0;
    if (a.mean_cols > 0 && n0 >= 2 * a.mean_cols) col = 2 * a.mean_cols;   // mean parts
    float* drow = a.dW + ((size_t)kv * kM + tid) * a.C + col;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
    for (int c0 = 0; c0 < kN; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_addr + c0, v);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        red_add_v4(drow + c0 + 4 * i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
    }
  } else if (nk > 0) {
    tc_fail(a.err, 96, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kN);
  }
}

// dx fp32 -> bf16 hi + lo (hi = round(x), lo = round(x - hi))
__global__ void gbw_split_kernel(const float4* __restrict__ x, size_t n4, uint2* __restrict__ hi,
                                 uint2* __restrict__ lo) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = x[i];
    const __nv_bfloat16 h0 = __float2bfloat16_rn(v.x), h1 = __float2bfloat16_rn(v.y);
    const __nv_bfloat16 h2 = __float2bfloat16_rn(v.z), h3 = __float2bfloat16_rn(v.w);
    uint2 H, L;
    H.x = sm100::pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
    H.y = sm100::pack_bf16x2(__bfloat162float(h2), __bfloat162float(h3));
    L.x = sm100::pack_bf16x2(v.x - __bfloat162float(h0), v.y - __bfloat162float(h1));
    L.y = sm100::pack_bf16x2(v.z - __bfloat162float(h2), v.w - __bfloat162float(h3));
    hi[i] = H;
    lo[i] = L;
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
namespace {
struct GbwLayout {
  size_t tc, xk, kt, dkt, dxk, dxq, dxc, xh, xl, total;
};
size_t al256w(size_t x) { return (x + 255) & ~(size_t)255; }
GbwLayout gbw_layout(const sas_problem& p) {
  GbwLayout L;
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const size_t brow = (size_t)p.batch * NBmax * p.num_kv_heads * gbw::H * 4;
  const size_t trow = (size_t)p.total_tokens * p.num_kv_heads * gbw::H * 4;
  size_t o = 0;
  L.tc = o;  o += al256w(gate_tc_workspace_bytes(p));
  L.xk = o;  o += al256w(brow);
  L.kt = o;  o += al256w(brow);
  L.dkt = o; o += al256w(brow);
  L.dxk = o; o += al256w(brow);
  L.dxq = o; o += al256w(trow);
  L.dxc = o; o += al256w(trow);
  L.xh = o;  o += al256w(trow / 2);   // dx as bf16 hi / lo parts for the tensor-core products
  L.xl = o;  o += al256w(trow / 2);
  L.total = o;
  return L;
}
}  // namespace

bool gate_bwd_supported(const sas_problem& p) {
  return gate_tc_supported(p) && p.gate_hidden == gbw::H && p.head_dim == 128 &&
         gate_heads(p) == p.num_kv_heads;
}

size_t gate_bwd_workspace_bytes(const sas_problem& p) { return gbw_layout(p).total; }

sas_status launch_gate_bwd(const sas_problem& p, const void* q_nope, const void* k_nope,
                           const float* pooled, const void* wq, const float* qnorm_w,
                           const void* wk, const float* knorm_w, const int32_t* idx,
                           const float* dlogg, float* dwq, float* dqnorm_w, float* dwk,
                           float* dknorm_w, void* workspace, cudaStream_t st) {
  const GbwLayout L = gbw_layout(p);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int Hkv = p.num_kv_heads, Hq = p.num_q_heads, G = Hq / Hkv, d = p.head_dim;
  const int T = p.total_tokens, B = p.block;
  const int NBmax = (p.max_seqlen + B - 1) / B;
  float* xk = reinterpret_cast<float*>(ws + L.xk);
  float* kt = reinterpret_cast<float*>(ws + L.kt);
  float* dkt = reinterpret_cast<float*>(ws + L.dkt);
  float* dxk = reinterpret_cast<float*>(ws + L.dxk);
  float* dxq = reinterpret_cast<float*>(ws + L.dxq);
  float* dxc = reinterpret_cast<float*>(ws + L.dxc);
  const size_t brow = (size_t)p.batch * NBmax * Hkv * gbw::H * 4;
  if (cudaMemsetAsync(dwq, 0, (size_t)Hkv * gbw::H * G * d * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dwk, 0, (size_t)Hkv * gbw::H * 3 * d * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dqnorm_w, 0, gbw::H * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dknorm_w, 0, gbw::H * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dkt, 0, brow, st) != cudaSuccess) {
    set_error("gate_bwd: clearing the outputs failed");
    return SAS_ERR_CUDA;
  }
  float *xq_all = nullptr, *xc_all = nullptr;
  const void* prefix_rows = nullptr;
  SAS_TRY(launch_gate_proj_tc(p, q_nope, k_nope, wq, wk, ws + L.tc, &xq_all, &xc_all, st,
                              &prefix_rows));
  const int nsm = sm_count();
  const __nv_bfloat16* qn = static_cast<const __nv_bfloat16*>(q_nope);
  const __nv_bfloat16* kn = static_cast<const __nv_bfloat16*>(k_nope);
  gbw_block_fwd_kernel<<<2 * nsm, gbw::kRowThreads, 0, st>>>(
      pooled, static_cast<const __nv_bfloat16*>(wk), knorm_w, p.cu_seqlens, p.gate_rope_cos,
      p.gate_rope_sin, p.batch, NBmax, Hkv, d, B, p.rms_eps, xk, kt);
  gbw_row_kernel<<<4 * nsm, gbw::kRowThreads, 0, st>>>(
      xq_all, xc_all, kt, idx, dlogg, qnorm_w, knorm_w, p.cu_seqlens, p.gate_rope_cos,
      p.gate_rope_sin, p.batch, T, NBmax, Hkv, B, p.topk + 1, p.rms_eps, dkt, dxq, dxc, dqnorm_w,
      dknorm_w);
  gbw_block_bwd_kernel<<<2 * nsm, gbw::kRowThreads, 0, st>>>(
      xk, dkt, knorm_w, p.cu_seqlens, p.gate_rope_cos, p.gate_rope_sin, p.batch, NBmax, Hkv, B,
      p.rms_eps, dxk, dknorm_w);
  // block-row outer products (few rows) on CUDA cores
  const int CQ = G * d, CK = 3 * d;
  const int tk = (CK / gbw::kTile) * (gbw::H / gbw::kTile) * Hkv;
  const int sk = max(1, min(64, 16 * nsm / tk));
  gbw_outer_kernel<1><<<dim3(CK / gbw::kTile, gbw::H / gbw::kTile, Hkv * sk), 64, 0, st>>>(
      dxk, qn, pooled, kn, p.cu_seqlens, p.batch, T, Hq, Hkv, d, B, NBmax, CK, sk, dwk);
  // token-row outer products on the tensor cores: dWq from dxq and the query heads, the
  // token part of dWk from dxc and the forward gate's prefix-pool rows
  __nv_bfloat16* xh = reinterpret_cast<__nv_bfloat16*>(ws + L.xh);
  __nv_bfloat16* xl = reinterpret_cast<__nv_bfloat16*>(ws + L.xl);
  CUtensorMap tXh, tXl, tQ, tP;
  if (!make_tmap_bf16_2d(&tXh, xh, (uint64_t)Hkv * gbw::H, T, (uint64_t)Hkv * gbw::H * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tXl, xl, (uint64_t)Hkv * gbw::H, T, (uint64_t)Hkv * gbw::H * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tQ, q_nope, (uint64_t)Hq * d, T, (uint64_t)Hq * d * 2, 64, 64) ||
      !make_tmap_bf16_2d(&tP, prefix_rows, (uint64_t)Hkv * 5 * d, T, (uint64_t)Hkv * 5 * d * 2,
                         64, 64)) {
    set_error("gate_bwd: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(gbw_wgrad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         gwt::kSmemBytes);
  });
  const int chunks = (T + gwt::kK - 1) / gwt::kK;
  auto wgrad = [&](const float* dx, const CUtensorMap& tY, int y_col_kv, int ncol_tiles, float* dW,
                   int C, int mean_cols) {
    const size_t n4 = (size_t)T * Hkv * gbw::H / 4;
    gbw_split_kernel<<<4 * nsm, 256, 0, st>>>(reinterpret_cast<const float4*>(dx), n4,
                                              reinterpret_cast<uint2*>(xh),
                                              reinterpret_cast<uint2*>(xl));
    const int ctas = ncol_tiles * Hkv;
    const int nsplit = max(1, min(chunks, (2 * nsm + ctas - 1) / ctas));
    WgradArgs wa{T, ((chunks + nsplit - 1) / nsplit) * gwt::kK, 0, y_col_kv, dW, C, mean_cols,
                 reinterpret_cast<int*>(ws)};
    gbw_wgrad_tc_kernel<<<dim3(ncol_tiles, Hkv, nsplit), gwt::kThreads, gwt::kSmemBytes, st>>>(
        tXh, tXl, tY, wa);
  };
  wgrad(dxq, tQ, G * d, CQ / gwt::kN, dwq, CQ, 0);
  wgrad(dxc, tP, 5 * d, 5 * d / gwt::kN, dwk, CK, d);
  return launch_status("gate backward", 11);   // + the prefix pass and two projection GEMMs
}

}  // namespace sas
