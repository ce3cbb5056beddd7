// Gate scores with the historical part on the tensor cores (A3), after the two projections:
// gate_qk_split_kernel normalises and rotates q~ and the current block's key, writes q~ split
// into tf32 hi + lo and the current block's score s[t, c_t]; gate_hist_tc_kernel computes
// s[t, j] = q~_t . k~_j / sqrt(h) for every block j before c_t, the -inf padding past c_t, and
// the logsumexp over j <= c_t. Model card "tencent/Simple-Attention-Sparsification", "Checkpoint configuration"
// (gate hidden 128); paper abstract (softmax over history plus the current block).
//
// The selection must agree with an exact evaluation except at near-ties, so the products keep
// fp32-like accuracy: q~ and k~ are split into x = hi + lo, hi the nearest tf32 value of x and
// lo = x - hi (|lo| <= 2^-11 |x|), and each tile accumulates hi.hi + hi.lo + lo.hi with three
// kind::tf32 MMAs into one fp32 TMEM accumulator. The dropped lo.lo term and the tf32 rounding
// of lo are below 2^-21 of |q_i k_i|, the size of the rounding of an fp32 dot product.
//
// CTA = (128-token tile of one sequence, gate head); tiles are taken longest first. The tile's
// q~ hi/lo (128 x 128 fp32 each, 128 KB) arrive once by TMA; the block keys stream in chunks of
// 128 blocks x 32 channels (hi and lo, 32 KB per stage, two stages):
//   S_chunk (M = 128 tokens, N = 128 blocks, K = 128) in TMEM, two buffers of 128 columns.
// Warp roles (256 threads): warp 0 lane 0 loads; warp 1 allocates TMEM and lane 0 issues the
// MMAs; warps 2-3 write the -inf padding past the last chunk; warps 4-7 own one token row per
// lane: scale, mask, online logsumexp, and the row's scores go out through a per-warp shared
// transpose so that each store instruction writes 32 consecutive blocks of one row.
// Every wait is bounded; a timeout records error code 97 (loads), 98 (MMA) or 99 (epilogue)
// in the workspace's error word.
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_gate.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace ghc {
constexpr int kM = 128, kN = 128, kH = 128;   // tokens, blocks per chunk, gate hidden
constexpr int kThreads = 256;
constexpr int kAtom = 128 * 128;              // [128 rows][128 B] = 16 KB (32 fp32 of K)
constexpr int kStages = 2;
constexpr int OFF_AHI = 0;                    // 4 K-atoms of q~ hi
constexpr int OFF_ALO = 4 * kAtom;            // 4 K-atoms of q~ lo
constexpr int OFF_B = 8 * kAtom;              // stage s: key hi atom, key lo atom
constexpr int OFF_TR = OFF_B + kStages * 2 * kAtom;   // [4 warps][32][33] fp32 transpose
constexpr int OFF_BAR = OFF_TR + 4 * 32 * 33 * 4;
// a_full, b_full[2], b_empty[2], acc_full[2], acc_empty[2], final
constexpr int kNumBars = 1 + 2 * kStages + 4 + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;
constexpr uint32_t kTmemCols = 256;
}  // namespace ghc

struct GhcArgs {
  const int32_t* cu;
  float* scores;   // [T][Hs][NBmax]
  float* lse;      // [T][Hs]
  int* err;
  int batch, Hs, Hkv, B, NBmax;
};

__global__ void split_tf32_kernel(const float* __restrict__ x, float* __restrict__ hi,
                                  float* __restrict__ lo, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float v = x[i], h = tf32_hi(v);
    hi[i] = h;
    lo[i] = v - h;
  }
}

// q~ and the current block's score for the tensor-core path: one warp per (token, gate head).
// The two projected rows (Qproj of the gate head, Kproj of the current block's prefix pool) are
// held as four elements per lane (channels lane + 32 u), so the rotate-half pairs (e, e + 64)
// sit in the same lane; RMSNorm (weight after the normalisation), rotary at t (query) and at
// c_t B (current block), then q~ split into tf32 hi + lo, and s[t, c_t] = q~ . k~cur / sqrt(h).
// The sums run in the same order as the shared-memory kernels' (lane partials over e = lane,
// lane + 32, ..., then the warp tree).
__global__ void __launch_bounds__(256) gate_qk_split_kernel(
    const float* __restrict__ qproj, const float* __restrict__ kproj, const float* __restrict__ qnorm_w,
    const float* __restrict__ knorm_w, const int32_t* __restrict__ cu, const float* __restrict__ rc,
    const float* __restrict__ rs, int batch, int T, int Hs, int Hkv, int B, int NBmax, float eps,
    float* __restrict__ qhi, float* __restrict__ qlo, float* __restrict__ scores) {
  constexpr int H = ghc::kH;
  const int lane = threadIdx.x & 31;
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  if (gw >= (long long)T * Hs) return;
  const int tg = (int)(gw / Hs), sh = (int)(gw - (long long)tg * Hs);
  const int kv = sh / (Hs / Hkv);
  const int b = seq_of(cu, batch, tg);
  const int t = tg - cu[b], c = t / B;
  auto norm_rope = [&](float* x, const float* __restrict__ w, int pos) {
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) ss += x[u] * x[u];
    ss = warp_sum(ss);
    const float rn = sqrtf(ss / (float)H + eps);
#pragma unroll
    for (int u = 0; u < 2; ++u) {   // pairs (lane + 32 u, lane + 32 u + 64)
      const int e = lane + 32 * u;
      const float a = x[u] / rn * w[e], bb = x[u + 2] / rn * w[e + H / 2];
      const float cs = rc[(size_t)pos * (H / 2) + e], sn = rs[(size_t)pos * (H / 2) + e];
      x[u] = a * cs - bb * sn;
      x[u + 2] = bb * cs + a * sn;
    }
  };
  float q[4], k[4];
  const float* qr = qproj + (size_t)gw * H;
  const float* kr = kproj + ((size_t)tg * Hkv + kv) * H;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    q[u] = qr[lane + 32 * u];
    k[u] = kr[lane + 32 * u];
  }
  norm_rope(q, qnorm_w, t);
  norm_rope(k, knorm_w, c * B);
  float dot = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float hi = tf32_hi(q[u]);
    qhi[(size_t)gw * H + lane + 32 * u] = hi;
    qlo[(size_t)gw * H + lane + 32 * u] = q[u] - hi;
    dot += q[u] * k[u];
  }
  dot = warp_sum(dot);
  if (lane == 0) scores[(size_t)gw * NBmax + c] = dot / sqrtf((float)H);
}

__global__ void __launch_bounds__(ghc::kThreads, 1)
    gate_hist_tc_kernel(const __grid_constant__ CUtensorMap tmAhi, const __grid_constant__ CUtensorMap tmAlo,
                        const __grid_constant__ CUtensorMap tmBhi, const __grid_constant__ CUtensorMap tmBlo,
                        const GhcArgs a) {
  using namespace ghc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = gridDim.x - 1 - blockIdx.x, b = blockIdx.y, sh = blockIdx.z;
  const int kv = sh / (a.Hs / a.Hkv);
  const int s0 = a.cu[b], L = a.cu[b + 1] - s0;
  const int t0 = tile * kM;
  if (t0 >= L) return;
  const int nt = min(kM, L - t0);
  const int c_last = (t0 + nt - 1) / a.B;     // historical blocks of the tile: j < c_last
  const int nch = (c_last + kN - 1) / kN;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* b_full = bars + 1;
  uint64_t* b_empty = b_full + kStages;
  uint64_t* acc_full = b_empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* final_bar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);

  if (tid == 0) {
    mbar_init(a_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(b_full + i, 1);
      mbar_init(b_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 128);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- loads ----------------
    if (lane == 0 && nch > 0) {
      prefetch_tmap(&tmAhi);
      prefetch_tmap(&tmAlo);
      prefetch_tmap(&tmBhi);
      prefetch_tmap(&tmBlo);
      mbar_arrive_expect_tx(a_full, 8 * kAtom);
      for (int ka = 0; ka < 4; ++ka) {
        tma_load_3d(sm + OFF_AHI + ka * kAtom, &tmAhi, a_full, ka * 32, sh, s0 + t0);
        tma_load_3d(sm + OFF_ALO + ka * kAtom, &tmAlo, a_full, ka * 32, sh, s0 + t0);
      }
      int issued = 0;
      for (int g = 0; g < 4 * nch; ++g) {
        const int slot = g % kStages, n = g >> 2, ks = g & 3;
        if (g >= kStages && !mbar_wait(b_empty + slot, ((g / kStages) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 97, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(b_full + slot, 2 * kAtom);
        uint8_t* dst = sm + OFF_B + slot * 2 * kAtom;
        tma_load_4d(dst, &tmBhi, b_full + slot, ks * 32, kv, n * kN, b);
        tma_load_4d(dst + kAtom, &tmBlo, b_full + slot, ks * 32, kv, n * kN, b);
        issued = g + 1;
      }
      mbar_wait_drain(a_full, 0);
      for (int g = max(0, issued - kStages); g < issued; ++g)   // none in flight at exit
        mbar_wait_drain(b_full + g % kStages, (g / kStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0 && nch > 0) {
      constexpr uint32_t kId = idesc_tf32_f32(kM, kN);
      bool ok = mbar_wait(a_full, 0, abort_flag);
      const uint32_t ahi = smem_u32(sm + OFF_AHI), alo = smem_u32(sm + OFF_ALO);
      const uint32_t bb = smem_u32(sm + OFF_B);
      for (int n = 0; ok && n < nch; ++n) {
        const int buf = n & 1;
        if (n >= 2 && !mbar_wait(acc_empty + buf, ((n >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + buf * kN;
        for (int ks = 0; ks < 4; ++ks) {
          const int g = n * 4 + ks, slot = g % kStages;
          if (!mbar_wait(b_full + slot, (g / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t bh = bb + slot * 2 * kAtom, bl = bh + kAtom;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {   // 8 channels (32 bytes) per MMA
            const uint32_t ao = ks * kAtom + k4 * 32, bo = k4 * 32;
            mma_tf32_ss(d, sdesc_sw128(ahi + ao, 16, 1024), sdesc_sw128(bh + bo, 16, 1024), kId,
                        (ks | k4) ? 1u : 0u);
            mma_tf32_ss(d, sdesc_sw128(ahi + ao, 16, 1024), sdesc_sw128(bl + bo, 16, 1024), kId, 1u);
            mma_tf32_ss(d, sdesc_sw128(alo + ao, 16, 1024), sdesc_sw128(bh + bo, 16, 1024), kId, 1u);
          }
          tc_commit(b_empty + slot);
        }
        if (!ok) break;
        tc_commit(acc_full + buf);
      }
      if (!ok) tc_fail(a.err, 98, abort_flag);
      tc_commit(final_bar);
      mbar_wait_drain(final_bar, 0);
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------- -inf past the last chunk (the current block's entry excepted) ----------
    const int jstart = nch * kN;
    for (int r = warp - 2; r < nt; r += 2) {
      const int c_t = (t0 + r) / a.B;
      float* srow = a.scores + ((size_t)(s0 + t0 + r) * a.Hs + sh) * a.NBmax;
      for (int j = jstart + lane; j < a.NBmax; j += 32)
        if (j != c_t) srow[j] = -INFINITY;
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: one token row per lane ----------------
    const int w4 = warp - 4;
    const int r = w4 * 32 + lane;
    const bool valid = r < nt;
    const int c_t = valid ? (t0 + r) / a.B : -1;
    const uint32_t lane_addr = (uint32_t)(w4 * 32) << 16;
    float* tr = reinterpret_cast<float*>(sm + OFF_TR) + w4 * 32 * 33;
    const float inv_sqrt_h = 0.0883883476483184406f;   // 1 / sqrt(128), correctly rounded
    float m2 = -INFINITY, l = 0.f;   // running max and sum, log2 units
    bool ok = true;
    for (int n = 0; n < nch; ++n) {
      const int buf = n & 1;
      if (!warp_wait(acc_full + buf, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int grp = 0; grp < 4; ++grp) {
        float v[32];
        tmem_ld32(tmem + lane_addr + buf * kN + grp * 32, v);
        if (grp == 3) {   // the buffer is free for chunk n + 2
          tc_fence_before();
          mbar_arrive(acc_empty + buf);
        }
        const int jb = n * kN + grp * 32;
        float gm = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] *= inv_sqrt_h;
          if (jb + i < c_t) gm = fmaxf(gm, v[i]);
        }
        if (gm != -INFINITY) {   // online logsumexp in log2 units
          const float g2 = gm * kLog2e;
          if (g2 > m2) {
            l = l * ex2_approx(m2 - g2);
            m2 = g2;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (jb + i < c_t) l += ex2_approx(fmaf(v[i], kLog2e, -m2));
        }
        // transpose through shared memory: row `lane` of this warp's 32 rows
#pragma unroll
        for (int i = 0; i < 32; ++i) tr[lane * 33 + i] = v[i];
        __syncwarp();
        for (int rr = 0; rr < 32; ++rr) {
          const int rrow = w4 * 32 + rr;
          const int crr = __shfl_sync(0xffffffffu, c_t, rr);
          const int j = jb + lane;
          if (rrow < nt && j < a.NBmax && j != crr) {
            const float x = tr[rr * 33 + lane];
            a.scores[((size_t)(s0 + t0 + rrow) * a.Hs + sh) * a.NBmax + j] = j < crr ? x : -INFINITY;
          }
        }
        __syncwarp();
      }
    }
    if (!ok) tc_fail(a.err, 99, abort_flag);
    if (valid) {   // the current block's score (written by gate_qk_split_kernel) closes the sum
      const size_t row = (size_t)(s0 + t0 + r) * a.Hs + sh;
      const float y = a.scores[row * a.NBmax + c_t] * kLog2e;
      const float M = fmaxf(m2, y);
      const float tot = (m2 == -INFINITY ? 0.f : l * ex2_approx(m2 - M)) + ex2_approx(y - M);
      a.lse[row] = (M + __log2f(tot)) * kLn2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
bool gate_hist_tc_supported(const sas_problem& p) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  return gate_tc_supported(p) && p.gate_hidden == ghc::kH && NBmax >= 1;
}

static size_t al256h(size_t x) { return (x + 255) & ~(size_t)255; }

size_t gate_hist_tc_workspace_bytes(const sas_problem& p) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const size_t keys = (size_t)p.batch * NBmax * p.num_kv_heads * ghc::kH;
  return 2 * al256h(keys * 4);
}

sas_status launch_gate_hist_tc(const sas_problem& p, const float* gkeys, const float* qproj,
                               const float* kproj, const float* qnorm_w, const float* knorm_w,
                               float* qhi, float* qlo, void* key_ws, float* scores, float* lse,
                               int* err, cudaStream_t st) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const int Hs = gate_heads(p), Hkv = p.num_kv_heads;
  {
    const long long warps = (long long)p.total_tokens * Hs;
    gate_qk_split_kernel<<<(int)((warps * 32 + 255) / 256), 256, 0, st>>>(
        qproj, kproj, qnorm_w, knorm_w, p.cu_seqlens, p.gate_rope_cos, p.gate_rope_sin, p.batch,
        p.total_tokens, Hs, Hkv, p.block, NBmax, p.rms_eps, qhi, qlo, scores);
  }
  const size_t keys = (size_t)p.batch * NBmax * Hkv * ghc::kH;
  float* ghi = (float*)key_ws;
  float* glo = (float*)((char*)key_ws + al256h(keys * 4));
  split_tf32_kernel<<<(int)std::min<size_t>((keys + 255) / 256, 4096), 256, 0, st>>>(gkeys, ghi, glo, keys);
  CUtensorMap tah, tal, tbh, tbl;
  const uint64_t adims[3] = {(uint64_t)ghc::kH, (uint64_t)Hs, (uint64_t)p.total_tokens};
  const uint32_t abox[3] = {32, 1, (uint32_t)ghc::kM};
  const uint64_t bdims[4] = {(uint64_t)ghc::kH, (uint64_t)Hkv, (uint64_t)NBmax, (uint64_t)p.batch};
  const uint32_t bbox[4] = {32, 1, (uint32_t)ghc::kN, 1};
  if (!make_tmap_f32_sw128(&tah, qhi, 3, adims, abox) || !make_tmap_f32_sw128(&tal, qlo, 3, adims, abox) ||
      !make_tmap_f32_sw128(&tbh, ghi, 4, bdims, bbox) || !make_tmap_f32_sw128(&tbl, glo, 4, bdims, bbox)) {
    set_error("gate_scores: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(gate_hist_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ghc::kSmemBytes);
  });
  GhcArgs a;
  a.cu = p.cu_seqlens;
  a.scores = scores;
  a.lse = lse;
  a.err = err;
  a.batch = p.batch;
  a.Hs = Hs;
  a.Hkv = Hkv;
  a.B = p.block;
  a.NBmax = NBmax;
  const dim3 grid((p.max_seqlen + ghc::kM - 1) / ghc::kM, p.batch, Hs);
  gate_hist_tc_kernel<<<grid, ghc::kThreads, ghc::kSmemBytes, st>>>(tah, tal, tbh, tbl, a);
  return SAS_OK;
}

}  // namespace sas
