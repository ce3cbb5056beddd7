// Tensor-core (tcgen05 / TMEM) backward of the gated sparse attention (A6), bf16, head_dim
// 128, KV block 64. The loss reaches the selector through standard backpropagation (paper
// abstract): besides dQ, dK, dV the backward returns the gradient of every kept block's
// log-gate, dlogg = sum over the G heads and the block's keys of dS = P (dP - D).
//
// Two passes, no atomics on any output, every sum in a fixed order:
//   query-major  CTA = (tile of Mq tokens x G heads = 128 rows, kv head), visiting the union
//                of the tile rows' blocks (as the forward). Per block: S = Q K^T and
//                dP = dO V^T (TMEM, double-buffered), dS = P (dP - D) -> bf16 shared tile,
//                dQ += dS K (TMEM). Row sums of dS over the G heads of a token give dlogg.
//   key-major    CTA = (pair of KV blocks = 128 keys, kv head), visiting only the tokens
//                that kept one of the two blocks: a pre-pass writes, per (kv, block pair),
//                a bitmask over tokens; the CTA walks its row in token order and gathers
//                128-row tiles (Mq tokens x G heads) of Q and dO with cp.async. Per tile:
//                S^T = K Q^T, dP^T = V dO^T (keys on TMEM lanes, rows on columns, so the
//                per-row statistics are per-column constants), P^T and dS^T -> bf16 shared
//                tiles, dV += P^T dO, dK += dS^T Q (TMEM).
// D = rowsum(dO * O) comes from the CUDA-core row-dot kernel.
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace tcb {
constexpr int kD = 128, kB = 64, kM = 128, kThreads = 384;   // query-major: 4 role warps + 2 dS warpgroups
constexpr int kHalf = kM * 128;          // 128 rows x 128 B
constexpr int kKVHalf = kB * 128;        // 64 rows x 128 B
constexpr int kStageBytes = 4 * kKVHalf; // K0 K1 V0 V1
constexpr int kTileBytes = kM * 128;     // 128 x 64 bf16 (dS tile)
constexpr int kStages = 2;
constexpr int kMaxSel = 2048;
constexpr int kMaxBlocks = 2048;
// query-major pass layout
constexpr int Q_OFF_Q = 0;
constexpr int Q_OFF_DO = Q_OFF_Q + 2 * kHalf;
constexpr int Q_OFF_KV = Q_OFF_DO + 2 * kHalf;
constexpr int Q_OFF_DS = Q_OFF_KV + kStages * kStageBytes;
constexpr int Q_OFF_SEL_IDX = Q_OFF_DS + 2 * kTileBytes;
constexpr int Q_OFF_SEL_LG = Q_OFF_SEL_IDX + kMaxSel * 4;
constexpr int Q_OFF_LIST = Q_OFF_SEL_LG + kMaxSel * 4;
constexpr int Q_OFF_MASK = Q_OFF_LIST + kMaxBlocks * 4;
constexpr int Q_OFF_RS = Q_OFF_MASK + kMaxBlocks / 8;          // [2 wg][2][128] floats
constexpr int Q_OFF_BAR = Q_OFF_RS + 4 * 128 * 4;
constexpr int Q_NBARS = 1 + 2 * kStages + 2 + 2 + 2 + 1;
constexpr int Q_OFF_MISC = Q_OFF_BAR + Q_NBARS * 8;
constexpr int Q_SMEM = Q_OFF_MISC + 64 + 1024;
// gathered key-major pass layout
constexpr int kGThreads = 384;           // warps 0-3 gather, 4 MMA, 8-11 softmax
constexpr int kMaxWords = 2048;          // token bitmask words per row (max_seqlen <= 65536)
constexpr int G_OFF_K = 0;               // [128 keys][128 d] as 2 halves
constexpr int G_OFF_V = G_OFF_K + 2 * kHalf;
constexpr int G_OFF_Q = G_OFF_V + 2 * kHalf;     // gathered [128 rows][128 d]
constexpr int G_OFF_DO = G_OFF_Q + 2 * kHalf;
constexpr int G_OFF_PT = G_OFF_DO + 2 * kHalf;   // P^T  [128 keys][128 rows] as 2 halves
constexpr int G_OFF_DST = G_OFF_PT + 2 * kHalf;  // dS^T [128 keys][128 rows]
constexpr int G_OFF_RC = G_OFF_DST + 2 * kHalf;  // [2][4][128] row constants
constexpr int G_OFF_WORDS = G_OFF_RC + 2 * 4 * 128 * 4;
constexpr int G_OFF_PREFIX = G_OFF_WORDS + kMaxWords * 4;
constexpr int G_OFF_PART = G_OFF_PREFIX + kMaxWords * 4;   // kGThreads partial counts
constexpr int G_OFF_BAR = G_OFF_PART + kGThreads * 4;
constexpr int G_NBARS = 6;
constexpr int G_OFF_MISC = G_OFF_BAR + G_NBARS * 8;
constexpr int G_SMEM = G_OFF_MISC + 64 + 1024;
}  // namespace tcb

struct TcBwdArgs {
  const int32_t* cu;
  const int32_t* idx;
  const float* logg;
  const float* lse;
  const float* drow;
  const uint32_t* pmask;      // [batch][Hkv][NP][W] token bitmask per block pair
  const __nv_bfloat16* q;     // raw pointers for the gathered copies
  const __nv_bfloat16* dout;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dlogg;
  int* err;
  int Hq, Hkv, G, K, Mq, NBmax, n_tiles, NP, W;
  float scale_log2, scale;
};


// ---------------------------------------------------------------------------------------
// pre-pass: bit t of pmask[b][kv][p] = token t of sequence b kept block 2p or 2p+1
// ---------------------------------------------------------------------------------------
__global__ void pair_mask_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cu,
                                 int batch, int T, int Hkv, int K, int NP, int W,
                                 uint32_t* __restrict__ pmask) {
  const int row = (int)(blockIdx.x * (size_t)blockDim.x + threadIdx.x);
  if (row >= T * Hkv) return;
  const int tg = row / Hkv, kv = row - tg * Hkv;
  const int b = seq_of(cu, batch, tg);
  const int t = tg - cu[b];
  uint32_t* base = pmask + ((size_t)(b * Hkv + kv) * NP) * W + (t >> 5);
  const uint32_t bit = 1u << (t & 31);
  const int32_t* ir = idx + (size_t)row * (K + 1);
  int prev = -1;
  for (int s = 0; s <= K; ++s) {
    const int j = ir[s];
    if (j < 0) break;
    const int p = j >> 1;
    if (p != prev && p < NP) atomicOr(base + (size_t)p * W, bit);
    prev = p;
  }
}

// ---------------------------------------------------------------------------------------
// query-major pass: dQ and dlogg
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(tcb::kThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const TcBwdArgs a) {
  using namespace tcb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = a.n_tiles - 1 - (int)blockIdx.x;
  const int b = blockIdx.y, kv = blockIdx.z;
  const int s0 = a.cu[b], L = a.cu[b + 1] - s0;
  const int t0 = tile * a.Mq;
  if (t0 >= L) return;
  const int nt = min(a.Mq, L - t0);
  const int G = a.G, K1 = a.K + 1;
  const int rows_used = G * a.Mq;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Q_OFF_BAR);
  uint64_t* qd_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* ds_full = s_full + 2;
  uint64_t* ds_free = ds_full + 2;
  uint64_t* dq_final = ds_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Q_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Q_OFF_MISC + 4);
  int* n_list_s = reinterpret_cast<int*>(sm + Q_OFF_MISC + 8);
  int32_t* sel_idx = reinterpret_cast<int32_t*>(sm + Q_OFF_SEL_IDX);
  float* sel_lg = reinterpret_cast<float*>(sm + Q_OFF_SEL_LG);
  int32_t* list = reinterpret_cast<int32_t*>(sm + Q_OFF_LIST);
  uint32_t* mask = reinterpret_cast<uint32_t*>(sm + Q_OFF_MASK);
  float* rs = reinterpret_cast<float*>(sm + Q_OFF_RS);

  const int nwords = (a.NBmax + 31) >> 5;
  for (int w = tid; w < nwords; w += kThreads) mask[w] = 0u;
  if (tid == 0) {
    mbar_init(qd_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(ds_full + i, 128);
      mbar_init(ds_free + i, 1);
    }
    mbar_init(dq_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (rows_used < kM) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int e = tid; e < (kM - rows_used) * 8; e += kThreads) {
      const int r = rows_used + (e >> 3), c = e & 7;
      reinterpret_cast<uint4*>(sm + Q_OFF_Q + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + Q_OFF_Q + kHalf + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + Q_OFF_DO + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + Q_OFF_DO + kHalf + r * 128)[c] = z;
    }
    fence_async_smem();
  }
  __syncthreads();
  for (int e = tid; e < nt * K1; e += kThreads) {
    const int tl = e / K1, sl = e - tl * K1;
    const size_t gi = ((size_t)(s0 + t0 + tl) * a.Hkv + kv) * K1 + sl;
    const int j = a.idx[gi];
    sel_idx[e] = j;
    sel_lg[e] = a.logg[gi];
    if (j >= 0 && j < a.NBmax) atomicOr(&mask[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t bits = (w < nwords) ? mask[w] : 0u;
      const int cnt = __popc(bits);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = base + incl - cnt;
      uint32_t bb = bits;
      while (bb) {
        const int bit = __ffs(bb) - 1;
        bb &= bb - 1u;
        list[pos++] = w * 32 + bit;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *n_list_s = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int nb = *n_list_s;
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {   // producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmDO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(qd_full, 4u * rows_used * 128u);
      tma_load_3d(sm + Q_OFF_Q, &tmQ, qd_full, 0, kv * G, s0 + t0);
      tma_load_3d(sm + Q_OFF_Q + kHalf, &tmQ, qd_full, 64, kv * G, s0 + t0);
      tma_load_3d(sm + Q_OFF_DO, &tmDO, qd_full, 0, kv * G, s0 + t0);
      tma_load_3d(sm + Q_OFF_DO + kHalf, &tmDO, qd_full, 64, kv * G, s0 + t0);
      int issued = 0;
      for (int n = 0; n < nb; ++n) {
        const int st = n % kStages;
        if (n >= kStages && !mbar_wait(kv_empty + st, ((n / kStages) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 11, abort_flag);
          break;
        }
        const int row = s0 + list[n] * kB;
        uint8_t* stg = sm + Q_OFF_KV + st * kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, kStageBytes);
        tma_load_3d(stg, &tmK, kv_full + st, 0, kv, row);
        tma_load_3d(stg + kKVHalf, &tmK, kv_full + st, 64, kv, row);
        tma_load_3d(stg + 2 * kKVHalf, &tmV, kv_full + st, 0, kv, row);
        tma_load_3d(stg + 3 * kKVHalf, &tmV, kv_full + st, 64, kv, row);
        issued = n + 1;
      }
      mbar_wait_drain(qd_full, 0);
      for (int n = max(0, issued - kStages); n < issued; ++n)
        mbar_wait_drain(kv_full + n % kStages, (n / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {   // MMA issuer
      constexpr uint32_t kIdS = idesc_bf16_f32(kM, kB, false, false);     // S, dP: N = 64 keys
      constexpr uint32_t kIdQ = idesc_bf16_f32(kM, kD, false, true);      // dQ: K as MN-major B
      const uint32_t q_addr = smem_u32(sm + Q_OFF_Q), do_addr = smem_u32(sm + Q_OFF_DO);
      bool ok = mbar_wait(qd_full, 0, abort_flag);
      if (ok) tc_fence_after();
      for (int n = 0; ok && n <= nb; ++n) {
        if (n < nb) {
          const int st = n % kStages, bb = n & 1;
          if (!mbar_wait(kv_full + st, (n / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + Q_OFF_KV + st * kStageBytes);
          const uint32_t v_addr = k_addr + 2 * kKVHalf;
          const uint32_t d_s = tmem + 128 + bb * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ao = (kk >> 2) * kHalf + (kk & 3) * 32;
            const uint32_t bo = (kk >> 2) * kKVHalf + (kk & 3) * 32;
            mma_bf16_ss(d_s, sdesc_sw128(q_addr + ao, 16, 1024), sdesc_sw128(k_addr + bo, 16, 1024),
                        kIdS, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ao = (kk >> 2) * kHalf + (kk & 3) * 32;
            const uint32_t bo = (kk >> 2) * kKVHalf + (kk & 3) * 32;
            mma_bf16_ss(d_s + 64, sdesc_sw128(do_addr + ao, 16, 1024),
                        sdesc_sw128(v_addr + bo, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full + bb);
        }
        if (n >= 1) {
          const int m = n - 1, mb = m & 1, st = m % kStages;
          if (!mbar_wait(ds_full + mb, (m >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ds_addr = smem_u32(sm + Q_OFF_DS + mb * kTileBytes);
          const uint32_t k_addr = smem_u32(sm + Q_OFF_KV + st * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem, sdesc_sw128(ds_addr + kk * 32, 16, 1024),
                        sdesc_sw128(k_addr + kk * 2048, kKVHalf, 1024), kIdQ,
                        (m > 0 || kk > 0) ? 1u : 0u);
          tc_commit(ds_free + mb);
          tc_commit(kv_empty + st);
        }
      }
      if (!ok) tc_fail(a.err, 12, abort_flag);
      tc_commit(dq_final);
      mbar_wait_drain(dq_final, 0);
    }
  } else if (warp >= 4) {   // dS warpgroup wg takes the union blocks n = wg, wg+2, ...
    const int wg = (warp - 4) >> 2;
    const int r = tid - 128 - wg * 128;   // TMEM lane r = query row r
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int tl = r / G, g = r - tl * G;
    const bool valid = r < G * nt;
    const int t = t0 + tl;
    const int ct = t / kB;
    const int32_t* my_idx = sel_idx + tl * K1;
    const float* my_lg = sel_lg + tl * K1;
    const size_t qrow = (size_t)(s0 + t) * a.Hq + kv * G + g;
    const float lse2 = valid ? a.lse[qrow] * kLog2e : 0.f;
    const float dd = valid ? a.drow[qrow] : 0.f;
    float* dl_row = a.dlogg + ((size_t)(s0 + t) * a.Hkv + kv) * K1;
    const bool leader = valid && g == 0;
    if (leader && wg == 0)
      for (int s = 0; s < K1; ++s)
        if (my_idx[s] < 0) dl_row[s] = 0.f;
    int sp = 0;
    bool ok = true;
    // After a failed wait a warp stops working but keeps iterating, so that the named
    // barrier below (G not dividing 32) is always reached by all four warps of the group.
    for (int n = wg; n < nb; n += 2) {
      const int bb = wg;
      const int j = list[n];
      float rsum = 0.f;
      bool hit = false;
      if (ok && !warp_wait(s_full + bb, (n >> 1) & 1, abort_flag)) ok = false;
      if (ok) {
        tc_fence_after();
        float bias = -INFINITY;
        if (valid) {
          while (sp < K1 && my_idx[sp] >= 0 && my_idx[sp] < j) ++sp;
          hit = sp < K1 && my_idx[sp] == j;
          if (hit) bias = my_lg[sp] * kLog2e;
        }
        uint32_t pk[kB / 2];
        if (__any_sync(0xffffffffu, hit)) {
          float s[kB], dp[kB];
          tmem_ld64(tmem + lane_addr + 128 + bb * 128, s);
          tmem_ld64(tmem + lane_addr + 128 + bb * 128 + 64, dp);
          const int limit = (j == ct) ? (t - j * kB) : (kB - 1);
          const float off = hit ? bias - lse2 : -INFINITY;   // P = 2^(s*scale + bias - lse)
#pragma unroll
          for (int c = 0; c < kB; c += 2) {
            const float p0 = (c <= limit) ? ex2_approx(fmaf(s[c], a.scale_log2, off)) : 0.f;
            const float p1 = (c + 1 <= limit) ? ex2_approx(fmaf(s[c + 1], a.scale_log2, off)) : 0.f;
            const float d0 = p0 * (dp[c] - dd), d1 = p1 * (dp[c + 1] - dd);
            rsum += d0 + d1;
            pk[c >> 1] = pack_bf16x2(d0, d1);
          }
        } else {   // no row of this warp kept block j: its dS rows are zero
#pragma unroll
          for (int c = 0; c < kB / 2; ++c) pk[c] = 0u;
        }
        if (n >= 2 && !warp_wait(ds_free + bb, ((n - 2) >> 1) & 1, abort_flag)) ok = false;
        if (ok) {
          const uint32_t prow = smem_u32(sm + Q_OFF_DS + bb * kTileBytes) + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(prow + ((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                         pk[4 * c + 3]);
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(ds_full + bb);
        }
      }
      // dlogg of this block: the row sums of dS over the G heads of the token
      if ((32 % G) == 0) {
        for (int off = 1; off < G; off <<= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, off);
        if (ok && leader && hit) dl_row[sp] = rsum;
      } else {
        float* rsb = rs + (wg * 2 + ((n >> 1) & 1)) * 128;   // double-buffered per group
        rsb[r] = rsum;
        named_bar(1 + wg, 128);
        if (ok && leader && hit) {
          float tot = 0.f;
          for (int u = 0; u < G; ++u) tot += rsb[tl * G + u];
          dl_row[sp] = tot;
        }
      }
    }
    if (ok) ok = warp_wait(dq_final, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* orow = a.dq + qrow * kD;
#pragma unroll 1
      for (int c0 = wg * 64; c0 < wg * 64 + 64; c0 += 32) {   // each group: half the columns
        float ov[32];
        tmem_ld32(tmem + lane_addr + c0, ov);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(ov[2 * i] * a.scale, ov[2 * i + 1] * a.scale);
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    } else {
      tc_fail(a.err, 13, abort_flag);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------
// key-major pass over gathered rows: dK and dV of a pair of KV blocks
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(tcb::kGThreads, 1)
    attn_bwd_dkdv_gather_kernel(const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmV, const TcBwdArgs a) {
  using namespace tcb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.x, b = blockIdx.y, kv = blockIdx.z;
  const int s0 = a.cu[b], L = a.cu[b + 1] - s0;
  const int j0 = 2 * pair, key0 = j0 * kB;
  if (key0 >= L) return;
  const int G = a.G, K1 = a.K + 1, Mq = a.Mq;
  const int rows_used = G * Mq;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + G_OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* qd_full = bars + 1;
  uint64_t* st_full = bars + 2;
  uint64_t* pt_full = bars + 3;
  uint64_t* dkv_done = bars + 4;
  uint64_t* dkv_final = bars + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + G_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + G_OFF_MISC + 4);
  int* n_tok_s = reinterpret_cast<int*>(sm + G_OFF_MISC + 8);
  float* rc = reinterpret_cast<float*>(sm + G_OFF_RC);          // [2][4][128]
  uint32_t* words = reinterpret_cast<uint32_t*>(sm + G_OFF_WORDS);
  int* prefix = reinterpret_cast<int*>(sm + G_OFF_PREFIX);
  int* part = reinterpret_cast<int*>(sm + G_OFF_PART);

  // ---- token list of this (kv, pair): tokens >= key0 of the pair's bitmask row ----
  const int w0 = key0 >> 5, w1 = (L + 31) >> 5;
  const int nw = min(w1 - w0, kMaxWords);
  const uint32_t* mrow = a.pmask + ((size_t)(b * a.Hkv + kv) * a.NP + pair) * a.W + w0;
  const int per = (nw + kGThreads - 1) / kGThreads;
  int cnt = 0;
  for (int i = tid * per; i < min(nw, (tid + 1) * per); ++i) {
    const uint32_t w = mrow[i];
    words[i] = w;
    cnt += __popc(w);
  }
  part[tid] = cnt;
  if (tid == 0) {
    for (int i = 0; i < G_NBARS; ++i) mbar_init(bars + i, (i == 1 || i == 3) ? 128 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int i = 0; i < kGThreads; ++i) {
      const int c = part[i];
      part[i] = run;
      run += c;
    }
    *n_tok_s = run;
  }
  __syncthreads();
  {
    int run = part[tid];
    for (int i = tid * per; i < min(nw, (tid + 1) * per); ++i) {
      prefix[i] = run;
      run += __popc(words[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int n_tok = *n_tok_s;
  const int n_tiles = (n_tok + Mq - 1) / Mq;
  const uint32_t tmem = *tmem_slot;
  constexpr int kColDV = 0, kColDK = 128, kColST = 256, kColDPT = 384;

  if (warp < 4) {   // gather: thread r builds row r of every tile
    const int r = tid;
    const int tl = r / G, g = r - tl * G;
    const uint32_t q_dst = smem_u32(sm + G_OFF_Q) + r * 128;
    const uint32_t do_dst = smem_u32(sm + G_OFF_DO) + r * 128;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int rank = i * Mq + tl;
      const bool valid = r < rows_used && rank < n_tok;
      int t = -1;
      if (valid) {   // the rank-th set bit of the row
        int lo = 0, hi = nw - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (prefix[mid] <= rank) lo = mid; else hi = mid - 1;
        }
        uint32_t bits = words[lo];
        for (int k = rank - prefix[lo]; k > 0; --k) bits &= bits - 1u;
        t = (w0 + lo) * 32 + (__ffs(bits) - 1);
      }
      // row constants: c1 = log-gate - lse (log2 units) per block of the pair, D, position
      float c10 = -INFINITY, c11 = -INFINITY, dd = 0.f;
      int pos = -1;
      size_t qrow = 0;
      if (valid) {
        pos = t;
        qrow = (size_t)(s0 + t) * a.Hq + kv * G + g;
        const float l2 = a.lse[qrow] * kLog2e;
        dd = a.drow[qrow];
        const size_t irow = ((size_t)(s0 + t) * a.Hkv + kv) * K1;
        for (int s = 0; s < K1; ++s) {
          const int jj = a.idx[irow + s];
          if (jj < 0 || jj > j0 + 1) break;
          if (jj == j0) c10 = a.logg[irow + s] * kLog2e - l2;
          if (jj == j0 + 1) c11 = a.logg[irow + s] * kLog2e - l2;
        }
      }
      if (i >= 1 && !mbar_wait(dkv_done, (i - 1) & 1, abort_flag)) {   // tiles free again
        tc_fail(a.err, 31, abort_flag);
        ok = false;
        break;
      }
      if (r < kM) {
        if (valid) {
          const __nv_bfloat16* qs = a.q + qrow * kD;
          const __nv_bfloat16* ds = a.dout + qrow * kD;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t off = (uint32_t)((c >> 3) * kHalf + (((c & 7) ^ (r & 7)) << 4));
            cp_async16(q_dst + off, qs + c * 8);
            cp_async16(do_dst + off, ds + c * 8);
          }
        } else {   // rows past the list: finite zeros (0 * garbage could be NaN in the MMAs)
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t off = (uint32_t)((c >> 3) * kHalf + (c & 7) * 16);
            st_shared_v4(q_dst + off, 0u, 0u, 0u, 0u);
            st_shared_v4(do_dst + off, 0u, 0u, 0u, 0u);
          }
        }
      }
      float* rcb = rc + (i & 1) * 4 * 128;
      rcb[r] = c10;
      rcb[128 + r] = c11;
      rcb[256 + r] = dd;
      rcb[384 + r] = __int_as_float(pos);
      cp_async_wait_all();
      fence_async_smem();
      mbar_arrive(qd_full);
    }
  } else if (warp == 4) {
    if (lane == 0 && n_tiles > 0) {   // K/V pair loads + MMA issue
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(kv_full, 8u * kKVHalf);
      for (int h = 0; h < 2; ++h)
        for (int jj = 0; jj < 2; ++jj) {
          tma_load_3d(sm + G_OFF_K + h * kHalf + jj * kKVHalf, &tmK, kv_full, 64 * h, kv,
                      s0 + key0 + jj * kB);
          tma_load_3d(sm + G_OFF_V + h * kHalf + jj * kKVHalf, &tmV, kv_full, 64 * h, kv,
                      s0 + key0 + jj * kB);
        }
      constexpr uint32_t kIdT = idesc_bf16_f32(kM, kM, false, false);   // S^T, dP^T
      constexpr uint32_t kIdG = idesc_bf16_f32(kM, kD, false, true);    // dV, dK: B MN-major
      const uint32_t k_addr = smem_u32(sm + G_OFF_K), v_addr = smem_u32(sm + G_OFF_V);
      const uint32_t q_addr = smem_u32(sm + G_OFF_Q), do_addr = smem_u32(sm + G_OFF_DO);
      const uint32_t pt_addr = smem_u32(sm + G_OFF_PT), dst_addr = smem_u32(sm + G_OFF_DST);
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      for (int i = 0; ok && i < n_tiles; ++i) {
        if (!mbar_wait(qd_full, i & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColST, sdesc_sw128(k_addr + o, 16, 1024),
                      sdesc_sw128(q_addr + o, 16, 1024), kIdT, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t o = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColDPT, sdesc_sw128(v_addr + o, 16, 1024),
                      sdesc_sw128(do_addr + o, 16, 1024), kIdT, kk > 0 ? 1u : 0u);
        }
        tc_commit(st_full);
        if (!mbar_wait(pt_full, i & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColDV, sdesc_sw128(pt_addr + ao, 16, 1024),
                      sdesc_sw128(do_addr + kk * 2048, kHalf, 1024), kIdG,
                      (i > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColDK, sdesc_sw128(dst_addr + ao, 16, 1024),
                      sdesc_sw128(q_addr + kk * 2048, kHalf, 1024), kIdG,
                      (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(dkv_done);
      }
      if (!ok) tc_fail(a.err, 32, abort_flag);
      tc_commit(dkv_final);
      mbar_wait_drain(dkv_final, 0);
      mbar_wait_drain(kv_full, 0);
    }
  } else if (warp >= 8) {   // thread k = TMEM lane k = key k of the pair
    const int k = tid - 256;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int kp = key0 + k;
    const int coff = (k >= kB) ? 128 : 0;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      if (!warp_wait(qd_full, i & 1, abort_flag)) { ok = false; break; }   // row constants ready
      if (!warp_wait(st_full, i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (i >= 1 && !warp_wait(dkv_done, (i - 1) & 1, abort_flag)) { ok = false; break; }
      const float* rcb = rc + (i & 1) * 4 * 128;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float sv[32], dv[32];
        tmem_ld32(tmem + lane_addr + kColST + cc * 32, sv);
        tmem_ld32(tmem + lane_addr + kColDPT + cc * 32, dv);
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int r = cc * 32 + c + u;
            const bool vis = kp <= __float_as_int(rcb[384 + r]);
            const float p = vis ? ex2_approx(fmaf(sv[c + u], a.scale_log2, rcb[coff + r])) : 0.f;
            p2[u] = p;
            d2[u] = vis ? p * (dv[c + u] - rcb[256 + r]) : 0.f;
          }
          pp[c >> 1] = pack_bf16x2(p2[0], p2[1]);
          pd[c >> 1] = pack_bf16x2(d2[0], d2[1]);
        }
        const int half = cc >> 1;
        const uint32_t rowp = smem_u32(sm + G_OFF_PT + half * kHalf) + k * 128;
        const uint32_t rowd = smem_u32(sm + G_OFF_DST + half * kHalf) + k * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (cc & 1) * 4 + q4;
          const uint32_t off = (uint32_t)((chunk ^ (k & 7)) << 4);
          st_shared_v4(rowp + off, pp[4 * q4], pp[4 * q4 + 1], pp[4 * q4 + 2], pp[4 * q4 + 3]);
          st_shared_v4(rowd + off, pd[4 * q4], pd[4 * q4 + 1], pd[4 * q4 + 2], pd[4 * q4 + 3]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(pt_full);
    }
    if (!ok) tc_fail(a.err, 33, abort_flag);
    const bool have = ok && n_tiles > 0 && warp_wait(dkv_final, 0, abort_flag);
    if (ok && n_tiles > 0 && !have) tc_fail(a.err, 34, abort_flag);
    // `have` and `n_tiles` are warp-uniform: the collective TMEM loads run on whole warps,
    // only the stores depend on the lane's key being inside the sequence.
    if (have || n_tiles == 0) {
      const bool store = kp < L;
      __nv_bfloat16* dkr = a.dk + ((size_t)(s0 + kp) * a.Hkv + kv) * kD;
      __nv_bfloat16* dvr = a.dv + ((size_t)(s0 + kp) * a.Hkv + kv) * kD;
      if (have) tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float kvv[32], vvv[32];
        if (have) {
          tmem_ld32(tmem + lane_addr + kColDK + c0, kvv);
          tmem_ld32(tmem + lane_addr + kColDV + c0, vvv);
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) kvv[u] = vvv[u] = 0.f;
        }
        if (!store) continue;
        uint32_t pk[16], pv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          pk[u] = pack_bf16x2(kvv[2 * u] * a.scale, kvv[2 * u + 1] * a.scale);
          pv[u] = pack_bf16x2(vvv[2 * u], vvv[2 * u + 1]);
        }
        uint4* dk4 = reinterpret_cast<uint4*>(dkr + c0);
        uint4* dv4 = reinterpret_cast<uint4*>(dvr + c0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          dk4[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          dv4[u] = make_uint4(pv[4 * u], pv[4 * u + 1], pv[4 * u + 2], pv[4 * u + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
bool attn_bwd_tc_supported(const sas_problem& p) {
  if (!attn_tc_supported(p)) return false;
  const int G = p.num_q_heads / p.num_kv_heads;
  const int Mq = tc_rows_per_tile(G);
  return Mq * (p.topk + 1) <= tcb::kMaxSel && (p.max_seqlen + 31) / 32 <= tcb::kMaxWords;
}

// bytes of the per-(kv, block pair) token bitmasks
size_t attn_bwd_tc_tmask_bytes(const sas_problem& p) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const size_t NP = (NBmax + 1) / 2, W = (p.max_seqlen + 31) / 32;
  return (size_t)p.batch * p.num_kv_heads * NP * W * 4;
}

sas_status launch_attn_bwd_tc(const sas_problem& p, const void* q, const void* k, const void* v,
                              const void* dout, const float* lse, const float* drow,
                              const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                              float* dlogg, uint32_t* tmask, int* err, cudaStream_t st) {
  const int G = p.num_q_heads / p.num_kv_heads;
  const int Mq = tc_rows_per_tile(G);
  CUtensorMap tq, tdo, tk, tv;
  if (!make_tmap_bf16_3d(&tq, q, 128, p.num_q_heads, p.total_tokens, 64, G, Mq) ||
      !make_tmap_bf16_3d(&tdo, dout, 128, p.num_q_heads, p.total_tokens, 64, G, Mq) ||
      !make_tmap_bf16_3d(&tk, k, 128, p.num_kv_heads, p.total_tokens, 64, 1, 64) ||
      !make_tmap_bf16_3d(&tv, v, 128, p.num_kv_heads, p.total_tokens, 64, 1, 64)) {
    set_error("attn_bwd: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  TcBwdArgs a;
  a.cu = p.cu_seqlens;
  a.idx = idx;
  a.logg = logg;
  a.lse = lse;
  a.drow = drow;
  a.pmask = tmask;
  a.q = (const __nv_bfloat16*)q;
  a.dout = (const __nv_bfloat16*)dout;
  a.dq = (__nv_bfloat16*)dq;
  a.dk = (__nv_bfloat16*)dk;
  a.dv = (__nv_bfloat16*)dv;
  a.dlogg = dlogg;
  a.err = err;
  a.Hq = p.num_q_heads;
  a.Hkv = p.num_kv_heads;
  a.G = G;
  a.K = p.topk;
  a.Mq = Mq;
  a.NBmax = (p.max_seqlen + p.block - 1) / p.block;
  a.n_tiles = (p.max_seqlen + Mq - 1) / Mq;
  a.NP = (a.NBmax + 1) / 2;
  a.W = (p.max_seqlen + 31) / 32;
  a.scale = 1.f / sqrtf(128.f);
  a.scale_log2 = kLog2e * a.scale;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tcb::Q_SMEM);
    cudaFuncSetAttribute(attn_bwd_dkdv_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tcb::G_SMEM);
  });
  if (cudaMemsetAsync(tmask, 0, attn_bwd_tc_tmask_bytes(p), st) != cudaSuccess) {
    set_error("attn_bwd: clearing the token bitmasks failed");
    return SAS_ERR_CUDA;
  }
  const int rows = p.total_tokens * p.num_kv_heads;
  pair_mask_kernel<<<(rows + 255) / 256, 256, 0, st>>>(idx, p.cu_seqlens, p.batch,
                                                        p.total_tokens, p.num_kv_heads, p.topk,
                                                        a.NP, a.W, tmask);
  attn_bwd_dq_tc_kernel<<<dim3(a.n_tiles, p.batch, p.num_kv_heads), tcb::kThreads, tcb::Q_SMEM,
                          st>>>(tq, tdo, tk, tv, a);
  attn_bwd_dkdv_gather_kernel<<<dim3(a.NP, p.batch, p.num_kv_heads), tcb::kGThreads, tcb::G_SMEM,
                                st>>>(tk, tv, a);
  return launch_status("attn_bwd (tensor cores)", 3);
}

}  // namespace sas
