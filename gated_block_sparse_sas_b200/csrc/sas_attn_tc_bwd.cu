// Tensor-core (tcgen05 / TMEM / TMA) backward of the gated sparse attention (A6), bf16,
// head_dim 128, KV block 64. The loss reaches the selector through standard
// backpropagation (paper abstract): besides dQ, dK, dV the backward returns the gradient
// of every kept block's log-gate, dlogg = sum over the G heads and the block's keys of
// dS = P (dP - D).
//
// Two passes over the same tile-union decomposition as the forward, so that no output is
// accumulated with atomics and every sum has a fixed order:
//   query-major  CTA = (tile of Mq tokens x G heads = 128 rows, kv head). Per union block:
//                S = Q K^T, dP = dO V^T (TMEM, double-buffered), dS = P (dP - D) in
//                registers -> bf16 shared tile, dQ += dS K (TMEM). Row sums of dS, reduced
//                over the G heads of a token, are that token's dlogg for the block.
//   key-major    CTA = (pair of KV blocks = 128 keys, kv head). For every tile whose union
//                holds either block (per-tile union bitmasks from a pre-pass): S^T = K Q^T,
//                dP^T = V dO^T (keys on TMEM lanes, rows on columns, so the per-row softmax
//                statistics are per-column constants), P^T and dS^T -> bf16 shared tiles,
//                dV += P^T dO, dK += dS^T Q (TMEM).
// D = rowsum(dO * O) comes from the CUDA-core row-dot kernel.
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace tcb {
constexpr int kD = 128, kB = 64, kM = 128, kThreads = 256;
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
constexpr int Q_OFF_RS = Q_OFF_MASK + kMaxBlocks / 8;          // 2 x 128 floats
constexpr int Q_OFF_BAR = Q_OFF_RS + 2 * 128 * 4;
constexpr int Q_NBARS = 1 + 2 * kStages + 2 + 2 + 2 + 1;
constexpr int Q_OFF_MISC = Q_OFF_BAR + Q_NBARS * 8;
constexpr int Q_SMEM = Q_OFF_MISC + 64 + 1024;
// key-major pass layout
constexpr int kMaxTiles = 4096;
constexpr int K_OFF_K = 0;                       // [128 keys][128 d] as 2 halves
constexpr int K_OFF_V = K_OFF_K + 2 * kHalf;
constexpr int K_OFF_Q = K_OFF_V + 2 * kHalf;     // [128 rows][128 d]
constexpr int K_OFF_DO = K_OFF_Q + 2 * kHalf;
constexpr int K_OFF_PT = K_OFF_DO + 2 * kHalf;   // P^T  [128 keys][128 rows] as 2 halves
constexpr int K_OFF_DST = K_OFF_PT + 2 * kHalf;  // dS^T [128 keys][128 rows]
constexpr int K_OFF_TL = K_OFF_DST + 2 * kHalf;
constexpr int K_OFF_RC = K_OFF_TL + kMaxTiles * 4;     // 2 x 5 x 128 floats
constexpr int K_OFF_CNT = K_OFF_RC + 2 * 5 * 128 * 4;
constexpr int K_OFF_BAR = K_OFF_CNT + 16 * 4;
constexpr int K_NBARS = 6;
constexpr int K_OFF_MISC = K_OFF_BAR + K_NBARS * 8;
constexpr int K_SMEM = K_OFF_MISC + 64 + 1024;
}  // namespace tcb

struct TcBwdArgs {
  const int32_t* cu;
  const int32_t* idx;
  const float* logg;
  const float* lse;
  const float* drow;
  const uint32_t* tmask;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dlogg;
  int* err;
  int Hq, Hkv, G, K, Mq, NBmax, n_tiles;
  float scale_log2, scale;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
}

// ---------------------------------------------------------------------------------------
// pre-pass: union bitmask of every (tile, kv head) -> tmask[b][tile][kv][word]
// ---------------------------------------------------------------------------------------
__global__ void tile_union_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cu,
                                  int Hkv, int K, int Mq, int NBmax, int n_tiles,
                                  uint32_t* __restrict__ tmask) {
  __shared__ uint32_t words[tcb::kMaxBlocks / 32];
  const int tile = blockIdx.x, b = blockIdx.y, kv = blockIdx.z;
  const int nwords = (NBmax + 31) >> 5;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) words[w] = 0u;
  __syncthreads();
  const int s0 = cu[b], L = cu[b + 1] - s0, t0 = tile * Mq, K1 = K + 1;
  if (t0 < L) {
    const int nt = min(Mq, L - t0);
    for (int e = threadIdx.x; e < nt * K1; e += blockDim.x) {
      const int tl = e / K1, sl = e - tl * K1;
      const int j = idx[((size_t)(s0 + t0 + tl) * Hkv + kv) * K1 + sl];
      if (j >= 0 && j < NBmax) atomicOr(&words[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  uint32_t* out = tmask + (((size_t)b * n_tiles + tile) * Hkv + kv) * nwords;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) out[w] = words[w];
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
  } else if (warp >= 4) {   // dS warpgroup: thread r = TMEM lane r = query row r
    const int r = tid - 128;
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
    if (leader)
      for (int s = 0; s < K1; ++s)
        if (my_idx[s] < 0) dl_row[s] = 0.f;
    int sp = 0;
    bool ok = true;
    // After a failed wait a warp stops working but keeps iterating, so that the named
    // barrier below (G not dividing 32) is always reached by all four warps.
    for (int n = 0; n < nb; ++n) {
      const int bb = n & 1;
      const int j = list[n];
      float rsum = 0.f;
      bool hit = false;
      if (ok && !warp_wait(s_full + bb, (n >> 1) & 1, abort_flag)) ok = false;
      if (ok) {
        tc_fence_after();
        float s[kB], dp[kB];
        tmem_ld32(tmem + lane_addr + 128 + bb * 128, s);
        tmem_ld32(tmem + lane_addr + 128 + bb * 128 + 32, s + 32);
        tmem_ld32(tmem + lane_addr + 128 + bb * 128 + 64, dp);
        tmem_ld32(tmem + lane_addr + 128 + bb * 128 + 96, dp + 32);
        float bias = -INFINITY;
        if (valid) {
          while (sp < K1 && my_idx[sp] >= 0 && my_idx[sp] < j) ++sp;
          hit = sp < K1 && my_idx[sp] == j;
          if (hit) bias = my_lg[sp] * kLog2e;
        }
        const int limit = (j == ct) ? (t - j * kB) : (kB - 1);
        uint32_t pk[kB / 2];
#pragma unroll
        for (int c = 0; c < kB; c += 2) {
          const float x0 = (c <= limit) ? fmaf(s[c], a.scale_log2, bias) : -INFINITY;
          const float x1 = (c + 1 <= limit) ? fmaf(s[c + 1], a.scale_log2, bias) : -INFINITY;
          const float p0 = exp2f(x0 - lse2), p1 = exp2f(x1 - lse2);
          const float d0 = p0 * (dp[c] - dd), d1 = p1 * (dp[c + 1] - dd);
          rsum += d0 + d1;
          pk[c >> 1] = pack_bf16x2(d0, d1);
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
        rs[bb * 128 + r] = rsum;
        named_bar(1, 128);
        if (ok && leader && hit) {
          float tot = 0.f;
          for (int u = 0; u < G; ++u) tot += rs[bb * 128 + tl * G + u];
          dl_row[sp] = tot;
        }
      }
    }
    if (ok) ok = warp_wait(dq_final, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* orow = a.dq + qrow * kD;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
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
// key-major pass: dK and dV of a pair of KV blocks
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(tcb::kThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                            const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const TcBwdArgs a) {
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
  const int nwords = (a.NBmax + 31) >> 5;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + K_OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* qd_full = bars + 1;
  uint64_t* st_full = bars + 2;
  uint64_t* pt_full = bars + 3;
  uint64_t* dkv_done = bars + 4;
  uint64_t* dkv_final = bars + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + K_OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + K_OFF_MISC + 4);
  int* n_list_s = reinterpret_cast<int*>(sm + K_OFF_MISC + 8);
  int32_t* tlist = reinterpret_cast<int32_t*>(sm + K_OFF_TL);
  float* rc = reinterpret_cast<float*>(sm + K_OFF_RC);   // [2][5][128]
  int* wcnt = reinterpret_cast<int*>(sm + K_OFF_CNT);

  if (tid == 0) {
    for (int i = 0; i < K_NBARS; ++i) mbar_init(bars + i, i == 3 ? 128 : 1);
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
      reinterpret_cast<uint4*>(sm + K_OFF_Q + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + K_OFF_Q + kHalf + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + K_OFF_DO + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + K_OFF_DO + kHalf + r * 128)[c] = z;
    }
    fence_async_smem();
  }
  // ordered list of the tiles whose union holds block j0 or j0+1 (tiles ending before key0 skipped)
  const int n_seq_tiles = (L + Mq - 1) / Mq;
  const int first_tile = key0 / Mq;
  const uint32_t want = 3u << (j0 & 31);
  int n_list = 0;
  for (int c0 = first_tile; c0 < n_seq_tiles; c0 += kThreads) {
    const int tt = c0 + tid;
    bool hit = false;
    if (tt < n_seq_tiles)
      hit = (a.tmask[(((size_t)b * a.n_tiles + tt) * a.Hkv + kv) * nwords + (j0 >> 5)] & want) != 0u;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) wcnt[warp] = __popc(m);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      if (w < warp) before += wcnt[w];
      total += wcnt[w];
    }
    if (hit) {
      const int pos = n_list + before + __popc(m & ((1u << lane) - 1u));
      if (pos < kMaxTiles) tlist[pos] = tt;
    }
    n_list += total;
    __syncthreads();
  }
  if (tid == 0) *n_list_s = min(n_list, kMaxTiles);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int ntl = *n_list_s;
  const uint32_t tmem = *tmem_slot;
  constexpr int kColDV = 0, kColDK = 128, kColST = 256, kColDPT = 384;

  if (warp == 0) {
    if (lane == 0 && ntl > 0) {   // producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmDO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(kv_full, 8u * kKVHalf);
      for (int h = 0; h < 2; ++h)
        for (int jj = 0; jj < 2; ++jj) {
          tma_load_3d(sm + K_OFF_K + h * kHalf + jj * kKVHalf, &tmK, kv_full, 64 * h, kv,
                      s0 + key0 + jj * kB);
          tma_load_3d(sm + K_OFF_V + h * kHalf + jj * kKVHalf, &tmV, kv_full, 64 * h, kv,
                      s0 + key0 + jj * kB);
        }
      int issued = 0;
      for (int i = 0; i < ntl; ++i) {
        if (i >= 1 && !mbar_wait(dkv_done, (i - 1) & 1, abort_flag)) {
          tc_fail(a.err, 21, abort_flag);
          break;
        }
        const int trow = s0 + tlist[i] * Mq;
        mbar_arrive_expect_tx(qd_full, 4u * rows_used * 128u);
        tma_load_3d(sm + K_OFF_Q, &tmQ, qd_full, 0, kv * G, trow);
        tma_load_3d(sm + K_OFF_Q + kHalf, &tmQ, qd_full, 64, kv * G, trow);
        tma_load_3d(sm + K_OFF_DO, &tmDO, qd_full, 0, kv * G, trow);
        tma_load_3d(sm + K_OFF_DO + kHalf, &tmDO, qd_full, 64, kv * G, trow);
        issued = i + 1;
      }
      mbar_wait_drain(kv_full, 0);
      if (issued > 0) mbar_wait_drain(qd_full, (issued - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && ntl > 0) {   // MMA issuer
      constexpr uint32_t kIdT = idesc_bf16_f32(kM, kM, false, false);   // S^T, dP^T: N = 128 rows
      constexpr uint32_t kIdG = idesc_bf16_f32(kM, kD, false, true);    // dV, dK: B MN-major
      const uint32_t k_addr = smem_u32(sm + K_OFF_K), v_addr = smem_u32(sm + K_OFF_V);
      const uint32_t q_addr = smem_u32(sm + K_OFF_Q), do_addr = smem_u32(sm + K_OFF_DO);
      const uint32_t pt_addr = smem_u32(sm + K_OFF_PT), dst_addr = smem_u32(sm + K_OFF_DST);
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      for (int i = 0; ok && i < ntl; ++i) {
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
          // dO / Q as MN-major B: 16 rows (K) per step, 64-column halves kHalf apart
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
      if (!ok) tc_fail(a.err, 22, abort_flag);
      tc_commit(dkv_final);
      mbar_wait_drain(dkv_final, 0);
    }
  } else if (warp >= 4) {   // thread k = TMEM lane k = key k of the pair
    const int k = tid - 128;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int kp = key0 + k;                       // in-sequence key position
    const bool second = k >= kB;
    bool ok = true;
    // After a failed wait a warp stops working but keeps iterating, so that every warp
    // reaches every named barrier.
    for (int i = 0; i < ntl; ++i) {
      // per-row constants of tile i (thread k handles row k): bias for j0 / j0+1, lse, D, pos
      float* rcb = rc + (i & 1) * 5 * 128;
      {
        const int r = k, tl = r / G, g = r - tl * G;
        const int tt0 = tlist[i] * Mq;
        const int ntt = min(Mq, L - tt0);
        float b0 = -INFINITY, b1 = -INFINITY, l2 = 0.f, dd = 0.f;
        int pos = -1;
        if (r < G * ntt) {
          const int t = tt0 + tl;
          pos = t;
          const size_t qrow = (size_t)(s0 + t) * a.Hq + kv * G + g;
          l2 = a.lse[qrow] * kLog2e;
          dd = a.drow[qrow];
          const size_t irow = ((size_t)(s0 + t) * a.Hkv + kv) * K1;
          for (int s = 0; s < K1; ++s) {
            const int jj = a.idx[irow + s];
            if (jj < 0 || jj > j0 + 1) break;
            if (jj == j0) b0 = a.logg[irow + s] * kLog2e;
            if (jj == j0 + 1) b1 = a.logg[irow + s] * kLog2e;
          }
        }
        rcb[r] = b0;
        rcb[128 + r] = b1;
        rcb[256 + r] = l2;
        rcb[384 + r] = dd;
        rcb[512 + r] = __int_as_float(pos);
      }
      named_bar(1, 128);
      if (ok && !warp_wait(st_full, i & 1, abort_flag)) ok = false;
      if (ok) tc_fence_after();
      if (ok && i >= 1 && !warp_wait(dkv_done, (i - 1) & 1, abort_flag)) ok = false;
      if (!ok) continue;
      const float* bsel = rcb + (second ? 128 : 0);
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
            const float bias = bsel[r];
            const bool vis = kp <= __float_as_int(rcb[512 + r]);
            const float x = vis ? fmaf(sv[c + u], a.scale_log2, bias) : -INFINITY;
            const float p = exp2f(x - rcb[256 + r]);
            p2[u] = p;
            d2[u] = p * (dv[c + u] - rcb[384 + r]);
          }
          pp[c >> 1] = pack_bf16x2(p2[0], p2[1]);
          pd[c >> 1] = pack_bf16x2(d2[0], d2[1]);
        }
        // element (key k, row r): half r/64, 16-byte chunk (r%64)/8, 128B swizzle by k
        const int half = cc >> 1;
        const uint32_t rowp = smem_u32(sm + K_OFF_PT + half * kHalf) + k * 128;
        const uint32_t rowd = smem_u32(sm + K_OFF_DST + half * kHalf) + k * 128;
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
    if (!ok) tc_fail(a.err, 23, abort_flag);
    const bool have = ok && ntl > 0 && warp_wait(dkv_final, 0, abort_flag);
    if (ok && ntl > 0 && !have) tc_fail(a.err, 24, abort_flag);
    // `have` and `ntl` are warp-uniform, so the collective TMEM loads below run on whole
    // warps; only the stores depend on the lane's key being inside the sequence.
    if (have || ntl == 0) {
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
  if (warp == 1) {
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
  return Mq * (p.topk + 1) <= tcb::kMaxSel && (p.max_seqlen + Mq - 1) / Mq <= tcb::kMaxTiles;
}

size_t attn_bwd_tc_tmask_bytes(const sas_problem& p) {
  const int G = p.num_q_heads / p.num_kv_heads;
  const int Mq = tc_rows_per_tile(G);
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  const size_t n_tiles = (p.max_seqlen + Mq - 1) / Mq;
  return (size_t)p.batch * n_tiles * p.num_kv_heads * ((NBmax + 31) / 32) * 4;
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
  a.tmask = tmask;
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
  a.scale = 1.f / sqrtf(128.f);
  a.scale_log2 = kLog2e * a.scale;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tcb::Q_SMEM);
    cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tcb::K_SMEM);
  });
  tile_union_kernel<<<dim3(a.n_tiles, p.batch, p.num_kv_heads), 128, 0, st>>>(
      idx, p.cu_seqlens, p.num_kv_heads, p.topk, Mq, a.NBmax, a.n_tiles, tmask);
  attn_bwd_dq_tc_kernel<<<dim3(a.n_tiles, p.batch, p.num_kv_heads), tcb::kThreads, tcb::Q_SMEM,
                          st>>>(tq, tdo, tk, tv, a);
  const int n_pairs = (a.NBmax + 1) / 2;
  attn_bwd_dkdv_tc_kernel<<<dim3(n_pairs, p.batch, p.num_kv_heads), tcb::kThreads, tcb::K_SMEM,
                            st>>>(tq, tdo, tk, tv, a);
  return launch_status("attn_bwd (tensor cores)", 3);
}

}  // namespace sas
