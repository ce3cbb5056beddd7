// Key-major tensor-core forward of the gated sparse attention (A5), bf16, head_dim 128, KV
// block 64.
//
// Every query token keeps its own K+1 blocks (README (b)), so the rows of a query tile share
// few blocks and a query-major tile computes mostly masked scores. This pass turns the
// selection around. A work item is one KV block j of one KV head of one sequence together
// with the query rows, inside one window of 4096 tokens, that kept j. Those rows are gathered
// into 128-row tiles (Mq tokens x the G heads of the KV head) and every MMA row is attended:
//   S = Q K_j^T (M=128, N=64, K=128)
//   P = 2^(S * log2e/sqrt(d) + log2e * log g_j - m_row)   (causal mask inside the current block)
//   O_part = P V_j (M=128, N=128, K=64),  l_part = row sum of P (fp32, before rounding)
// O_part and l_part are added into fp32 accumulators with L2 reductions. Splitting the
// softmax sums over blocks this way is exact regrouping because each row uses ONE reference
// m_row for all of its blocks (abstract: the gate enters the softmax in log form, so a
// row's logits are z = q.k/sqrt(d) + log g whatever block they come from):
//   m_row = (logit of the row's own key) + 32, in log2 units.
// The own key t is always visible (current block, always kept), so the row maximum is at
// least m_row - 32 and no block's contribution that matters can underflow. A row whose maximum
// logit exceeds its own-key logit by more than about 140 log2 units (~97 nats) would overflow
// fp32; the finishing pass reports that through the error word.
// The finishing pass writes O = O_acc / l and LSE = (m_row + log2 l) ln 2. Summation order of
// the reductions is not fixed, so results can differ in the last fp32 bits from run to run.
//
// Preparation (device only, no host synchronisation): m_row per (token, query head), and
// the inverted selection lists (sas_km.cuh).
//
// Main kernel: persistent, one CTA per SM; items are taken in ascending order from an atomic
// counter, so the CTAs work on neighbouring windows and the accumulator rows they update stay
// in L2. Warp roles (512 threads):
//   warps 0-3   gather. Thread r builds row r of each tile: list entry -> token and log-gate,
//               m_row, the Q row by cp.async into a 128B-swizzled K-major tile (2 stages),
//               row constants (bias, causal limit, destination row) into a 4-slot ring.
//               Thread 0 fetches items and loads each item's K/V block by TMA (2 stages).
//   warp 4      TMEM allocation; lane 0 issues the MMAs, S of tile n before PV of tile n-1.
//   warps 8-11  softmax: TMEM lane r = tile row r; P as bf16 pairs over its S columns,
//               l_part into a TMEM column once the epilogue has released tile n-2.
//   warps 12-15 epilogue: O_part and l_part out of TMEM; thread r writes row r to a shared
//               buffer and hands it to the TMA unit as one 512-byte bulk fp32 reduction
//               (cp.reduce.async.bulk .add.f32) into O_acc.
// Every wait is bounded; a timeout records an error code in the workspace and all roles
// wind down (copies drained, MMAs completed, TMEM released).
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_km.cuh"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace kmf {
constexpr int kD = 128, kB = 64, kM = 128;
constexpr int kThreads = 512;
constexpr float kRefShift = 32.f;        // m_row = own-key logit + 32 (log2 units)
constexpr int kKVHalf = kB * 128;        // [64 keys][64 d] bf16, 128B rows: 8 KB
constexpr int kKVStage = 4 * kKVHalf;    // K0 K1 V0 V1
constexpr int kQHalf = kM * 128;         // [128 rows][64 d]: 16 KB
constexpr int kQStage = 2 * kQHalf;
constexpr int kEpiStride = 132;          // floats per row of the epilogue buffer (528 B)
constexpr int OFF_KV = 0;
constexpr int OFF_Q = OFF_KV + 2 * kKVStage;
constexpr int OFF_EPI = OFF_Q + 2 * kQStage;                   // [4 warps][32][132] fp32
constexpr int OFF_RC = OFF_EPI + 4 * 32 * kEpiStride * 4;      // [4 slots][3][128]
constexpr int OFF_HDR = OFF_RC + 4 * 3 * kM * 4;               // [4 slots][2] int
constexpr int OFF_BAR = OFF_HDR + 4 * 2 * 4;
constexpr int kNumBars = 2 + 2 + 2 + 2 + 4 + 4 + 2 + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
// TMEM columns: S0 0..63, S1 64..127 (P as bf16 pairs over the first 32 columns of its S),
// O0 128..255, O1 256..383, l_part of buffer b in column 384 + b
constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0, kColO = 128, kColL = 384;
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagStop = 4;
}  // namespace kmf

struct KmFwdArgs {
  const int32_t* cu;
  const __nv_bfloat16* q;
  const int2* list;        // (token | slot << 24, log-gate bits) grouped by item
  const int32_t* cnt;      // per entry
  const int32_t* off;      // per entry
  const int32_t* items;    // non-empty entries, ascending
  const int32_t* ctl;      // [0] = number of items
  int* next_item;
  const float* mref;
  float* oacc;             // [T][Hq][128]
  float* lacc;             // [T][Hq]
  int* err;
  int batch, Hq, Hkv, G, Mq, P;
  int R;                   // gate heads per KV head (1, or G with one gate per query head)
  float scale_log2;
};

// ---------------------------------------------------------------------------------------
// preparation
// ---------------------------------------------------------------------------------------
// m_row = (q_t,h . k_t,kv / sqrt(d) + log g_current) log2e + 32; one warp per (token, gate
// head): the gate head's G query heads (G = Hq / Hs here), keys of KV head kv / R
__global__ void km_rowref_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                 const int32_t* __restrict__ idx, const float* __restrict__ logg,
                                 const int32_t* __restrict__ cu, int batch, int T, int Hq, int Hkv,
                                 int R, int G, int K, float scale_log2, float* __restrict__ mref) {
  const int lane = threadIdx.x & 31;
  const int gw = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  if (gw >= T * Hkv) return;
  const int tg = gw / Hkv, kv = gw - tg * Hkv;   // Hkv counts gate heads here
  const int Hk = Hkv / R, kh = kv / R;
  const int b = seq_of(cu, batch, tg);
  const int c = (tg - cu[b]) / kmf::kB;
  const size_t irow = (size_t)gw * (K + 1);
  float lg = 0.f;
  for (int s0 = 0; s0 <= K; s0 += 32) {
    const int s = s0 + lane;
    const bool hit = s <= K && idx[irow + s] == c;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      const float v = hit ? logg[irow + s] : 0.f;
      lg = __shfl_sync(0xffffffffu, v, src);
      break;
    }
  }
  const uint2 kr = *reinterpret_cast<const uint2*>(k + ((size_t)tg * Hk + kh) * kmf::kD + lane * 4);
  const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.x));
  const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.y));
  for (int g = 0; g < G; ++g) {
    const size_t row = (size_t)tg * Hq + kv * G + g;
    const uint2 qr = *reinterpret_cast<const uint2*>(q + row * kmf::kD + lane * 4);
    const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr.x));
    const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr.y));
    const float dot = warp_sum(q01.x * k01.x + q01.y * k01.y + q23.x * k23.x + q23.y * k23.y);
    if (lane == 0) mref[row] = fmaf(dot, scale_log2, lg * kLog2e) + kmf::kRefShift;
  }
}

// O = O_acc / l (bf16), LSE = (m_row + log2 l) ln 2; one warp per (token, query head).
__global__ void km_finalize_kernel(const float* __restrict__ oacc, const float* __restrict__ lacc,
                                   const float* __restrict__ mref, int rows,
                                   __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                   int* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  if (row >= rows) return;
  const float l = lacc[row];
  const bool good = l > 0.f && isfinite(l);
  const float inv = good ? 1.f / l : 0.f;
  const float4 x = reinterpret_cast<const float4*>(oacc + (size_t)row * kmf::kD)[lane];
  uint2 pk = make_uint2(0u, 0u);   // a row outside the reference's range (error 60) is 0
  if (good) {
    pk.x = pack_bf16x2(x.x * inv, x.y * inv);
    pk.y = pack_bf16x2(x.z * inv, x.w * inv);
  }
  reinterpret_cast<uint2*>(o + (size_t)row * kmf::kD)[lane] = pk;
  if (lane == 0) {
    lse[row] = good ? (mref[row] + log2f(l)) * kLn2 : -INFINITY;
    if (!good) atomicCAS(err, 0, 60);
  }
}

// ---------------------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kmf::kThreads, 1)
    attn_fwd_km_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const KmFwdArgs a) {
  using namespace kmf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, Mq = a.Mq;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 2;
  uint64_t* q_full = bars + 4;
  uint64_t* q_empty = bars + 6;
  uint64_t* rc_full = bars + 8;
  uint64_t* rc_empty = bars + 12;
  uint64_t* s_full = bars + 16;
  uint64_t* p_full = bars + 18;
  uint64_t* o_full = bars + 20;
  uint64_t* o_empty = bars + 22;
  uint64_t* final_bar = bars + 24;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(sm + OFF_MISC + 8);
  float* rcf = reinterpret_cast<float*>(sm + OFF_RC);   // slot s: bias [128], limit [128], dst [128]
  int* rci = reinterpret_cast<int*>(sm + OFF_RC);
  int* hdr = reinterpret_cast<int*>(sm + OFF_HDR);      // slot s: flags, K/V stage

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
      mbar_init(q_full + i, 128);
      mbar_init(q_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 128);
      mbar_init(o_full + i, 1);
      mbar_init(o_empty + i, 128);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(rc_full + i, 128);
      mbar_init(rc_empty + i, 128);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = a.ctl[0];

  if (warp < 4) {
    // ------------------------------ gather ------------------------------
    const int r = tid;
    const int tl = r / G, g = r - tl * G;
    const bool row_ok = r < G * Mq;
    bool ok = true;
    int n = 0, item_seq = 0;
    if (r == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    while (true) {
      if (r == 0) bcast[0] = atomicAdd(a.next_item, 1);
      named_bar(1, 128);
      const int it = bcast[0];
      const bool stop = *abort_flag != 0 || it >= n_items;
      named_bar(1, 128);   // every thread has read bcast before thread 0 rewrites it
      if (stop) break;
      const int e = a.items[it];
      const int cnt = a.cnt[e], off = a.off[e];
      const km::Item itm = km::decode(e, a.batch, a.P);
      const int kv = itm.kv, b = itm.b, j = itm.j;
      const int s0 = a.cu[b];
      const int kvs = item_seq & 1;
      if (r == 0 && ok) {   // this item's K/V block
        if (item_seq >= 2 && !mbar_wait(kv_empty + kvs, ((item_seq >> 1) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 51, abort_flag);
          ok = false;
        } else {
          uint8_t* stg = sm + OFF_KV + kvs * kKVStage;
          const int row = s0 + j * kB;
          mbar_arrive_expect_tx(kv_full + kvs, kKVStage);
          const int kh = kv / a.R;   // the item's gate head reads KV head kh
          tma_load_3d(stg, &tmK, kv_full + kvs, 0, kh, row);
          tma_load_3d(stg + kKVHalf, &tmK, kv_full + kvs, 64, kh, row);
          tma_load_3d(stg + 2 * kKVHalf, &tmV, kv_full + kvs, 0, kh, row);
          tma_load_3d(stg + 3 * kKVHalf, &tmV, kv_full + kvs, 64, kh, row);
        }
      }
      ++item_seq;
      const int ntile = (cnt + Mq - 1) / Mq;
      const int jk0 = j * kB;
      int2 nxt = make_int2(0, 0);
      if (row_ok && tl < cnt) nxt = a.list[off + tl];
      for (int m = 0; m < ntile; ++m, ++n) {
        const int rank = m * Mq + tl;
        const bool valid = row_ok && rank < cnt;
        const int2 ent = nxt;
        if (row_ok && rank + Mq < cnt) nxt = a.list[off + rank + Mq];   // next tile's entry
        const int tg = ent.x & 0xFFFFFF;
        const size_t qrow = (size_t)tg * a.Hq + kv * G + g;
        const float mr = valid ? a.mref[qrow] : 0.f;
        const int qs = n & 1, rs = n & 3;
        if (ok && n >= 2 && !mbar_wait(q_empty + qs, ((n >> 1) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 52, abort_flag);
          ok = false;
        }
        if (ok && n >= 4 && !mbar_wait(rc_empty + rs, ((n >> 2) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 53, abort_flag);
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);   // warp-uniform: the copies below are cooperative
        if (!ok) continue;   // keep the loop shape: the item fetch barriers stay matched
        // the warp's 32 rows, two rows per step: lane l copies 16-byte piece l & 15 of row
        // 2 i + (l >> 4) (two whole 256-byte rows per copy instruction); rows past the list
        // become finite zeros (0 times garbage could be NaN in the MMA)
        {
          const uint32_t stage = smem_u32(sm + OFF_Q) + qs * kQStage;
          const long long my_row = valid ? (long long)qrow : -1ll;
          const int c = lane & 15;
#pragma unroll 4
          for (int i = 0; i < 16; ++i) {
            const int rr = 2 * i + (lane >> 4);
            const long long row = __shfl_sync(0xffffffffu, my_row, rr);
            const int R = (r & ~31) + rr;   // tile row
            const uint32_t o = (uint32_t)(R * 128 + (c >> 3) * kQHalf + (((c & 7) ^ (R & 7)) << 4));
            if (row >= 0) cp_async16(stage + o, a.q + row * kD + c * 8);
            else st_shared_v4(stage + o, 0u, 0u, 0u, 0u);
          }
        }
        float* rcb = rcf + rs * 3 * kM;
        rcb[r] = valid ? __int_as_float(ent.y) * kLog2e - mr : -INFINITY;
        // last visible key column of block j for this row (all 64 unless j is its current block)
        reinterpret_cast<int*>(rcb)[kM + r] = valid ? min(kB - 1, tg - s0 - jk0) : -1;
        reinterpret_cast<int*>(rcb)[2 * kM + r] = valid ? (int)qrow : -1;
        if (r == 0) {
          hdr[rs * 2] = (m == 0 ? kFlagFirst : 0) | (m == ntile - 1 ? kFlagLast : 0);
          hdr[rs * 2 + 1] = kvs;
        }
        cp_async_wait_all();
        fence_async_smem();
        mbar_arrive(q_full + qs);
        mbar_arrive(rc_full + rs);
      }
    }
    if (ok && *abort_flag == 0) {   // stop marker for the MMA, softmax and epilogue roles
      const int rs = n & 3;
      if (n >= 4 && !mbar_wait(rc_empty + rs, ((n >> 2) - 1) & 1, abort_flag)) {
        tc_fail(a.err, 54, abort_flag);
      } else {
        if (r == 0) hdr[rs * 2] = kFlagStop;
        mbar_arrive(rc_full + rs);
      }
    }
    // no TMA copy may still be in flight when the CTA exits
    if (r == 0)
      for (int i = max(0, item_seq - 2); i < item_seq; ++i)
        mbar_wait_drain(kv_full + (i & 1), (i >> 1) & 1);
  } else if (warp == 4) {
    // ------------------------------ MMA issue ------------------------------
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kM, kB, false, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(kM, kD, false, true);
      bool ok = true;
      int item_seq = 0;
      int pend = -1, pend_kvs = 0, pend_last = 0;
      auto issue_pv = [&](int m, int kvs, int last) -> bool {
        const int tb = m & 1;
        if (!mbar_wait(p_full + tb, (m >> 1) & 1, abort_flag)) return false;
        if (m >= 2 && !mbar_wait(o_empty + tb, ((m >> 1) - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm + OFF_KV + kvs * kKVStage + 2 * kKVHalf);
        const uint32_t p_col = tmem + kColS + tb * kB;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // O_part = P V: A = P from TMEM, B = V (MN-major)
          mma_bf16_ts(tmem + kColO + tb * kD, p_col + kk * 8,
                      sdesc_sw128(v_addr + kk * 2048, kKVHalf, 1024), kIdO, kk > 0 ? 1u : 0u);
        tc_commit(o_full + tb);
        if (last) tc_commit(kv_empty + kvs);
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int rs = n & 3, qs = n & 1;
        if (!mbar_wait(rc_full + rs, (n >> 2) & 1, abort_flag)) { ok = false; break; }
        const int flags = hdr[rs * 2], kvs = hdr[rs * 2 + 1];
        if (flags & kFlagStop) break;
        if (flags & kFlagFirst) {
          if (!mbar_wait(kv_full + kvs, (item_seq >> 1) & 1, abort_flag)) { ok = false; break; }
          ++item_seq;
        }
        if (!mbar_wait(q_full + qs, (n >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sm + OFF_Q + qs * kQStage);
        const uint32_t k_addr = smem_u32(sm + OFF_KV + kvs * kKVStage);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // S = Q K^T: both K-major in shared memory
          mma_bf16_ss(tmem + kColS + (n & 1) * kB,
                      sdesc_sw128(q_addr + (kk >> 2) * kQHalf + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(k_addr + (kk >> 2) * kKVHalf + (kk & 3) * 32, 16, 1024), kIdS,
                      kk > 0 ? 1u : 0u);
        tc_commit(s_full + (n & 1));
        tc_commit(q_empty + qs);
        if (pend >= 0 && !issue_pv(pend, pend_kvs, pend_last)) { ok = false; break; }
        pend = n;
        pend_kvs = kvs;
        pend_last = flags & kFlagLast;
      }
      if (ok && pend >= 0 && !issue_pv(pend, pend_kvs, pend_last)) ok = false;
      if (!ok) tc_fail(a.err, 55, abort_flag);
      tc_commit(final_bar);
      mbar_wait_drain(final_bar, 0);   // all MMAs done before the TMEM is released
    }
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------ softmax ------------------------------
    const int r = tid - 256;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    for (int n = 0;; ++n) {
      const int rs = n & 3, tb = n & 1;
      if (!warp_wait(rc_full + rs, (n >> 2) & 1, abort_flag)) { ok = false; break; }
      if (hdr[rs * 2] & kFlagStop) break;
      const float bias = rcf[rs * 3 * kM + r];
      const int limit = rci[rs * 3 * kM + kM + r];
      if (!warp_wait(s_full + tb, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_col = tmem + lane_addr + kColS + tb * kB;
      uint32_t pk[kB / 2];
      float lsum = 0.f;
      if (__any_sync(0xffffffffu, limit >= 0)) {
        float s[kB];
        tmem_ld64(s_col, s);
        if (limit >= kB - 1) {
#pragma unroll
          for (int c = 0; c < kB; c += 2) {
            const float p0 = ex2_approx(fmaf(s[c], a.scale_log2, bias));
            const float p1 = ex2_approx(fmaf(s[c + 1], a.scale_log2, bias));
            lsum += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
        } else {   // current block (or a row past the list, limit -1): keys above t masked
#pragma unroll
          for (int c = 0; c < kB; c += 2) {
            const float p0 = c <= limit ? ex2_approx(fmaf(s[c], a.scale_log2, bias)) : 0.f;
            const float p1 = c + 1 <= limit ? ex2_approx(fmaf(s[c + 1], a.scale_log2, bias)) : 0.f;
            lsum += p0 + p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < kB / 2; ++c) pk[c] = 0u;
      }
      tmem_st32(s_col, reinterpret_cast<const float*>(pk));   // P over the S columns
      // l_part column of this buffer: the epilogue of tile n-2 must have read it
      if (n >= 2 && !warp_wait(o_empty + tb, ((n >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      tmem_st1(tmem + lane_addr + kColL + tb, lsum);
      tc_fence_before();
      mbar_arrive(p_full + tb);
    }
    if (!ok) tc_fail(a.err, 56, abort_flag);
  } else if (warp >= 12) {
    // ------------------------------ epilogue ------------------------------
    const int r = tid - 384, ew = warp - 12;
    const uint32_t lane_addr = (uint32_t)(ew * 32) << 16;
    const uint32_t buf = smem_u32(sm + OFF_EPI) + (uint32_t)(ew * 32 * kEpiStride * 4);
    bool ok = true;
    for (int n = 0;; ++n) {
      const int rs = n & 3, tb = n & 1;
      if (!warp_wait(rc_full + rs, (n >> 2) & 1, abort_flag)) { ok = false; break; }
      if (hdr[rs * 2] & kFlagStop) break;
      const int dst = rci[rs * 3 * kM + 2 * kM + r];
      if (!warp_wait(o_full + tb, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t my_row = buf + (uint32_t)(lane * kEpiStride * 4);
      bulk_wait_read0();   // the previous tile's reduction has read this row's buffer
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_addr + kColO + tb * kD + c0, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_shared_v4(my_row + (uint32_t)((c0 + 4 * i) * 4), __float_as_uint(v[4 * i]),
                       __float_as_uint(v[4 * i + 1]), __float_as_uint(v[4 * i + 2]),
                       __float_as_uint(v[4 * i + 3]));
      }
      const float lsum = tmem_ld1(tmem + lane_addr + kColL + tb);
      tc_fence_before();
      mbar_arrive(o_empty + tb);   // TMEM buffer free for tile n+2
      fence_async_smem();          // the row is read by the TMA unit (async proxy)
      if (dst >= 0) {
        bulk_reduce_add_f32(a.oacc + (size_t)dst * kD, my_row, kD * 4);
        atomicAdd(a.lacc + dst, lsum);
      }
      bulk_commit();
      mbar_arrive(rc_empty + rs);
    }
    bulk_wait0();   // every reduction complete before the CTA exits
    if (!ok) tc_fail(a.err, 57, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
namespace {
struct KmLayout {
  size_t mref, oacc, lacc, lists, total;
};

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

KmLayout km_layout(const sas_problem& p) {
  KmLayout L;
  const size_t rows = (size_t)p.total_tokens * p.num_q_heads;
  size_t o = 256;   // word 0: error code
  L.mref = o;  o += al256(rows * 4);
  L.oacc = o;  o += al256(rows * kmf::kD * 4);
  L.lacc = o;  o += al256(rows * 4);
  L.lists = o; o += km_lists_bytes(p);
  L.total = o;
  return L;
}
}  // namespace

bool attn_fwd_km_supported(const sas_problem& p) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  return attn_tc_supported(p) && km_supported(p) && NBmax <= km::kMaxBins;
}

size_t attn_fwd_km_workspace_bytes(const sas_problem& p) { return km_layout(p).total; }

sas_status launch_attn_fwd_km(const sas_problem& p, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* logg, void* o, float* lse,
                              void* workspace, cudaStream_t st) {
  const KmLayout L = km_layout(p);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws);
  float* mref = reinterpret_cast<float*>(ws + L.mref);
  float* oacc = reinterpret_cast<float*>(ws + L.oacc);
  float* lacc = reinterpret_cast<float*>(ws + L.lacc);
  const KmLists lists = km_lists_carve(p, ws + L.lists);
  const int Hs = gate_heads(p);
  const int G = p.num_q_heads / Hs;   // query heads per gate head (the rows of a token)
  const int Hkv = p.num_kv_heads;
  const int R = Hs / Hkv;
  const int T = p.total_tokens;
  const float scale_log2 = kLog2e / sqrtf(128.f);

  CUtensorMap tk, tv;
  if (!make_tmap_bf16_3d(&tk, k, 128, Hkv, T, 64, 1, 64) ||
      !make_tmap_bf16_3d(&tv, v, 128, Hkv, T, 64, 1, 64)) {
    set_error("attn_fwd: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  // O_acc and l_acc are adjacent: one clear
  if (cudaMemsetAsync(oacc, 0, L.lists - L.oacc, st) != cudaSuccess) {
    set_error("attn_fwd: clearing the accumulators failed");
    return SAS_ERR_CUDA;
  }
  const int wpr = T * Hs;
  km_rowref_kernel<<<(wpr + 7) / 8, 256, 0, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                  idx, logg, p.cu_seqlens, p.batch, T,
                                                  p.num_q_heads, Hs, R, G, p.topk, scale_log2, mref);
  SAS_TRY(launch_km_lists(p, idx, logg, lists, st));

  KmFwdArgs a;
  a.cu = p.cu_seqlens;
  a.q = (const __nv_bfloat16*)q;
  a.list = lists.list;
  a.cnt = lists.cnt;
  a.off = lists.off;
  a.items = lists.items;
  a.ctl = lists.ctl;
  a.next_item = lists.ctl + 1;
  a.mref = mref;
  a.oacc = oacc;
  a.lacc = lacc;
  a.err = err;
  a.batch = p.batch;
  a.Hq = p.num_q_heads;
  a.Hkv = Hkv;
  a.G = G;
  a.R = R;
  a.Mq = tc_rows_per_tile(G);
  a.P = lists.P;
  a.scale_log2 = scale_log2;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(attn_fwd_km_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kmf::kSmemBytes);
  });
  attn_fwd_km_kernel<<<sm_count(), kmf::kThreads, kmf::kSmemBytes, st>>>(tk, tv, a);
  const int rows = T * p.num_q_heads;
  km_finalize_kernel<<<(rows + 7) / 8, 256, 0, st>>>(oacc, lacc, mref, rows,
                                                     (__nv_bfloat16*)o, lse, err);
  return launch_status("attn_fwd (key-major tensor cores)", 3);
}

}  // namespace sas
