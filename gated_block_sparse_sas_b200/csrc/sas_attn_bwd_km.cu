// Key-major tensor-core backward of the gated sparse attention (A6), bf16, head_dim 128, KV
// block 64. The loss reaches the selector through standard backpropagation (paper
// abstract): besides dQ, dK, dV it returns, for every kept block, the gradient of its
// log-gate, dlogg = sum over the G heads and the block's keys of dS = P (dP - D).
//
// Work items are those of the key-major forward (sas_km.cuh): one KV block j of one KV head
// of one sequence with the query rows of one 4096-token window that kept it, gathered into
// 128-row tiles (Mq tokens x G heads). Per tile, with the forward's LSE and D = rowsum(dO O):
//   S = Q K_j^T, dP = dO V_j^T                        (M=128 rows, N=64 keys, K=128)
//   P = 2^(S log2e/sqrt(d) + log2e (log g - LSE)),  dS = P (dP - D)   (causal mask on the
//   current block); dlogg(token, slot) = sum of dS over the token's G rows and the 64 keys
//   dV_j^T += dO^T P,  dK_j^T += Q^T dS / sqrt(d)     (M=128 d, N=64 keys, K=128 rows)
//   dQ_rows = dS K_j / sqrt(d)                         (M=128 rows, N=128 d, K=64 keys)
// dV^T and dK^T stay in TMEM over the item and are added to fp32 dK/dV accumulators at its
// end; dQ of every tile is added to an fp32 accumulator with L2 reductions; a last pass
// rounds the three accumulators to bf16, applying the 1/sqrt(d) of dK and dQ there (the MMAs
// take the unscaled dS). dlogg needs no reduction: each kept
// (token, block) pair lives in exactly one tile. Summation order of the reductions is not
// fixed, so gradients can differ in the last fp32 bits from run to run.
//
// Warp roles (512 threads):
//   warps 0-3   gather. Thread r builds row r of each tile: list entry -> token, slot and
//               log-gate; LSE and D; the Q and dO rows by cp.async into 128B-swizzled K-major
//               tiles (2 stages); row constants into a 4-slot ring. Thread 0 fetches items and
//               passes each item's K/V block to the loader.
//   warp 5      K/V loader: lane 0 loads an item's K and V block by TMA into the single stage
//               once the previous item's gradient MMAs have released it.
//   warp 4      TMEM allocation; lane 0 issues the MMAs, event-driven: S/dP of the next tile
//               and the gradient MMAs of the oldest pending tile, each once its inputs are ready.
//   warps 8-11  dS: TMEM lane r = row r: P and dS as bf16 into shared tiles (operands of the
//               gradient MMAs), in packed f32x2 arithmetic (the pass is issue-bound); the causal
//               mask only in tiles that need it; dlogg summed over the token's G rows.
//   warps 12-15 epilogue: dQ of the tile from TMEM, 32 columns at a time, into a dense per-warp
//               buffer [32 rows][32 columns] (each lane's 16-byte pieces rotated by lane so the
//               stores hit distinct banks), then one TMA tensor reduction (cp.reduce.async.bulk
//               .tensor .add, fp32) per token: the G rows of a token are its G adjacent query
//               heads in dQ_acc and G adjacent lanes of one warp (a warp holds floor(32 / G)
//               whole tokens; G = 5: 24 tokens per tile) (a Q/dO stage is free as soon as the tile's gradient MMAs are
//               done); at an item's end dK/dV from TMEM (lane = d, column = key) into the
//               accumulators.
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

namespace kmb {
constexpr int kD = 128, kB = 64, kM = 128;
constexpr int kThreads = 512;
constexpr int kHalf = kM * 128;              // [128 rows][64 d] bf16: 16 KB
constexpr int kTile = 2 * kHalf;             // [128 rows][128 d] as two d halves: 32 KB
constexpr int kStage = 2 * kTile;            // Q tile, dO tile
constexpr int kEpiBytes = 32 * 32 * 4;       // a warp's dQ buffer: [32 rows][32 fp32 columns]
constexpr int kKVHalf = kB * 128;            // [64 keys][64 d]: 8 KB
constexpr int OFF_QD = 0;                    // 2 stages
constexpr int OFF_K = OFF_QD + 2 * kStage;   // [64 keys][128 d] as two halves
constexpr int OFF_V = OFF_K + 2 * kKVHalf;
constexpr int OFF_P = OFF_V + 2 * kKVHalf;   // [128 rows][64 keys] bf16, 128B-swizzled rows
constexpr int OFF_DS = OFF_P + kM * 128;
constexpr int kRcArrays = 5;                 // c1, D, limit, dst, dlogg index
constexpr int OFF_RC = OFF_DS + kM * 128;    // [4 slots][5][128]
constexpr int OFF_EPI = OFF_RC + 4 * kRcArrays * kM * 4;  // [4 warps][32 rows][32] fp32
constexpr int OFF_HDR = OFF_EPI + 4 * kEpiBytes;           // [4 slots][4]
constexpr int OFF_DESC = OFF_HDR + 4 * 4 * 4;             // [2 slots][2] item K/V rows, kv
constexpr int OFF_BAR = OFF_DESC + 2 * 2 * 4;
constexpr int kNumBars = 28;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
// TMEM columns: S 0..63, dP 64..127, dQ0 128..255, dQ1 256..383, dV^T 384..447, dK^T 448..511
constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 0, kColDP = 64, kColDQ = 128, kColDV = 384, kColDK = 448;
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagStop = 4;
}  // namespace kmb

// Two fp32 lanes at once (sm_100 packed f32x2 arithmetic): d = a * b + c, d = a - b, d = a * b,
// d = a + b on the pairs (a0, a1), (b0, b1), (c0, c1).
__device__ __forceinline__ void fma_x2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                       float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void sub_x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul_x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add_x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

struct KmBwdArgs {
  const int32_t* cu;
  const __nv_bfloat16* q;
  const __nv_bfloat16* dout;
  const int2* list;
  const int32_t* cnt;
  const int32_t* off;
  const int32_t* items;
  const int32_t* ctl;
  int* next_item;
  const float* lse;
  const float* drow;
  float* dq_acc;     // [T][Hq][128]
  float* dk_acc;     // [T][Hkv][128]
  float* dv_acc;
  float* dlogg;      // [T][Hkv][K+1]
  int* err;
  int batch, Hq, Hkv, G, Mq, P, K1;
  int Hs, R;         // gate heads, gate heads per KV head (1, or G with one gate per query head)
  float scale_log2, scale;
};

__global__ void __launch_bounds__(kmb::kThreads, 1)
    attn_bwd_km_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDQ, const KmBwdArgs a) {
  using namespace kmb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, Mq = a.Mq;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* qd_full = bars + 2;     // [2]
  uint64_t* qd_empty = bars + 4;    // [2]
  uint64_t* rc_full = bars + 6;     // [4]
  uint64_t* rc_empty = bars + 10;   // [4]
  uint64_t* s_full = bars + 14;
  uint64_t* s_free = bars + 15;
  uint64_t* ps_full = bars + 16;
  uint64_t* ps_empty = bars + 17;
  uint64_t* dq_full = bars + 18;    // [2]
  uint64_t* dq_empty = bars + 20;   // [2]
  uint64_t* dkv_empty = bars + 22;
  uint64_t* final_bar = bars + 23;
  uint64_t* item_full = bars + 24;   // [2]
  uint64_t* item_empty = bars + 26;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(sm + OFF_MISC + 8);
  float* rcf = reinterpret_cast<float*>(sm + OFF_RC);
  int* rci = reinterpret_cast<int*>(sm + OFF_RC);
  int* hdr = reinterpret_cast<int*>(sm + OFF_HDR);   // slot: flags, first key row, keys, kv
  volatile int* desc = reinterpret_cast<volatile int*>(sm + OFF_DESC);

  if (tid == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(qd_full + i, 128);
      mbar_init(qd_empty + i, 1);
      mbar_init(dq_full + i, 1);
      mbar_init(dq_empty + i, 128);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(rc_full + i, 128);
      mbar_init(rc_empty + i, 128);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(ps_full, 128);
    mbar_init(ps_empty, 1);
    mbar_init(dkv_empty, 128);
    mbar_init(final_bar, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(item_full + i, 1);
      mbar_init(item_empty + i, 1);
    }
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
  auto rc_slot = [&](int rs, int arr) { return rs * kRcArrays * kM + arr * kM; };

  if (warp < 4) {
    // ------------------------------ gather ------------------------------
    // a token's G rows never straddle two warps: a warp holds floor(32 / G) whole tokens
    // (G = 5: six tokens in lanes 0..29, lanes 30 and 31 idle), so the dS and epilogue warps
    // can sum and reduce a token's rows together (Mq = 4 floor(32 / G) tokens per tile)
    const int r = tid;
    const int tpw = 32 / G, lr = r & 31;
    const int tl = (r >> 5) * tpw + lr / G, g = lr % G;
    const bool row_ok = lr < tpw * G;
    bool ok = true;
    int n = 0, item_seq = 0;
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
      const int kv = itm.kv, j = itm.j;
      const int s0 = a.cu[itm.b], L = a.cu[itm.b + 1] - s0;
      const int key0 = s0 + j * kB;
      if (r == 0 && ok) {   // hand the item's K/V block to the loader (warp 5)
        const int ds = item_seq & 1;
        if (item_seq >= 2 && !mbar_wait(item_empty + ds, ((item_seq >> 1) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 71, abort_flag);
          ok = false;
        } else {
          desc[ds * 2] = key0;
          desc[ds * 2 + 1] = kv / a.R;   // the KV head the item's gate head reads
          mbar_arrive(item_full + ds);
        }
      }
      ++item_seq;
      const int ntile = (cnt + Mq - 1) / Mq;
      int2 nxt = make_int2(0, 0);
      if (row_ok && tl < cnt) nxt = a.list[off + tl];
      for (int m = 0; m < ntile; ++m, ++n) {
        const int rank = m * Mq + tl;
        const bool valid = row_ok && rank < cnt;
        const int2 ent = nxt;
        if (row_ok && rank + Mq < cnt) nxt = a.list[off + rank + Mq];   // next tile's entry
        const int tg = ent.x & 0xFFFFFF, slot = ent.x >> 24;
        const size_t qrow = (size_t)tg * a.Hq + kv * G + g;
        const float lse_v = valid ? a.lse[qrow] : 0.f;
        const float d_v = valid ? a.drow[qrow] : 0.f;
        const int qs = n & 1, rs = n & 3;
        if (ok && n >= 2 && !mbar_wait(qd_empty + qs, ((n >> 1) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 72, abort_flag);
          ok = false;
        }
        if (ok && n >= 4 && !mbar_wait(rc_empty + rs, ((n >> 2) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 73, abort_flag);
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);   // warp-uniform: the copies below are cooperative
        if (!ok) continue;   // keep the loop shape: the item fetch barriers stay matched
        // the warp's 32 rows, two rows per step: lane l copies 16-byte piece l & 15 of row
        // 2 i + (l >> 4), so each copy instruction reads two whole 256-byte rows (coalesced)
        // instead of one 16-byte piece of 32 rows; rows past the list become zeros (0 times
        // garbage could be NaN in the MMAs)
        {
          const uint32_t stage = smem_u32(sm + OFF_QD + qs * kStage);
          const long long my_row = valid ? (long long)qrow : -1ll;
          const int c = lane & 15;
#pragma unroll 4
          for (int i = 0; i < 16; ++i) {
            const int rr = 2 * i + (lane >> 4);
            const long long row = __shfl_sync(0xffffffffu, my_row, rr);
            const int R = (r & ~31) + rr;   // tile row
            const uint32_t o = (uint32_t)(R * 128 + (c >> 3) * kHalf + (((c & 7) ^ (R & 7)) << 4));
            if (row >= 0) {
              cp_async16(stage + o, a.q + row * kD + c * 8);
              cp_async16(stage + kTile + o, a.dout + row * kD + c * 8);
            } else {
              st_shared_v4(stage + o, 0u, 0u, 0u, 0u);
              st_shared_v4(stage + kTile + o, 0u, 0u, 0u, 0u);
            }
          }
        }
        rcf[rc_slot(rs, 0) + r] = valid ? (__int_as_float(ent.y) - lse_v) * kLog2e : -INFINITY;
        rcf[rc_slot(rs, 1) + r] = d_v;
        rci[rc_slot(rs, 2) + r] = valid ? min(kB - 1, tg - key0) : -1;
        rci[rc_slot(rs, 3) + r] = valid ? (int)qrow : -1;
        rci[rc_slot(rs, 4) + r] = valid ? (tg * a.Hs + kv) * a.K1 + slot : -1;
        if (r == 0) {
          hdr[rs * 4] = (m == 0 ? kFlagFirst : 0) | (m == ntile - 1 ? kFlagLast : 0);
          hdr[rs * 4 + 1] = key0;
          hdr[rs * 4 + 2] = min(kB, L - j * kB);
          hdr[rs * 4 + 3] = kv / a.R;
        }
        cp_async_wait_all();
        fence_async_smem();
        mbar_arrive(qd_full + qs);
        mbar_arrive(rc_full + rs);
      }
    }
    if (ok && *abort_flag == 0) {   // stop marker for the MMA, dS and epilogue roles
      const int rs = n & 3;
      if (n >= 4 && !mbar_wait(rc_empty + rs, ((n >> 2) - 1) & 1, abort_flag)) {
        tc_fail(a.err, 74, abort_flag);
      } else {
        if (r == 0) hdr[rs * 4] = kFlagStop;
        mbar_arrive(rc_full + rs);
      }
    }
    if (r == 0 && ok && *abort_flag == 0) {   // ... and for the loader
      const int ds = item_seq & 1;
      if (item_seq >= 2 && !mbar_wait(item_empty + ds, ((item_seq >> 1) - 1) & 1, abort_flag)) {
        tc_fail(a.err, 78, abort_flag);
      } else {
        desc[ds * 2] = -1;
        mbar_arrive(item_full + ds);
      }
    }
  } else if (warp == 5) {
    // ------------------------------ K/V loader ------------------------------
    // One stage: item i's block is loaded once the gradient MMAs of item i-1 are done.
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int i = 0;; ++i) {
        const int ds = i & 1;
        if (!mbar_wait(item_full + ds, (i >> 1) & 1, abort_flag)) break;
        const int key0 = desc[ds * 2], kv = desc[ds * 2 + 1];
        mbar_arrive(item_empty + ds);
        if (key0 < 0) break;
        if (i >= 1 && !mbar_wait(kv_empty, (i - 1) & 1, abort_flag)) {
          tc_fail(a.err, 79, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(kv_full, 4 * kKVHalf);
        tma_load_3d(sm + OFF_K, &tmK, kv_full, 0, kv, key0);
        tma_load_3d(sm + OFF_K + kKVHalf, &tmK, kv_full, 64, kv, key0);
        tma_load_3d(sm + OFF_V, &tmV, kv_full, 0, kv, key0);
        tma_load_3d(sm + OFF_V + kKVHalf, &tmV, kv_full, 64, kv, key0);
        issued = i + 1;
      }
      if (issued >= 1) mbar_wait_drain(kv_full, (issued - 1) & 1);   // no TMA in flight at exit
    }
  } else if (warp == 4) {
    // ------------------------------ MMA issue ------------------------------
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kM, kB, false, false);   // S, dP
      constexpr uint32_t kIdKV = idesc_bf16_f32(kD, kB, true, true);    // dV^T, dK^T
      constexpr uint32_t kIdQ = idesc_bf16_f32(kM, kD, false, true);    // dQ
      const uint32_t k_addr = smem_u32(sm + OFF_K), v_addr = smem_u32(sm + OFF_V);
      const uint32_t p_addr = smem_u32(sm + OFF_P), ds_addr = smem_u32(sm + OFF_DS);
      // Event-driven issue: S/dP of the next tile and the gradient MMAs of the oldest
      // pending tile are each issued as soon as their inputs are ready, so neither waits
      // for the other's producer (the gather of tile n+1 does not hold up the gradients of
      // tile n, and an item's last gradients release the K/V stage without waiting for the
      // next item's block).
      auto issue_grads = [&](int m, int flags) {
        const uint32_t q_addr = smem_u32(sm + OFF_QD + (m & 1) * kStage);
        const uint32_t do_addr = q_addr + kTile;
        const bool first = flags & kFlagFirst;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // dV^T += dO^T P: A = dO tile (MN-major), B = P (MN-major)
          mma_bf16_ss(tmem + kColDV, sdesc_sw128(do_addr + kk * 2048, kHalf, 1024),
                      sdesc_sw128(p_addr + kk * 2048, kHalf, 1024), kIdKV,
                      (!first || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // dK^T += Q^T dS
          mma_bf16_ss(tmem + kColDK, sdesc_sw128(q_addr + kk * 2048, kHalf, 1024),
                      sdesc_sw128(ds_addr + kk * 2048, kHalf, 1024), kIdKV,
                      (!first || kk > 0) ? 1u : 0u);
        // the tile's Q/dO stage is read by no later MMA: release it to the gather before dQ
        tc_commit(qd_empty + (m & 1));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // dQ = dS K: A = dS (K-major), B = K (MN-major)
          mma_bf16_ss(tmem + kColDQ + (m & 1) * kD, sdesc_sw128(ds_addr + kk * 32, 16, 1024),
                      sdesc_sw128(k_addr + kk * 2048, kKVHalf, 1024), kIdQ, kk > 0 ? 1u : 0u);
        tc_commit(ps_empty);
        tc_commit(dq_full + (m & 1));
        if (flags & kFlagLast) tc_commit(kv_empty);
      };
      bool ok = true, stop = false;
      int n_s = 0, n_g = 0;          // next tile for S/dP, next tile for the gradients
      int hflags = -1;               // header of tile n_s once read
      int item_seq = 0, cur_item = 0;
      int g_flags[4], g_item[4];     // tiles with S issued and gradients pending (n_g..n_s-1)
      long long t_last = clock64();
      while (true) {
        bool progress = false;
        if (!stop) {
          const int rs = n_s & 3;
          if (hflags < 0 && mbar_test(rc_full + rs, (n_s >> 2) & 1)) {
            hflags = hdr[rs * 4];
            if (hflags & kFlagStop) stop = true;
          }
          if (hflags >= 0 && !stop) {
            bool ready = !(hflags & kFlagFirst) || mbar_test(kv_full, item_seq & 1);
            ready = ready && mbar_test(qd_full + (n_s & 1), (n_s >> 1) & 1);
            ready = ready && (n_s == 0 || mbar_test(s_free, (n_s - 1) & 1));
            if (ready) {
              if (hflags & kFlagFirst) cur_item = item_seq++;
              tc_fence_after();
              const uint32_t q_addr = smem_u32(sm + OFF_QD + (n_s & 1) * kStage);
              const uint32_t do_addr = q_addr + kTile;
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {   // S = Q K^T, dP = dO V^T (all K-major)
                const uint32_t ro = (kk >> 2) * kHalf + (kk & 3) * 32;
                const uint32_t ko = (kk >> 2) * kKVHalf + (kk & 3) * 32;
                mma_bf16_ss(tmem + kColS, sdesc_sw128(q_addr + ro, 16, 1024),
                            sdesc_sw128(k_addr + ko, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
                mma_bf16_ss(tmem + kColDP, sdesc_sw128(do_addr + ro, 16, 1024),
                            sdesc_sw128(v_addr + ko, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
              }
              tc_commit(s_full);
              g_flags[n_s & 3] = hflags;
              g_item[n_s & 3] = cur_item;
              ++n_s;
              hflags = -1;
              progress = true;
            }
          }
        }
        if (n_g < n_s) {
          const int m = n_g, fl = g_flags[m & 3], it = g_item[m & 3];
          bool ready = mbar_test(ps_full, m & 1);
          ready = ready && (m < 2 || mbar_test(dq_empty + (m & 1), ((m >> 1) - 1) & 1));
          ready = ready && (!(fl & kFlagFirst) || it < 1 || mbar_test(dkv_empty, (it - 1) & 1));
          if (ready) {
            tc_fence_after();
            issue_grads(m, fl);
            ++n_g;
            progress = true;
          }
        }
        if (stop && n_g == n_s) break;
        if (progress) {
          t_last = clock64();
        } else if (*abort_flag || clock64() - t_last > kWaitCycles) {
          ok = false;
          break;
        }
      }
      if (!ok) tc_fail(a.err, 75, abort_flag);
      tc_commit(final_bar);
      mbar_wait_drain(final_bar, 0);   // all MMAs done before the TMEM is released
    }
  } else if (warp >= 8 && warp < 12) {
    // ------------------------------ dS ------------------------------
    const int r = tid - 256;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t p_row = smem_u32(sm + OFF_P) + r * 128;
    const uint32_t ds_row = smem_u32(sm + OFF_DS) + r * 128;
    bool ok = true;
    for (int n = 0;; ++n) {
      const int rs = n & 3;
      if (!warp_wait(rc_full + rs, (n >> 2) & 1, abort_flag)) { ok = false; break; }
      if (hdr[rs * 4] & kFlagStop) break;
      const float c1 = rcf[rc_slot(rs, 0) + r];
      const float dd = rcf[rc_slot(rs, 1) + r];
      const int limit = rci[rc_slot(rs, 2) + r];
      const int dli = rci[rc_slot(rs, 4) + r];
      if (!warp_wait(s_full, n & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t pp[kB / 2], pd[kB / 2];
      // keys past the row's limit are masked only in the current block's tiles; rows past the
      // list have c1 = -inf, so their P is 0 without a mask
      const bool masked = !__all_sync(0xffffffffu, limit >= kB - 1 || limit < 0);
      const float sl = a.scale_log2;
      float dl0 = 0.f, dl1 = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float sv[32], dv[32];
        tmem_ld32(tmem + lane_addr + kColS + h * 32, sv);
        tmem_ld32(tmem + lane_addr + kColDP + h * 32, dv);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float x0, x1, p0, p1, t0, t1, s0, s1;
          fma_x2(x0, x1, sv[c], sv[c + 1], sl, sl, c1, c1);
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
          if (masked) {
            const int key = h * 32 + c;
            p0 = key <= limit ? p0 : 0.f;
            p1 = key + 1 <= limit ? p1 : 0.f;
          }
          sub_x2(t0, t1, dv[c], dv[c + 1], dd, dd);
          mul_x2(s0, s1, p0, p1, t0, t1);   // dS (the 1/sqrt(d) of dK and dQ is applied at the end)
          add_x2(dl0, dl1, dl0, dl1, s0, s1);
          pp[(h * 32 + c) >> 1] = pack_bf16x2(p0, p1);
          pd[(h * 32 + c) >> 1] = pack_bf16x2(s0, s1);
        }
      }
      float dlsum = dl0 + dl1;
      tc_fence_before();
      mbar_arrive(s_free);   // S and dP read: the next tile's MMAs may overwrite them
      // the gradient MMAs of tile n-1 have read the previous P and dS
      if (n >= 1 && !warp_wait(ps_empty, (n - 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t o = (uint32_t)((c ^ (r & 7)) << 4);
        st_shared_v4(p_row + o, pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
        st_shared_v4(ds_row + o, pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
      }
      fence_async_smem();
      // dlogg of (token, slot) = sum over the token's G rows: G adjacent lanes of this warp,
      // the first at a multiple of G
      if ((G & (G - 1)) == 0) {   // a power of two: butterfly over the G lanes
        for (int o = 1; o < G; o <<= 1) dlsum += __shfl_xor_sync(0xffffffffu, dlsum, o);
      } else {                    // G = 5: the token's first lane adds its next G - 1 lanes
        float sum = dlsum;
        for (int o = 1; o < G; ++o) sum += __shfl_down_sync(0xffffffffu, dlsum, o);
        dlsum = sum;
      }
      if (dli >= 0 && ((r & 31) % G) == 0) a.dlogg[dli] = dlsum;
      mbar_arrive(ps_full);
    }
    if (!ok) tc_fail(a.err, 76, abort_flag);
  } else if (warp >= 12) {
    // ------------------------------ epilogue ------------------------------
    const int r = tid - 384, ew = warp - 12;
    const uint32_t lane_addr = (uint32_t)(ew * 32) << 16;
    // one reduction box per token: its G rows, adjacent lanes of one warp (see the gather)
    const bool issuer = (lane % G) == 0;
    const int rot = lane & 7;
    const uint32_t my_row = smem_u32(sm + OFF_EPI) + (uint32_t)(ew * kEpiBytes + lane * 128);
    if (lane == 0) prefetch_tmap(&tmDQ);
    bool ok = true;
    for (int n = 0;; ++n) {
      const int rs = n & 3, qs = n & 1;
      if (!warp_wait(rc_full + rs, (n >> 2) & 1, abort_flag)) { ok = false; break; }
      const int flags = hdr[rs * 4];
      if (flags & kFlagStop) break;
      const int dst = rci[rc_slot(rs, 3) + r];
      if (!warp_wait(dq_full + qs, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int tok = dst >= 0 ? dst / a.Hq : 0, head = dst - tok * a.Hq;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + lane_addr + kColDQ + qs * kD + c0, v);
        if (c0 == kD - 32) {
          tc_fence_before();
          mbar_arrive(dq_empty + qs);   // TMEM dQ buffer free for tile n+2
        }
        // piece k of the store sequence is column group (k + rot) & 7 of this lane's row
        float4 w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
#pragma unroll
        for (int b = 1; b < 8; b <<= 1) {
          const bool on = (rot & b) != 0;
          float4 t[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) t[i] = w[(i + b) & 7];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            w[i].x = on ? t[i].x : w[i].x;
            w[i].y = on ? t[i].y : w[i].y;
            w[i].z = on ? t[i].z : w[i].z;
            w[i].w = on ? t[i].w : w[i].w;
          }
        }
        bulk_wait_read0();   // the previous chunk's reductions have read the buffer
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_shared_v4(my_row + (uint32_t)(((i + rot) & 7) << 4), __float_as_uint(w[i].x),
                       __float_as_uint(w[i].y), __float_as_uint(w[i].z), __float_as_uint(w[i].w));
        fence_async_smem();   // the rows are read by the TMA unit (async proxy)
        __syncwarp();
        if (issuer && dst >= 0) tma_reduce_add_3d(&tmDQ, my_row, c0, head, tok);
        bulk_commit();
      }
      if (flags & kFlagLast) {      // the item's dK^T, dV^T are complete (same commit as dQ)
        const int key0 = hdr[rs * 4 + 1], nkeys = hdr[rs * 4 + 2], kv = hdr[rs * 4 + 3];
        // thread r = TMEM lane r = channel d = r; column c = key c of the block
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          float dvv[32], dkv_[32];
          tmem_ld32(tmem + lane_addr + kColDV + h * 32, dvv);
          tmem_ld32(tmem + lane_addr + kColDK + h * 32, dkv_);
          if (h == 1) {
            tc_fence_before();
            mbar_arrive(dkv_empty);
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int key = h * 32 + c;
            if (key < nkeys) {
              const size_t o = ((size_t)(key0 + key) * a.Hkv + kv) * kD + r;
              atomicAdd(a.dv_acc + o, dvv[c]);
              atomicAdd(a.dk_acc + o, dkv_[c]);
            }
          }
        }
      }
      mbar_arrive(rc_empty + rs);
    }
    bulk_wait0();   // every reduction complete before the CTA exits
    if (!ok) tc_fail(a.err, 77, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// fp32 accumulators -> bf16 gradients (n4 groups of 4 values)
__global__ void km_bwd_finalize_kernel(const float4* __restrict__ acc, size_t n4,
                                       uint2* __restrict__ out, float scale) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 x = acc[i];
    out[i] = make_uint2(pack_bf16x2(x.x * scale, x.y * scale), pack_bf16x2(x.z * scale, x.w * scale));
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
namespace {
struct KmBwdLayout {
  size_t drow, dq, dk, dv, lists, total;
};

size_t al256b(size_t x) { return (x + 255) & ~(size_t)255; }

KmBwdLayout kmb_layout(const sas_problem& p) {
  KmBwdLayout L;
  const size_t rq = (size_t)p.total_tokens * p.num_q_heads;
  const size_t rk = (size_t)p.total_tokens * p.num_kv_heads;
  size_t o = 256;   // word 0: error code
  L.drow = o;  o += al256b(rq * 4);
  L.dq = o;    o += al256b(rq * kmb::kD * 4);
  L.dk = o;    o += al256b(rk * kmb::kD * 4);
  L.dv = o;    o += al256b(rk * kmb::kD * 4);
  L.lists = o; o += km_lists_bytes(p);
  L.total = o;
  return L;
}
}  // namespace

bool attn_bwd_km_supported(const sas_problem& p) { return attn_fwd_km_supported(p); }

size_t attn_bwd_km_workspace_bytes(const sas_problem& p) { return kmb_layout(p).total; }

sas_status launch_attn_bwd_km(const sas_problem& p, const void* q, const void* k, const void* v,
                              const void* o, const void* dout, const float* lse,
                              const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                              float* dlogg, void* workspace, cudaStream_t st) {
  const KmBwdLayout L = kmb_layout(p);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws);
  float* drow = reinterpret_cast<float*>(ws + L.drow);
  float* dq_acc = reinterpret_cast<float*>(ws + L.dq);
  float* dk_acc = reinterpret_cast<float*>(ws + L.dk);
  float* dv_acc = reinterpret_cast<float*>(ws + L.dv);
  const KmLists lists = km_lists_carve(p, ws + L.lists);
  const int Hs = gate_heads(p);
  const int G = p.num_q_heads / Hs;   // query heads per gate head (the rows of a token)
  const int Hkv = p.num_kv_heads;
  const int T = p.total_tokens;

  CUtensorMap tk, tv, tdq;
  const uint32_t box_rows = (uint32_t)G;   // the epilogue's box: one token's G rows
  if (!make_tmap_bf16_3d(&tk, k, 128, Hkv, T, 64, 1, 64) ||
      !make_tmap_bf16_3d(&tv, v, 128, Hkv, T, 64, 1, 64) ||
      !make_tmap_f32_3d(&tdq, dq_acc, 128, p.num_q_heads, T, 32, box_rows, 1)) {
    set_error("attn_bwd: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  if (cudaMemsetAsync(dq_acc, 0, L.lists - L.dq, st) != cudaSuccess ||
      cudaMemsetAsync(dlogg, 0, (size_t)T * Hs * (p.topk + 1) * 4, st) != cudaSuccess) {
    set_error("attn_bwd: clearing the accumulators failed");
    return SAS_ERR_CUDA;
  }
  SAS_TRY(launch_rowdot(p, o, dout, drow, st));
  SAS_TRY(launch_km_lists(p, idx, logg, lists, st));

  KmBwdArgs a;
  a.cu = p.cu_seqlens;
  a.q = (const __nv_bfloat16*)q;
  a.dout = (const __nv_bfloat16*)dout;
  a.list = lists.list;
  a.cnt = lists.cnt;
  a.off = lists.off;
  a.items = lists.items;
  a.ctl = lists.ctl;
  a.next_item = lists.ctl + 1;
  a.lse = lse;
  a.drow = drow;
  a.dq_acc = dq_acc;
  a.dk_acc = dk_acc;
  a.dv_acc = dv_acc;
  a.dlogg = dlogg;
  a.err = err;
  a.batch = p.batch;
  a.Hq = p.num_q_heads;
  a.Hkv = Hkv;
  a.G = G;
  a.Hs = Hs;
  a.R = Hs / Hkv;
  a.Mq = 4 * (32 / G);   // whole tokens per warp (G = 5: 24 tokens, 120 of the 128 rows)
  a.P = lists.P;
  a.K1 = p.topk + 1;
  a.scale = 1.f / sqrtf(128.f);
  a.scale_log2 = kLog2e * a.scale;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(attn_bwd_km_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kmb::kSmemBytes);
  });
  attn_bwd_km_kernel<<<sm_count(), kmb::kThreads, kmb::kSmemBytes, st>>>(tk, tv, tdq, a);
  const size_t nq4 = (size_t)T * p.num_q_heads * kmb::kD / 4;
  const size_t nk4 = (size_t)T * Hkv * kmb::kD / 4;
  km_bwd_finalize_kernel<<<4 * sm_count(), 256, 0, st>>>((const float4*)dq_acc, nq4, (uint2*)dq, a.scale);
  km_bwd_finalize_kernel<<<4 * sm_count(), 256, 0, st>>>((const float4*)dk_acc, nk4, (uint2*)dk, a.scale);
  km_bwd_finalize_kernel<<<4 * sm_count(), 256, 0, st>>>((const float4*)dv_acc, nk4, (uint2*)dv, 1.f);
  return launch_status("attn_bwd (key-major tensor cores)", 4);
}

}  // namespace sas
