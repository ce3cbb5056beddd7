// Tensor-core (tcgen05 / TMEM / TMA) gated sparse attention forward (A5), bf16, head_dim
// 128, KV block 64.
//
// The method selects blocks per query token (README (b)), so a tensor-core tile of query
// rows has no single block list. A CTA takes a tile of Mq consecutive tokens x the G query
// heads of one KV head (Mq*G <= 128 rows, the MMA's M) and visits the UNION of its rows'
// selected blocks in ascending order; each row adds its own log-gate to the blocks it kept
// and -inf to the others (abstract: the gate sits inside the softmax in log form). Work per
// visited block: S = Q K^T (M=128, N=64, K=128) and O += P V (M=128, N=128, K=64).
//
// Warp roles (384 threads):
//   warp 0 lane 0   TMA producer: K/V blocks of the union through a 4-stage ring (one 3-D
//                   box per 64-column half, block row = s0 + j*64)
//   warp 1 lane 0   MMA issuer: S = Q K^T with A = Q from TMEM, O += P V with A = P from
//                   TMEM (only the B operands, K and V, are read from shared memory)
//   warp 1          TMEM allocation / release (512 columns)
//   warps 4..11     two softmax warpgroups; warpgroup w stages head-dim half w of the
//                   tile's Q rows into TMEM, then takes the union blocks n = w, w+2, ... with
//                   its own O accumulator (O0 0..127, O1 128..255) and S buffer (256..,
//                   320..). Thread r owns TMEM lane r = query row r (token r/G, head r%G):
//                   scale, log-gate, causal mask, online max with lazy O rescale (only when
//                   the row max grows by more than 2^8), P as bf16 pairs over the first 32
//                   columns of its S buffer. The epilogue merges the two partial softmaxes
//                   (as split-K) and writes O and LSE
// Every pipeline wait is bounded; a timeout sets the workspace error word and all roles
// wind down (in-flight TMA drained, MMAs completed, TMEM released) instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace tcf {
constexpr int kD = 128;                 // head dim
constexpr int kB = 64;                  // keys per block
constexpr int kM = 128;                 // rows per tile
constexpr int kStages = 4;
constexpr int kThreads = 384;           // 4 role warps + two softmax warpgroups
constexpr int kMaxSel = 4096;           // staged (tokens x slots) per tile
constexpr int kMaxBlocks = 2048;        // NBmax
constexpr int kKVHalf = kB * 128;       // one 64-column half of a K or V block: 8 KB
constexpr int kStageBytes = 4 * kKVHalf;  // K0 K1 V0 V1
constexpr int OFF_KV = 0;
constexpr int OFF_SEL_IDX = OFF_KV + kStages * kStageBytes;
constexpr int OFF_SEL_LG = OFF_SEL_IDX + kMaxSel * 4;
constexpr int OFF_LIST = OFF_SEL_LG + kMaxSel * 4;
constexpr int OFF_MASK = OFF_LIST + kMaxBlocks * 4;
constexpr int OFF_XCH = OFF_MASK + kMaxBlocks / 8;   // [2 warpgroups][m, l][128 rows]
constexpr int OFF_BAR = OFF_XCH + 2 * 2 * 128 * 4;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;   // + slack for 1024-byte alignment
// TMEM columns: O0 0..127, O1 128..255, S0 256..319, S1 320..383 (P of a block is written
// as bf16 pairs over the first 32 columns of its S buffer), Q 384..447 (bf16 pairs)
constexpr uint32_t kTmemCols = 512;
constexpr int kColS = 256;
constexpr int kColQ = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
}  // namespace tcf

struct TcFwdArgs {
  const int32_t* cu;
  const int32_t* idx;
  const float* logg;
  const __nv_bfloat16* q;
  __nv_bfloat16* o;
  float* lse;
  int* err;
  int Hq, Hkv, G, K, Mq, NBmax, n_tiles;
  float scale_log2;
};

__global__ void __launch_bounds__(tcf::kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const TcFwdArgs a) {
  using namespace tcf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = a.n_tiles - 1 - (int)blockIdx.x;   // longest (latest) tiles first
  const int b = blockIdx.y, kv = blockIdx.z;
  const int s0 = a.cu[b], L = a.cu[b + 1] - s0;
  const int t0 = tile * a.Mq;
  if (t0 >= L) return;
  const int nt = min(a.Mq, L - t0);
  const int G = a.G, K1 = a.K + 1;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* q_ready = bars;                  // Q staged in TMEM (256 softmax threads)
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_final = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  int* n_list_s = reinterpret_cast<int*>(sm + OFF_MISC + 8);
  int32_t* sel_idx = reinterpret_cast<int32_t*>(sm + OFF_SEL_IDX);
  float* sel_lg = reinterpret_cast<float*>(sm + OFF_SEL_LG);
  int32_t* list = reinterpret_cast<int32_t*>(sm + OFF_LIST);
  uint32_t* mask = reinterpret_cast<uint32_t*>(sm + OFF_MASK);

  // ------------------------------ setup ------------------------------
  const int nwords = (a.NBmax + 31) >> 5;
  for (int w = tid; w < nwords; w += kThreads) mask[w] = 0u;
  if (tid == 0) {
    mbar_init(q_ready, 256);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 128);
      mbar_init(pv_done + i, 1);
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
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
  if (warp == 0) {   // ascending union list
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

  // ------------------------------ roles ------------------------------
  if (warp == 0) {
    if (lane == 0) {   // TMA producer: K/V blocks of the union
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int n = 0; n < nb; ++n) {
        const int st = n % kStages;
        if (n >= kStages && !mbar_wait(kv_empty + st, ((n / kStages) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 1, abort_flag);
          break;
        }
        const int row = s0 + list[n] * kB;
        uint8_t* stg = sm + OFF_KV + st * kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, kStageBytes);
        tma_load_3d(stg, &tmK, kv_full + st, 0, kv, row);
        tma_load_3d(stg + kKVHalf, &tmK, kv_full + st, 64, kv, row);
        tma_load_3d(stg + 2 * kKVHalf, &tmV, kv_full + st, 0, kv, row);
        tma_load_3d(stg + 3 * kKVHalf, &tmV, kv_full + st, 64, kv, row);
        issued = n + 1;
      }
      // no copy may still be in flight when the CTA exits
      for (int n = max(0, issued - kStages); n < issued; ++n)
        mbar_wait_drain(kv_full + n % kStages, (n / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {   // MMA issuer
      constexpr uint32_t kIdescQK = idesc_bf16_f32(kM, kB, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kM, kD, false, true);
      bool ok = mbar_wait(q_ready, 0, abort_flag);
      if (ok) tc_fence_after();
      for (int n = 0; ok && n <= nb; ++n) {
        if (n < nb) {
          const int st = n % kStages, bb = n & 1;
          if (!mbar_wait(kv_full + st, (n / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + OFF_KV + st * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // S = Q K^T: A = Q from TMEM, B = K (K-major smem)
            const uint64_t bd = sdesc_sw128(k_addr + (kk >> 2) * kKVHalf + (kk & 3) * 32, 16, 1024);
            mma_bf16_ts(tmem + kColS + bb * kB, tmem + kColQ + kk * 8, bd, kIdescQK,
                        kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full + bb);
        }
        if (n >= 1) {
          const int m = n - 1, pb = m & 1, st = m % kStages;
          if (!mbar_wait(p_full + pb, (m >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sm + OFF_KV + st * kStageBytes + 2 * kKVHalf);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // O += P V: A = P from TMEM, B = V (MN-major smem)
            const uint64_t bd = sdesc_sw128(v_addr + kk * 2048, kKVHalf, 1024);
            // even blocks accumulate into O0, odd blocks into O1 (one per softmax warpgroup)
            mma_bf16_ts(tmem + pb * kD, tmem + kColS + pb * kB + kk * 8, bd, kIdescPV,
                        (m > 1 || kk > 0) ? 1u : 0u);
          }
          tc_commit(pv_done + pb);
          tc_commit(kv_empty + st);
        }
      }
      if (!ok) tc_fail(a.err, 2, abort_flag);
      tc_commit(o_final);
      mbar_wait_drain(o_final, 0);   // all MMAs done before the TMEM is released
    }
  } else if (warp >= 4) {   // softmax: warpgroup wg takes the union blocks n = wg, wg+2, ...
    const int wg = (warp - 4) >> 2;
    const int r = tid - 128 - wg * 128;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int tl = r / G;
    const bool valid = r < G * nt;
    const int t = t0 + tl;
    const int ct = t / kB;
    const int hq = kv * G + (r % G);
    const int32_t* my_idx = sel_idx + tl * K1;
    const float* my_lg = sel_lg + tl * K1;
    const uint32_t o_col = wg * kD;                    // this warpgroup's O accumulator
    const uint32_t s_col = kColS + wg * kB;            // and S / P buffer
    {   // stage this row of Q in TMEM: warpgroup wg writes head-dim half wg (bf16 pairs)
      uint32_t qw[32];
      if (valid) {
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)(s0 + t) * a.Hq + hq) * kD + wg * 64);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 u = src[i];
          qw[4 * i] = u.x; qw[4 * i + 1] = u.y; qw[4 * i + 2] = u.z; qw[4 * i + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) qw[i] = 0u;
      }
      tmem_st32(tmem + lane_addr + kColQ + wg * 32, reinterpret_cast<const float*>(qw));
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    float m_ref = -INFINITY, l_sum = 0.f;
    int sp = 0;
    bool ok = true;
    for (int n = wg; n < nb; n += 2) {
      const int j = list[n];
      if (!warp_wait(s_full + wg, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      // PV(n-2), this warpgroup's previous block, was issued before QK(n) and so has already
      // completed: O and the P columns are free (the wait returns at once)
      if (n >= 2 && !warp_wait(pv_done + wg, ((n - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float bias = -INFINITY;
      if (valid) {
        while (sp < K1 && my_idx[sp] >= 0 && my_idx[sp] < j) ++sp;
        if (sp < K1 && my_idx[sp] == j) bias = my_lg[sp] * kLog2e;
      }
      const bool has = bias != -INFINITY;
      uint32_t pk[kB / 2];
      if (__any_sync(0xffffffffu, has)) {
        float s[kB];
        tmem_ld64(tmem + lane_addr + s_col, s);
        const int limit = (j == ct) ? (t - j * kB) : (kB - 1);   // last visible key column
        float smax = -INFINITY;                                   // max of the raw scores
        if (limit == kB - 1) {
#pragma unroll
          for (int c = 0; c < kB; ++c) smax = fmaxf(smax, s[c]);
        } else {
#pragma unroll
          for (int c = 0; c < kB; ++c)
            if (c <= limit) smax = fmaxf(smax, s[c]);
        }
        const float rmax = has ? fmaf(smax, a.scale_log2, bias) : -INFINITY;
        const bool grow = rmax > m_ref + kRescaleThreshold;
        const float m_new = grow ? rmax : m_ref;
        const float alpha = grow ? ex2_approx(m_ref - m_new) : 1.f;
        const bool need_o = grow && (m_ref != -INFINITY);
        if (__any_sync(0xffffffffu, need_o)) {
#pragma unroll 1
          for (int c0 = 0; c0 < kD; c0 += 32) {
            float ov[32];
            tmem_ld32(tmem + lane_addr + o_col + c0, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            tmem_st32(tmem + lane_addr + o_col + c0, ov);
          }
        }
        l_sum *= alpha;
        m_ref = m_new;
        // p = 2^(s*scale + bias - m): one FMA and one ex2 per score; rows without the
        // block (bias = -inf) and masked keys give exactly 0
        const float off = has ? bias - m_ref : -INFINITY;
        float psum = 0.f;
#pragma unroll
        for (int c = 0; c < kB; c += 2) {
          const float p0 = (c <= limit) ? ex2_approx(fmaf(s[c], a.scale_log2, off)) : 0.f;
          const float p1 = (c + 1 <= limit) ? ex2_approx(fmaf(s[c + 1], a.scale_log2, off)) : 0.f;
          psum += p0 + p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l_sum += psum;
      } else {   // no row of this warp kept block j: its P row is zero, m and l unchanged
#pragma unroll
        for (int c = 0; c < kB / 2; ++c) pk[c] = 0u;
      }
      tmem_st32(tmem + lane_addr + s_col, reinterpret_cast<const float*>(pk));   // P over S
      tc_fence_before();
      mbar_arrive(p_full + wg);
    }
    // merge the two partial softmaxes: O = (O0 2^(m0-M) + O1 2^(m1-M)) / (l0 2^(m0-M) + l1 2^(m1-M))
    float* xch = reinterpret_cast<float*>(sm + OFF_XCH);
    xch[wg * 256 + r] = m_ref;
    xch[wg * 256 + 128 + r] = l_sum;
    named_bar(1, 256);   // both warpgroups, always reached
    const float m0 = xch[r], l0 = xch[128 + r], m1 = xch[256 + r], l1 = xch[384 + r];
    const float M = fmaxf(m0, m1);
    const float f0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M);
    const float f1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
    const float l = l0 * f0 + l1 * f1;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    if (ok) ok = warp_wait(o_final, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* orow = a.o + ((size_t)(s0 + t) * a.Hq + hq) * kD;
#pragma unroll 1
      for (int c0 = wg * 64; c0 < wg * 64 + 64; c0 += 32) {   // each warpgroup: half the columns
        // an accumulator that no PV wrote (union of 0 or 1 blocks) holds garbage: skip it
        // (nb is CTA-uniform, so the collective loads stay warp-uniform)
        float o0[32], o1[32];
        if (nb > 0) tmem_ld32(tmem + lane_addr + c0, o0);
        else for (int i = 0; i < 32; ++i) o0[i] = 0.f;
        if (nb > 1) tmem_ld32(tmem + lane_addr + kD + c0, o1);
        else for (int i = 0; i < 32; ++i) o1[i] = 0.f;
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2((o0[2 * i] * f0 + o1[2 * i] * f1) * inv,
                                (o0[2 * i + 1] * f0 + o1[2 * i + 1] * f1) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (valid && wg == 0) a.lse[(size_t)(s0 + t) * a.Hq + hq] = (M + log2f(l)) * kLn2;
    } else {
      tc_fail(a.err, 3, abort_flag);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D bf16 map over [n2][n1][n0] (n0 contiguous) with a (b0, b1, b2) box, 128B swizzle.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                       uint32_t b0, uint32_t b1, uint32_t b2) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_rows_per_tile(int G) { return G == 5 ? 25 : 128 / G; }

bool attn_tc_supported(const sas_problem& p) {
  const int G = p.num_q_heads / p.num_kv_heads;
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  return p.dtype == SAS_BF16 && p.head_dim == 128 && p.block == 64 && NBmax <= tcf::kMaxBlocks &&
         tc_rows_per_tile(G) * (p.topk + 1) <= tcf::kMaxSel && encode_fn() != nullptr;
}

sas_status launch_attn_fwd_tc(const sas_problem& p, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* logg, void* o, float* lse, int* err,
                              cudaStream_t st) {
  const int G = p.num_q_heads / p.num_kv_heads;
  const int Mq = tc_rows_per_tile(G);
  CUtensorMap tk, tv;
  if (!make_tmap_bf16_3d(&tk, k, 128, p.num_kv_heads, p.total_tokens, 64, 1, 64) ||
      !make_tmap_bf16_3d(&tv, v, 128, p.num_kv_heads, p.total_tokens, 64, 1, 64)) {
    set_error("attn_fwd: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  TcFwdArgs a;
  a.cu = p.cu_seqlens;
  a.idx = idx;
  a.logg = logg;
  a.q = (const __nv_bfloat16*)q;
  a.o = (__nv_bfloat16*)o;
  a.lse = lse;
  a.err = err;
  a.Hq = p.num_q_heads;
  a.Hkv = p.num_kv_heads;
  a.G = G;
  a.K = p.topk;
  a.Mq = Mq;
  a.NBmax = (p.max_seqlen + p.block - 1) / p.block;
  a.n_tiles = (p.max_seqlen + Mq - 1) / Mq;
  a.scale_log2 = kLog2e / sqrtf(128.f);
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tcf::kSmemBytes);
  });
  dim3 grid(a.n_tiles, p.batch, p.num_kv_heads);
  attn_fwd_tc_kernel<<<grid, tcf::kThreads, tcf::kSmemBytes, st>>>(tk, tv, a);
  return launch_status("attn_fwd (tensor cores)", 1);
}

}  // namespace sas
