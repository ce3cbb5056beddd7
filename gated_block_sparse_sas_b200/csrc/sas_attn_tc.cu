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
// Warp roles (256 threads):
//   warp 0 lane 0   TMA producer: Q tile once, then K/V blocks of the union through a
//                   3-stage ring (one 3-D box per 64-row half, block row = s0 + j*64)
//   warp 1 lane 0   MMA issuer: QK^T into one of two TMEM S buffers, PV into TMEM O
//   warp 1          TMEM allocation / release (256 columns: O 0..127, S0 128..191,
//                   S1 192..255)
//   warps 4..7      softmax: thread r owns TMEM lane r = query row r (token r/G, head r%G);
//                   scale, log-gate, causal mask, online max with lazy O rescale (only when
//                   the row max grows by more than 2^8), P to shared memory (bf16, 128B
//                   swizzle), epilogue O/l and LSE
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
constexpr int kStages = 3;
constexpr int kThreads = 256;
constexpr int kMaxSel = 4096;           // staged (tokens x slots) per tile
constexpr int kMaxBlocks = 2048;        // NBmax
constexpr int kHalf = kM * 128;         // one 64-column half of the Q tile: 16 KB
constexpr int kKVHalf = kB * 128;       // one 64-column half of a K or V block: 8 KB
constexpr int kStageBytes = 4 * kKVHalf;  // K0 K1 V0 V1
constexpr int kPBytes = kM * 128;       // P tile: 128 rows x 64 keys bf16
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + 2 * kHalf;
constexpr int OFF_P = OFF_KV + kStages * kStageBytes;
constexpr int OFF_SEL_IDX = OFF_P + 2 * kPBytes;
constexpr int OFF_SEL_LG = OFF_SEL_IDX + kMaxSel * 4;
constexpr int OFF_LIST = OFF_SEL_LG + kMaxSel * 4;
constexpr int OFF_MASK = OFF_LIST + kMaxBlocks * 4;
constexpr int OFF_BAR = OFF_MASK + kMaxBlocks / 8;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;   // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 256;
constexpr int kColS = 128;              // S buffers start column
constexpr float kRescaleThreshold = 8.0f;  // log2 units
}  // namespace tcf

struct TcFwdArgs {
  const int32_t* cu;
  const int32_t* idx;
  const float* logg;
  __nv_bfloat16* o;
  float* lse;
  int* err;
  int Hq, Hkv, G, K, Mq, NBmax, n_tiles;
  float scale_log2;
};

__global__ void __launch_bounds__(tcf::kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const TcFwdArgs a) {
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
  const int rows_used = G * a.Mq;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* q_full = bars;
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
    mbar_init(q_full, 1);
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
  if (rows_used < kM) {   // rows the Q box leaves untouched must hold zeros, not stale data
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int e = tid; e < (kM - rows_used) * 8; e += kThreads) {
      const int r = rows_used + (e >> 3), c = e & 7;
      reinterpret_cast<uint4*>(sm + OFF_Q + r * 128)[c] = z;
      reinterpret_cast<uint4*>(sm + OFF_Q + kHalf + r * 128)[c] = z;
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
    if (lane == 0) {   // TMA producer
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, 2u * rows_used * 128u);
      tma_load_3d(sm + OFF_Q, &tmQ, q_full, 0, kv * G, s0 + t0);
      tma_load_3d(sm + OFF_Q + kHalf, &tmQ, q_full, 64, kv * G, s0 + t0);
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
      mbar_wait_drain(q_full, 0);
      for (int n = max(0, issued - kStages); n < issued; ++n)
        mbar_wait_drain(kv_full + n % kStages, (n / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {   // MMA issuer
      constexpr uint32_t kIdescQK = idesc_bf16_f32(kM, kB, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kM, kD, false, true);
      const uint32_t q_addr = smem_u32(sm + OFF_Q);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      if (ok) tc_fence_after();
      for (int n = 0; ok && n <= nb; ++n) {
        if (n < nb) {
          const int st = n % kStages, bb = n & 1;
          if (!mbar_wait(kv_full + st, (n / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + OFF_KV + st * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = sdesc_sw128(q_addr + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(k_addr + (kk >> 2) * kKVHalf + (kk & 3) * 32, 16, 1024);
            mma_bf16_ss(tmem + kColS + bb * kB, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full + bb);
        }
        if (n >= 1) {
          const int m = n - 1, pb = m & 1, st = m % kStages;
          if (!mbar_wait(p_full + pb, (m >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t p_addr = smem_u32(sm + OFF_P + pb * kPBytes);
          const uint32_t v_addr = smem_u32(sm + OFF_KV + st * kStageBytes + 2 * kKVHalf);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(p_addr + kk * 32, 16, 1024);
            // V as the MN-major B operand: 64-column halves kKVHalf apart, 8-key groups 1 KB apart
            const uint64_t bd = sdesc_sw128(v_addr + kk * 2048, kKVHalf, 1024);
            mma_bf16_ss(tmem, ad, bd, kIdescPV, (m > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(pv_done + pb);
          tc_commit(kv_empty + st);
        }
      }
      if (!ok) tc_fail(a.err, 2, abort_flag);
      tc_commit(o_final);
      mbar_wait_drain(o_final, 0);   // all MMAs done before the TMEM is released
    }
  } else if (warp >= 4) {   // softmax warpgroup
    const int r = tid - 128;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int tl = r / G;
    const bool valid = r < G * nt;
    const int t = t0 + tl;
    const int ct = t / kB;
    const int32_t* my_idx = sel_idx + tl * K1;
    const float* my_lg = sel_lg + tl * K1;
    float m_ref = -INFINITY, l_sum = 0.f;
    int sp = 0;
    bool ok = true;
    for (int n = 0; n < nb; ++n) {
      const int bb = n & 1;
      const int j = list[n];
      if (!warp_wait(s_full + bb, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float s[kB];
      tmem_ld32(tmem + lane_addr + kColS + bb * kB, s);
      tmem_ld32(tmem + lane_addr + kColS + bb * kB + 32, s + 32);
      float bias = -INFINITY;
      if (valid) {
        while (sp < K1 && my_idx[sp] >= 0 && my_idx[sp] < j) ++sp;
        if (sp < K1 && my_idx[sp] == j) bias = my_lg[sp] * kLog2e;
      }
      const int limit = (j == ct) ? (t - j * kB) : (kB - 1);   // last visible key column
      float rmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kB; ++c) {
        const float x = (c <= limit) ? fmaf(s[c], a.scale_log2, bias) : -INFINITY;
        s[c] = x;
        rmax = fmaxf(rmax, x);
      }
      const bool grow = rmax > m_ref + kRescaleThreshold;
      const float m_new = grow ? rmax : m_ref;
      const float alpha = grow ? exp2f(m_ref - m_new) : 1.f;
      const bool need_o = grow && (m_ref != -INFINITY);
      if (__any_sync(0xffffffffu, need_o)) {
        // O may only be touched once PV(n-1) has completed
        if (!warp_wait(pv_done + ((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          float ov[32];
          tmem_ld32(tmem + lane_addr + c0, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tmem + lane_addr + c0, ov);
        }
      }
      l_sum *= alpha;
      m_ref = m_new;
      if (n >= 2 && !warp_wait(pv_done + bb, ((n - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
      const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
      float psum = 0.f;
      uint32_t pk[kB / 2];
#pragma unroll
      for (int c = 0; c < kB; c += 2) {
        const float p0 = exp2f(s[c] - ref), p1 = exp2f(s[c + 1] - ref);
        psum += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l_sum += psum;
      const uint32_t prow = smem_u32(sm + OFF_P + bb * kPBytes) + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(prow + ((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                     pk[4 * c + 3]);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + bb);
    }
    if (ok) ok = warp_wait(o_final, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv = (l_sum > 0.f) ? 1.f / l_sum : 0.f;
      const int hq = kv * G + (r % G);
      __nv_bfloat16* orow = a.o + ((size_t)(s0 + t) * a.Hq + hq) * kD;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float ov[32];
        tmem_ld32(tmem + lane_addr + c0, ov);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(ov[2 * i] * inv, ov[2 * i + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (valid) a.lse[(size_t)(s0 + t) * a.Hq + hq] = (m_ref + log2f(l_sum)) * kLn2;
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
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_3d(&tq, q, 128, p.num_q_heads, p.total_tokens, 64, G, Mq) ||
      !make_tmap_bf16_3d(&tk, k, 128, p.num_kv_heads, p.total_tokens, 64, 1, 64) ||
      !make_tmap_bf16_3d(&tv, v, 128, p.num_kv_heads, p.total_tokens, 64, 1, 64)) {
    set_error("attn_fwd: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  TcFwdArgs a;
  a.cu = p.cu_seqlens;
  a.idx = idx;
  a.logg = logg;
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
  attn_fwd_tc_kernel<<<grid, tcf::kThreads, tcf::kSmemBytes, st>>>(tq, tk, tv, a);
  return launch_status("attn_fwd (tensor cores)", 1);
}

}  // namespace sas
