// Tensor-core projections of the gate scores (A3), bf16 inputs, d = 128, h = 128.
//
// Per token t and kv head the gate needs two projections (model card: Query projection,
// Q/K normalization; the current block's key pools its visible prefix):
//   qproj_t = Wq . concat_g q_nope[t, kv*G+g]                       (G*d -> h)
//   kproj_t = Wk . [max, min, mean of k_nope over tokens c_t*B .. t]  (3d -> h)
// Both are bf16 x bf16 products: exact in fp32, so tcgen05 MMAs with fp32 accumulation
// compute them to fp32 accuracy. The prefix max and min of bf16 values are bf16 values; the
// prefix mean is an fp32 value, written as the sum of three bf16 parts (hi, mid, lo: 24
// significant bits), and the Wk columns of the mean are read three times by the B operand's
// TMA coordinates. So kproj is one GEMM with K = 640 over
//   A_k[t] = [pmax (d) | pmin (d) | mean_hi (d) | mean_mid (d) | mean_lo (d)]   (bf16)
// and qproj one GEMM with K = G*d straight from q_nope.
//
// GEMM kernel: C[m, kv, 0:128] (fp32) = A[m, a_col + k] . B[kv*128 + n, b_col(k)] over k;
// CTA = (128-row tile, kv head), 128 threads: warp 0 lane 0 loads A and B tiles (64 columns
// x 128 rows, 128B swizzle) by TMA into a 3-stage ring, warp 1 lane 0 issues the MMAs into a
// 128-column TMEM accumulator, all four warps write the rows out (TMEM lane = row).
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace gtc {
constexpr int kM = 128, kN = 128, kBK = 64;
constexpr int kStages = 3;
constexpr int kTileA = kM * 128;         // [128 rows][64 bf16]: 16 KB
constexpr int kTileB = kN * 128;
constexpr int kStage = kTileA + kTileB;
constexpr int kThreads = 128;
constexpr int OFF_BAR = kStages * kStage;
constexpr int OFF_MISC = OFF_BAR + (2 * kStages + 1) * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
constexpr int kKCols = 640;              // A_k row: pmax, pmin, mean hi / mid / lo
}  // namespace gtc

struct GemmArgs {
  int M, K;
  int a_col_kv;     // A column offset per kv head
  int b_mean3;      // B columns: 0 direct; 1: [0, 256) direct, then 256 + (k - 256) mod 128
  float* C;
  int ldc;          // floats between rows of C
  int* err;
};

__global__ void __launch_bounds__(gtc::kThreads)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs a) {
  using namespace gtc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kM, kv = blockIdx.y;
  const int nk = a.K / kBK;
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
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {   // TMA producer
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    int issued = 0;
    for (int ks = 0; ks < nk; ++ks) {
      const int st = ks % kStages;
      if (ks >= kStages && !mbar_wait(empty + st, ((ks / kStages) - 1) & 1, abort_flag)) {
        tc_fail(a.err, 91, abort_flag);
        break;
      }
      const int k0 = ks * kBK;
      const int bcol = (a.b_mean3 && k0 >= 256) ? 256 + ((k0 - 256) & 127) : k0;
      uint8_t* stg = sm + st * kStage;
      mbar_arrive_expect_tx(full + st, kStage);
      tma_load_2d(stg, &tmA, full + st, kv * a.a_col_kv + k0, m0);
      tma_load_2d(stg + kTileA, &tmB, full + st, bcol, kv * kN);
      issued = ks + 1;
    }
    for (int ks = max(0, issued - kStages); ks < issued; ++ks)
      mbar_wait_drain(full + ks % kStages, (ks / kStages) & 1);
  } else if (warp == 1 && lane == 0) {   // MMA issue
    constexpr uint32_t kId = idesc_bf16_f32(kM, kN, false, false);
    bool ok = true;
    for (int ks = 0; ks < nk; ++ks) {
      const int st = ks % kStages;
      if (!mbar_wait(full + st, (ks / kStages) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(sm + st * kStage), b_addr = a_addr + kTileA;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024),
                    sdesc_sw128(b_addr + kk * 32, 16, 1024), kId, (ks > 0 || kk > 0) ? 1u : 0u);
      tc_commit(empty + st);
    }
    if (!ok) tc_fail(a.err, 92, abort_flag);
    tc_commit(done);
    mbar_wait_drain(done, 0);
  }
  __syncwarp();
  // epilogue: thread r = TMEM lane r = row m0 + r
  const bool have = warp_wait(done, 0, abort_flag) && nk > 0;
  if (have) {
    tc_fence_after();
    const int m = m0 + tid;
    float* crow = a.C + (size_t)m * a.ldc + (size_t)kv * kN;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
    for (int c0 = 0; c0 < kN; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + lane_addr + c0, v);
      if (m < a.M) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<float4*>(crow + c0)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  } else if (nk > 0) {
    tc_fail(a.err, 93, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// A_k rows: per (block j of sequence b, kv head) the running max / min / mean of k_nope over
// the block's tokens, one thread per channel.
__global__ void __launch_bounds__(128) gate_prefix_kernel(const __nv_bfloat16* __restrict__ k_nope,
                                                          const int32_t* __restrict__ cu, int Hkv,
                                                          int B, __nv_bfloat16* __restrict__ ak) {
  const int j = blockIdx.x, b = blockIdx.y, kv = blockIdx.z, c = threadIdx.x;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int t0 = j * B;
  if (t0 >= L) return;
  const int t1 = min(L, t0 + B);
  float mx = 0.f, mn = 0.f, sum = 0.f;
  for (int t = t0; t < t1; ++t) {
    const size_t row = (size_t)(s0 + t) * Hkv + kv;
    const float x = __bfloat162float(k_nope[row * 128 + c]);
    const int r = t - t0;
    mx = r == 0 ? x : fmaxf(mx, x);
    mn = r == 0 ? x : fminf(mn, x);
    sum = r == 0 ? x : sum + x;
    const float mean = sum / (float)(r + 1);
    const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
    const float r1 = mean - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    __nv_bfloat16* dst = ak + row * gtc::kKCols;
    dst[c] = __float2bfloat16_rn(mx);   // exact: a bf16 value
    dst[128 + c] = __float2bfloat16_rn(mn);
    dst[256 + c] = hi;
    dst[384 + c] = mid;
    dst[512 + c] = lo;
  }
}

// ---------------------------------------------------------------------------------------
bool gate_tc_supported(const sas_problem& p) {
  return tma_available() && p.dtype == SAS_BF16 && p.head_dim == 128 && p.gate_hidden == 128 &&
         p.block <= 128 && ((p.num_q_heads / gate_heads(p)) * 128) % gtc::kBK == 0;
}

static size_t al256g(size_t x) { return (x + 255) & ~(size_t)255; }

size_t gate_tc_workspace_bytes(const sas_problem& p) {
  const size_t rows = (size_t)p.total_tokens * p.num_kv_heads;
  const size_t qrows = (size_t)p.total_tokens * gate_heads(p);
  return 256 + al256g(rows * gtc::kKCols * 2) + al256g(qrows * 128 * 4) + al256g(rows * 128 * 4);
}

sas_status launch_gate_proj_tc(const sas_problem& p, const void* q_nope, const void* k_nope,
                               const void* wq, const void* wk, void* workspace, float** qproj,
                               float** kproj, cudaStream_t st, const void** prefix_rows) {
  // qproj per gate head s (Hs of them; Gs query heads each), kproj per KV head
  const int T = p.total_tokens, Hkv = p.num_kv_heads, Hq = p.num_q_heads, Hs = gate_heads(p);
  const int G = Hq / Hs;
  const size_t rows = (size_t)T * Hkv;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws);
  __nv_bfloat16* ak = reinterpret_cast<__nv_bfloat16*>(ws + 256);
  if (prefix_rows != nullptr) *prefix_rows = ak;   // [T, Hkv, 640]: max | min | mean hi, mid, lo
  *qproj = reinterpret_cast<float*>(ws + 256 + al256g(rows * gtc::kKCols * 2));
  *kproj = *qproj + al256g((size_t)T * Hs * 128 * 4) / 4;
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  gate_prefix_kernel<<<dim3(NBmax, p.batch, Hkv), 128, 0, st>>>((const __nv_bfloat16*)k_nope,
                                                                p.cu_seqlens, Hkv, p.block, ak);
  CUtensorMap tAq, tBq, tAk, tBk;
  if (!make_tmap_bf16_2d(&tAq, q_nope, (uint64_t)Hq * 128, T, (uint64_t)Hq * 128 * 2, 64, 128) ||
      !make_tmap_bf16_2d(&tBq, wq, (uint64_t)G * 128, (uint64_t)Hs * 128, (uint64_t)G * 128 * 2,
                         64, 128) ||
      !make_tmap_bf16_2d(&tAk, ak, (uint64_t)Hkv * gtc::kKCols, T, (uint64_t)Hkv * gtc::kKCols * 2,
                         64, 128) ||
      !make_tmap_bf16_2d(&tBk, wk, 384, (uint64_t)Hkv * 128, 384 * 2, 64, 128)) {
    set_error("gate projections: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(gemm_bf16_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         gtc::kSmemBytes);
  });
  const dim3 qgrid((T + gtc::kM - 1) / gtc::kM, Hs), kgrid((T + gtc::kM - 1) / gtc::kM, Hkv);
  GemmArgs aq{T, G * 128, G * 128, 0, *qproj, Hs * 128, err};
  gemm_bf16_tc_kernel<<<qgrid, gtc::kThreads, gtc::kSmemBytes, st>>>(tAq, tBq, aq);
  GemmArgs ak_args{T, gtc::kKCols, gtc::kKCols, 1, *kproj, Hkv * 128, err};
  gemm_bf16_tc_kernel<<<kgrid, gtc::kThreads, gtc::kSmemBytes, st>>>(tAk, tBk, ak_args);
  return SAS_OK;
}

}  // namespace sas
