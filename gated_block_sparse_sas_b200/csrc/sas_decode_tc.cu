// Tensor-core split-K attention of the sparse decode step (A7), bf16, head_dim 128, KV block 64.
// The newest token of each sequence attends to its kept blocks only (model card: a 2,048-token
// budget = Top-K historical blocks + the current block); the gate and Top-K run before this
// kernel and leave the selection in the workspace.
//
// CTA = (kv head, sequence, split of the kept-block slots). Kept blocks are taken in pairs
// (128 keys): both blocks' K rows, then their V rows, arrive by TMA (3-D boxes of 64 keys x 64
// channels, 128B swizzle) into a ring of three 32 KB slots (K of pair n, V of pair n, K of pair
// n+1, ...; two CTAs fit on an SM), and per pair
//   S^T = K Q^T        (M = 128 keys, N = 16: the G query heads padded with zero rows, K = d)
//   P   = 2^(S^T log2e/sqrt(d) + log2e log g_block - m_h)   (0 past the sequence end)
//   O^T += V^T P        (M = 128 channels, N = 16, K = 128 keys), accumulated in TMEM.
// Each head uses one fixed reference m_h = (logit of the token's own key) + 32 in log2 units,
// the same for every split, so no running maximum or rescale is needed and the splits merge by
// plain sums (the own key sits in the current block, which is always kept: the largest logit
// is at least m_h - 32). A head whose largest logit exceeds its own key's by more than ~140
// log2 units would overflow; that is reported through the error word (code 61).
//
// Warp roles (256 threads): warp 0 lane 0 loads K/V; warp 1 allocates TMEM and lane 0 issues
// the MMAs; warps 4-7 are the 128 lanes of S^T (one key each: P, masking, row sums) and, at
// the end, of O^T (one channel each). Every wait is bounded; a timeout records an error code.
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace dtc {
constexpr int kD = 128, kB = 64;
constexpr int kThreads = 256;
constexpr int kHalfBlk = kB * 128;          // one block, one 64-channel half: [64 keys][128 B] = 8 KB
constexpr int kHalfPair = 2 * kHalfBlk;     // both blocks of a pair, one half: [128 keys][128 B]
constexpr int kKV = 2 * kHalfPair;          // K (or V) of a pair: 32 KB = one ring slot
constexpr int kSlots = 3;
constexpr int kN = 16;                      // padded head count (MMA N)
constexpr int OFF_STAGE = 0;
constexpr int OFF_Q = kSlots * kKV;         // [16 heads][128 d] K-major: 2 halves x 2 KB
constexpr int OFF_P = OFF_Q + 2 * kN * 128; // 2 buffers x P^T [16 heads][128 keys]: 2 halves x 2 KB
constexpr int OFF_BLK = OFF_P + 2 * 2 * kN * 128;   // [128] kept block ids, [128] log-gates (log2)
constexpr int OFF_RED = OFF_BLK + 2 * 128 * 4;      // [4 warps][16] row-sum partials
constexpr int OFF_MREF = OFF_RED + 4 * kN * 4;      // [16]
constexpr int OFF_BAR = OFF_MREF + kN * 4;
constexpr int kNumBars = 2 * kSlots + 2 + 2 + 2 + 1;   // full, empty, s_full, p_full, p_empty, final
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
constexpr uint32_t kTmemCols = 64;          // S0 0..15, S1 16..31, O^T 32..47
constexpr int kColS = 0, kColO = 32;
}  // namespace dtc

struct DecTcArgs {
  const __nv_bfloat16* q;       // [batch][Hq][128] (rotated)
  const __nv_bfloat16* kc;      // [batch][Hkv][capacity][128]
  const int32_t* seqlens;
  const int32_t* sel_idx;       // [batch][Hkv][K+1]
  const float* sel_logg;
  float* part_ml;               // [batch][Hkv][nsplit][G][2]: m (log2), l
  float* part_acc;              // [batch][Hkv][nsplit][G][128]
  int* err;
  int Hkv, G, capacity, K, nsplit;
  float scale_log2;
  const int32_t* pt;            // paged caches: page of block j of sequence b ([batch][NBmax]); or null
  int nbmax, num_pages;
  int R;                        // gate heads per KV head: Hkv above counts gate heads, and gate
                                // head kv reads the K/V of KV head kv / R (of Hkv / R)
};

__global__ void __launch_bounds__(dtc::kThreads, 2)
    decode_attn_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const DecTcArgs a) {
  using namespace dtc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
  const int G = a.G, Hq = a.Hkv * G, K1 = a.K + 1;
  const int Lraw = a.seqlens[b];
  bool len_ok = Lraw >= 1 && Lraw <= a.capacity;
  int own_page = 0;   // paged caches: the page of the newest token's block, range-checked
  if (len_ok && a.pt != nullptr) {
    own_page = a.pt[(size_t)b * a.nbmax + (Lraw - 1) / kB];   // pt rows are per sequence
    len_ok = own_page >= 0 && own_page < a.num_pages;
  }
  const bool seq_ok = len_ok;
  const int L = seq_ok ? Lraw : 0;
  const int per = (K1 + a.nsplit - 1) / a.nsplit;
  const int sl0 = split * per, sl1 = min(K1, sl0 + per);
  const size_t srow = ((size_t)b * a.Hkv + kv) * K1;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* full = bars;                 // [3] ring slots
  uint64_t* empty = bars + kSlots;       // [3]
  uint64_t* s_full = bars + 2 * kSlots;  // [2]
  uint64_t* p_full = s_full + 2;         // [2]
  uint64_t* p_empty = p_full + 2;        // [2]
  uint64_t* final_bar = p_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  int* nblk_s = reinterpret_cast<int*>(sm + OFF_MISC + 8);
  int* blk_j = reinterpret_cast<int*>(sm + OFF_BLK);
  float* blk_b = reinterpret_cast<float*>(sm + OFF_BLK + 128 * 4);
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  float* mref = reinterpret_cast<float*>(sm + OFF_MREF);

  // ---------------- setup ----------------
  if (warp == 0) {   // this split's kept blocks in slot order (valid ones only)
    int n = 0;
    for (int s0 = sl0; s0 < sl1; s0 += 32) {
      const int sl = s0 + lane;
      int j = -1;
      float lg = 0.f;
      if (sl < sl1 && seq_ok) {
        j = a.sel_idx[srow + sl];
        lg = a.sel_logg[srow + sl];
      }
      const bool keep = j >= 0 && j * kB < L;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int pos = n + __popc(m & ((1u << lane) - 1u));
        blk_j[pos] = j;
        blk_b[pos] = lg * kLog2e;
      }
      n += __popc(m);
    }
    if (lane == 0) {
      *nblk_s = n;
      for (int i = 0; i < kSlots; ++i) {
        mbar_init(full + i, 1);
        mbar_init(empty + i, 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(s_full + i, 1);
        mbar_init(p_full + i, 128);
        mbar_init(p_empty + i, 1);
      }
      mbar_init(final_bar, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  } else if (warp == 2 || warp == 3) {   // Q tile: rows h < G = q heads, rows >= G zero; P^T zero
    const int t = tid - 64;
    for (int e = t; e < kN * 16; e += 64) {   // 16 chunks of 8 channels per head row
      const int h = e >> 4, c = e & 15;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (h < G && seq_ok)
        v = *reinterpret_cast<const uint4*>(a.q + ((size_t)b * Hq + kv * G + h) * kD + c * 8);
      const uint32_t dst = smem_u32(sm + OFF_Q) + (c >> 3) * (kN * 128) + h * 128 + (((c & 7) ^ (h & 7)) << 4);
      st_shared_v4(dst, v.x, v.y, v.z, v.w);
    }
    for (int e = t; e < 2 * 2 * kN * 128 / 16; e += 64)
      st_shared_v4(smem_u32(sm + OFF_P) + e * 16, 0u, 0u, 0u, 0u);
  } else if (warp >= 4) {   // m_h = (q_h . k_own / sqrt(d) + log g_current) log2e + 32
    const int w4 = warp - 4;
    float lg_cur = 0.f;
    if (seq_ok) {
      const int c = (L - 1) / kB;
      for (int s0 = 0; s0 < K1; s0 += 32) {
        const int s = s0 + lane;
        const bool hit = s < K1 && a.sel_idx[srow + s] == c;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
          const float v = hit ? a.sel_logg[srow + s] : 0.f;
          lg_cur = __shfl_sync(0xffffffffu, v, __ffs(m) - 1);
          break;
        }
      }
    }
    for (int h = w4; h < G; h += 4) {
      float dot = 0.f;
      if (seq_ok) {
        const int Hk = a.Hkv / a.R, kh = kv / a.R;
        const size_t own = a.pt != nullptr
                               ? ((size_t)own_page * Hk + kh) * kB + (L - 1) % kB
                               : ((size_t)b * Hk + kh) * a.capacity + (L - 1);
        const uint2 kr = *reinterpret_cast<const uint2*>(a.kc + own * kD + lane * 4);
        const uint2 qr = *reinterpret_cast<const uint2*>(a.q + ((size_t)b * Hq + kv * G + h) * kD + lane * 4);
        const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.x));
        const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.y));
        const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr.x));
        const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr.y));
        dot = q01.x * k01.x + q01.y * k01.y + q23.x * k23.x + q23.y * k23.y;
      }
      dot = warp_sum(dot);
      if (lane == 0) mref[h] = fmaf(dot, a.scale_log2, lg_cur * kLog2e) + 32.f;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nblk = *nblk_s;
  const int npairs = (nblk + 1) >> 1;

  if (warp == 0) {
    // ---------------- K/V loads ----------------
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int Hk = a.Hkv / a.R, kh = kv / a.R;   // K/V of the gate head's KV head
      const int z = b * Hk + kh;
      int issued = 0;   // ring loads issued: load i = K (i even) or V (i odd) of pair i / 2
      for (int i = 0; i < 2 * npairs; ++i) {
        const int slot = i % kSlots;
        if (i >= kSlots && !mbar_wait(empty + slot, ((i / kSlots) - 1) & 1, abort_flag)) {
          tc_fail(a.err, 81, abort_flag);
          break;
        }
        const int n = i >> 1;
        const CUtensorMap* map = (i & 1) ? &tmV : &tmK;
        uint8_t* dst = sm + OFF_STAGE + slot * kKV;
        const int ja = blk_j[2 * n];
        const int jb = (2 * n + 1 < nblk) ? blk_j[2 * n + 1] : ja;   // odd count: masked copy
        // block j's 64 keys: rows j*64.. of (b, kv) in the contiguous cache, or all 64 rows of
        // (page of j, kv) in the paged one (pages range-checked by the gate; a TMA box outside
        // the tensor is filled, never read)
        int ya = ja * kB, yb = jb * kB, za = z, zb = z;
        if (a.pt != nullptr) {
          ya = yb = 0;
          za = a.pt[(size_t)b * a.nbmax + ja] * Hk + kh;
          zb = a.pt[(size_t)b * a.nbmax + jb] * Hk + kh;
        }
        mbar_arrive_expect_tx(full + slot, kKV);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tma_load_3d(dst + h * kHalfPair, map, full + slot, 64 * h, ya, za);
          tma_load_3d(dst + h * kHalfPair + kHalfBlk, map, full + slot, 64 * h, yb, zb);
        }
        issued = i + 1;
      }
      for (int i = max(0, issued - kSlots); i < issued; ++i)   // none in flight at exit
        mbar_wait_drain(full + i % kSlots, (i / kSlots) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, kN, false, false);   // S^T = K Q^T
      constexpr uint32_t kIdO = idesc_bf16_f32(128, kN, true, false);    // O^T += V^T P
      const uint32_t q_addr = smem_u32(sm + OFF_Q);
      bool ok = true;
      auto pv = [&](int m) -> bool {
        const int vi = 2 * m + 1, vslot = vi % kSlots;
        if (!mbar_wait(full + vslot, (vi / kSlots) & 1, abort_flag)) return false;
        if (!mbar_wait(p_full + (m & 1), (m >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm + OFF_STAGE + vslot * kKV);
        const uint32_t p_addr = smem_u32(sm + OFF_P + (m & 1) * 2 * kN * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 16 keys per step; A = V (MN-major), B = P^T (K-major)
          mma_bf16_ss(tmem + kColO, sdesc_sw128(v_addr + kk * 2048, kHalfPair, 1024),
                      sdesc_sw128(p_addr + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024),
                      kIdO, (m > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty + vslot);
        tc_commit(p_empty + (m & 1));
        return true;
      };
      for (int n = 0; n < npairs; ++n) {
        const int st = n & 1, ki = 2 * n, kslot = ki % kSlots;
        if (!mbar_wait(full + kslot, (ki / kSlots) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm + OFF_STAGE + kslot * kKV);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 16 channels per step
          mma_bf16_ss(tmem + kColS + st * kN,
                      sdesc_sw128(k_addr + (kk >> 2) * kHalfPair + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(q_addr + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024),
                      kIdS, kk > 0 ? 1u : 0u);
        tc_commit(s_full + st);
        tc_commit(empty + kslot);   // K of pair n is read by no later MMA
        if (n >= 1 && !pv(n - 1)) { ok = false; break; }
      }
      if (ok && npairs >= 1 && !pv(npairs - 1)) ok = false;
      if (!ok) tc_fail(a.err, 82, abort_flag);
      tc_commit(final_bar);
      mbar_wait_drain(final_bar, 0);
    }
  } else if (warp >= 4) {
    // ---------------- P (one key per lane), then O^T (one channel per lane) ----------------
    const int r = tid - 128;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    float lsum[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) lsum[h] = 0.f;
    float mr[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) mr[h] = h < G ? mref[h] : 0.f;
    bool ok = true;
    for (int n = 0; n < npairs; ++n) {
      const int st = n & 1;
      if (!warp_wait(s_full + st, (n >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float s[kN];
      tmem_ld16(tmem + lane_addr + kColS + st * kN, s);
      const int bi = 2 * n + (r >> 6);
      const int key = r & 63;
      const bool valid = bi < nblk && blk_j[bi] * kB + key < L;
      const float bias = valid ? blk_b[bi] : 0.f;
      float p[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        p[h] = (valid && h < G) ? ex2_approx(fmaf(s[h], a.scale_log2, bias - mr[h])) : 0.f;
        lsum[h] += p[h];
      }
      if (n >= 2 && !warp_wait(p_empty + st, ((n >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      // P^T[h][key r] as bf16 (K-major B operand: rows = heads, 128B-swizzled 64-key halves)
      uint8_t* pb = sm + OFF_P + st * 2 * kN * 128 + (r >> 6) * (kN * 128);
      const int kk = r & 63;
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G)
          *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((((kk >> 3) ^ (h & 7)) << 4) | ((kk & 7) << 1))) =
              __float2bfloat16_rn(p[h]);
      // keys past the sequence end (or of a missing block): V row := 0 once the copy has landed
      const int vi = 2 * n + 1, vslot = vi % kSlots;
      if (__any_sync(0xffffffffu, !valid) && !warp_wait(full + vslot, (vi / kSlots) & 1, abort_flag)) {
        ok = false;
        break;
      }
      if (!valid) {
        uint8_t* vrow = sm + OFF_STAGE + vslot * kKV + (r >> 6) * kHalfBlk + (r & 63) * 128;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int c = 0; c < 8; ++c) st_shared_v4(smem_u32(vrow + h2 * kHalfPair + c * 16), 0u, 0u, 0u, 0u);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + st);
    }
    if (!ok) tc_fail(a.err, 83, abort_flag);
    // row sums per head over the 128 key lanes
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float v = warp_sum(lsum[h]);
      if (lane == 0 && h < G) red[(warp - 4) * kN + h] = v;
    }
    const bool have = ok && npairs >= 1 && warp_wait(final_bar, 0, abort_flag);
    float o[kN];
    if (have) {
      tc_fence_after();
      tmem_ld16(tmem + lane_addr + kColO, o);
    }
    named_bar(1, 128);   // the 4 row-sum warps, reached on every path
    const size_t prow = (((size_t)b * a.Hkv + kv) * a.nsplit + split) * G;
    for (int h = 0; h < G; ++h) a.part_acc[(prow + h) * kD + r] = have ? o[h] : 0.f;
    if (r < G) {
      const float l = red[r] + red[kN + r] + red[2 * kN + r] + red[3 * kN + r];
      const bool any = have && l > 0.f;
      a.part_ml[(prow + r) * 2] = any ? mref[r] : -INFINITY;
      a.part_ml[(prow + r) * 2 + 1] = any ? l : 0.f;
      if (any && !isfinite(l)) atomicCAS(a.err, 0, 61);
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
bool decode_attn_tc_supported(const sas_decode_problem& p) {
  const int G = p.num_q_heads / gate_heads(p);
  return tma_available() && p.dtype == SAS_BF16 && p.head_dim == 128 && p.block == 64 && G <= 8 &&
         p.topk + 1 <= 128;
}

sas_status launch_decode_attn_tc(const sas_decode_problem& p, const void* q, const void* kc,
                                 const void* vc, const int32_t* sel_idx, const float* sel_logg,
                                 float* part_ml, float* part_acc, int* err, int ns,
                                 const DecodePaging& pg, cudaStream_t st) {
  CUtensorMap tk, tv;
  // contiguous: [batch*Hkv][capacity][128]; paged: [num_pages*Hkv][64][128]
  const uint64_t rows = pg.pt != nullptr ? (uint64_t)pg.num_pages * p.num_kv_heads
                                         : (uint64_t)p.batch * p.num_kv_heads;
  const uint64_t keys = pg.pt != nullptr ? (uint64_t)dtc::kB : (uint64_t)p.capacity;
  if (!make_tmap_bf16_3d(&tk, kc, 128, keys, rows, 64, 64, 1) ||
      !make_tmap_bf16_3d(&tv, vc, 128, keys, rows, 64, 64, 1)) {
    set_error("decode: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  DecTcArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.kc = (const __nv_bfloat16*)kc;
  a.seqlens = p.seqlens;
  a.sel_idx = sel_idx;
  a.sel_logg = sel_logg;
  a.part_ml = part_ml;
  a.part_acc = part_acc;
  a.err = err;
  a.Hkv = gate_heads(p);                       // gate heads: CTAs, selections, partials
  a.G = p.num_q_heads / gate_heads(p);         // query heads per gate head
  a.R = gate_heads(p) / p.num_kv_heads;
  a.capacity = p.capacity;
  a.K = p.topk;
  a.nsplit = ns;
  a.scale_log2 = kLog2e / sqrtf(128.f);
  a.pt = pg.pt;
  a.nbmax = (p.capacity + p.block - 1) / p.block;
  a.num_pages = pg.num_pages;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(decode_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         dtc::kSmemBytes);
  });
  decode_attn_tc_kernel<<<dim3(gate_heads(p), p.batch, ns), dtc::kThreads, dtc::kSmemBytes, st>>>(
      tk, tv, a);
  return SAS_OK;
}

}  // namespace sas
