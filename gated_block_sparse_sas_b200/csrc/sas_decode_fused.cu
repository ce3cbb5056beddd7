// Fused sparse decode step (A7) for bf16, head_dim 128, KV block 64: one persistent launch runs
// the gate, the Top-K selection, the split-K attention over the kept blocks and the merge of the
// splits. Model card "tencent/Simple-Attention-Sparsification": the released setup decodes with
// a 2,048-token budget (Top-K historical blocks plus the current block); Chinese guide, caveat 3:
// the budget caps the tokens each query attends to, not the KV cache.
//
// Why one launch: the gate of a (sequence, gate head) row is a chain of dependent steps
// (projections, scores over every cached block key, logsumexp, Top-K) that keeps little memory
// traffic in flight, while the attention streams the kept K/V blocks at full bandwidth. As
// separate launches the gate runs alone first; here CTAs that are still selecting share the
// SMs with CTAs that already stream attention.
//
// Work items, handed out in this order by one atomic counter:
//   P  (gate head, part, 8 sequences): Qproj (part 0, over the G pre-rotary query heads) or
//      Kproj of the pooled current block (part 1, max, min, mean), RMSNorm, gate rotary;
//      weights read once for 8 sequences. Result in the workspace; count on pflag.
//   S  (sequence, gate head): cached block keys stream into shared memory by bulk copies
//      (issued before the P item is waited for), scores q~.k~/sqrt(h), logsumexp over the
//      visible blocks, Top-K -> selection; then sflag.
//   A  (sequence, gate head, split): the attention of the tensor-core decode kernel over the
//      split's kept blocks (K/V by TMA into a 3-slot ring, S^T = K Q^T and O^T += V^T P on
//      tcgen05, one fixed reference per head), partial sums to the workspace; the last split of
//      a row to finish merges the row into O.
// An item waits only for items that come earlier in the order, and those never wait for later
// ones, so every wait ends once the earlier item's CTA (running, since it claimed the item)
// finishes it. Every wait is bounded anyway: a wait that gives up records an error code and
// raises the workspace's abort word, which ends every other wait and stops every CTA.
//
// (Interleaving the queue so that a row's A items follow its S item a few sequences later was
// slower: A items then wait for selections still running.)
//
// Shared memory is reused between item kinds: P items keep their inputs in the K/V ring, S items
// stream key chunks through the ring and keep the score row in the Q/P region. mbarrier phases
// are counted across items (every thread of the CTA keeps the same counters).
#include <cuda.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_decode_select.cuh"
#include "sas_kernels.h"
#include "sas_sm100.cuh"

namespace sas {
using namespace sm100;

namespace dfz {
constexpr int kThreads = kDecThreads;       // 256
constexpr int kD = 128, kB = 64, kN = 16;
constexpr int kPB = 4;                      // sequences per P item
constexpr int kHalfBlk = kB * 128;          // one block, one 64-channel half: 8 KB
constexpr int kHalfPair = 2 * kHalfBlk;     // both blocks of a pair, one half
constexpr int kKV = 2 * kHalfPair;          // K (or V) of a pair: 32 KB = one ring slot
constexpr int kSlots = 3;
constexpr int OFF_STAGE = 0;
constexpr int OFF_Q = kSlots * kKV;                 // Q tile [16 heads][128 d], 2 halves of 2 KB
constexpr int OFF_P = OFF_Q + 2 * kN * 128;         // 2 buffers x P^T [16 heads][128 keys]
constexpr int OFF_BLK = OFF_P + 2 * 2 * kN * 128;   // [128] kept block ids, [128] log-gates (log2)
constexpr int OFF_RED = OFF_BLK + 2 * 128 * 4;      // [4 warps][16] row-sum partials
constexpr int OFF_MREF = OFF_RED + 4 * kN * 4;      // [16]
constexpr int OFF_BAR = OFF_MREF + kN * 4;
// full[3], empty[3], s_full[2], p_full[2], p_empty[2], final, gate-key chunks gfull[3]
constexpr int kNumBars = 2 * kSlots + 2 + 2 + 2 + 1 + kSlots;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;
// S items: the score row s[0..NBmax] at OFF_Q, then xq[H], xk[H]; the radix histogram at
// OFF_BLK; block reductions at OFF_RED
constexpr int kMaxNB = 2048;
constexpr int OFF_GS = OFF_Q;
constexpr int OFF_GX = OFF_Q + (((kMaxNB + 1) * 4 + 15) & ~15);
static_assert(OFF_GX + 2 * 128 * 4 <= OFF_BLK, "score row and gate vectors overflow the Q/P region");
static_assert(kPB * (8 * 128 + 128) * 4 <= kSlots * kKV, "P item inputs overflow the ring");
constexpr uint32_t kTmemCols = 64;          // S0 0..15, S1 16..31, O^T 32..47
constexpr int kColS = 0, kColO = 32;
// workspace header words
constexpr int kHdrErr = 0, kHdrNext = 1, kHdrAbort = 2;
}  // namespace dfz

struct FzArgs {
  const __nv_bfloat16* q;        // [batch][Hq][128] rotated queries
  const __nv_bfloat16* q_nope;   // [batch][Hq][128] pre-rotary queries (gate input)
  const __nv_bfloat16* kc;       // K cache (the own key's logit sets the fixed reference)
  const __nv_bfloat16* gkc;      // gate-key cache [batch][Hkv][NBmax][H] or pages [np][Hkv][H]
  const float* cur_pool;         // [batch][Hkv][3][128]: running max, min, sum of the current block
  const __nv_bfloat16* wq;       // [Hs][H][G*128]
  const float* qnorm_w;          // [H]
  const __nv_bfloat16* wk;       // [Hkv][H][384]
  const float* knorm_w;          // [H]
  const int32_t* seqlens;        // [batch]
  const float* rc;               // gate rotary tables [capacity][H/2]
  const float* rs;
  const int32_t* pt;             // paged caches: page of block j of sequence b, or null
  int num_pages;
  __nv_bfloat16* o;              // [batch][Hq][128]
  int32_t* idx_out;              // optional [batch][Hs][K+1]
  float* logg_out;
  int* hdr;                      // workspace header: error, next item, abort
  int* pflag;                    // [nchunk][Hs]: P items done (2 = both parts)
  int* sflag;                    // [batch][Hs]: selection written
  int* done;                     // [batch][Hs]: attention splits finished
  int32_t* sel_idx;              // [batch][Hs][K+1]
  float* sel_logg;
  float* gq;                     // [batch][Hs][2][H]: q~ and the current block's key
  float* part_ml;                // [batch][Hs][ns][G][2]: m (log2), l
  float* part_acc;               // [batch][Hs][ns][G][128]
  int batch, Hq, Hkv, Hs, G, R, K, capacity, nbmax, ns, ungated;
  int nP, nS, nA;
  float eps, scale_log2;
};

namespace {

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// Bounded wait (one thread) until *flag >= target; false on timeout or when another CTA raised
// the abort word.
__device__ bool wait_flag(const int* flag, int target, const int* abort_word) {
  if (ld_acquire(flag) >= target) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(100);
    if (ld_acquire(flag) >= target) return true;
    if (ld_volatile(abort_word)) return false;
    if (clock64() - t0 > kWaitCycles) return false;
  }
}

// Record a failure: the first error code wins; every CTA stops at its next check.
__device__ __forceinline__ void fz_fail(const FzArgs& a, int code, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicCAS(a.hdr + dfz::kHdrErr, 0, code);
  atomicExch(a.hdr + dfz::kHdrAbort, 1);
}

// One bulk copy global -> shared, completing on `bar` (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool seq_len_ok(int L, int capacity) { return L >= 1 && L <= capacity; }

// ---------------------------------------------------------------------------------------------
// P item: part 0 = Qproj over the gate head's G concatenated pre-rotary query heads; part 1 =
// Kproj of the current block's pooled (max, min, mean) key. Then RMSNorm (weight after the
// normalisation) and the gate rotary at t = L - 1 (query) or c B (current block start).
// ---------------------------------------------------------------------------------------------
template <int H>
__device__ void proj_item(const FzArgs& a, uint8_t* sm, int sh, int part, int chunk) {
  using namespace dfz;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv = sh / a.R, Gg = a.Hq / a.Hs;   // Gg: query heads of the gate head
  const int n_in = part == 0 ? Gg * kD : 3 * kD;
  const int b0 = chunk * kPB, nb = min(kPB, a.batch - b0);
  float* xin = reinterpret_cast<float*>(sm + OFF_STAGE);   // [kPB][n_in]
  float* xo = xin + kPB * n_in;                            // [kPB][H]
  for (int e = tid; e < kPB * n_in; e += kThreads) {
    const int bi = e / n_in, r = e - bi * n_in, b = b0 + bi;
    float x = 0.f;
    if (bi < nb) {
      const int L = a.seqlens[b];
      if (seq_len_ok(L, a.capacity)) {
        if (part == 0) {
          x = __bfloat162float(a.q_nope[((size_t)b * a.Hq + (size_t)sh * Gg) * kD + r]);
        } else {
          const int pr = r / kD, ch = r - pr * kD;
          const int n = L - ((L - 1) / kB) * kB;   // tokens of the current block so far
          x = a.cur_pool[(((size_t)b * a.Hkv + kv) * 3 + pr) * kD + ch];
          if (pr == 2) x = x / (float)n;
        }
      }
    }
    xin[e] = x;
  }
  __syncthreads();
  // output rows: four per warp step, lanes across the input in 16-byte weight vectors (two per
  // lane per row in flight); each weight vector serves the kPB sequences
  constexpr int RR = 4;
  const __nv_bfloat16* W = part == 0 ? a.wq + (size_t)sh * H * n_in : a.wk + (size_t)kv * H * n_in;
  const int nv = n_in / 8;
  for (int row0 = warp * RR; row0 < H; row0 += kDecWarps * RR) {
    float acc[RR][kPB];
#pragma unroll
    for (int u = 0; u < RR; ++u)
#pragma unroll
      for (int bi = 0; bi < kPB; ++bi) acc[u][bi] = 0.f;
    for (int v0 = 0; v0 < nv; v0 += 64) {
      uint4 raw[RR][2];
#pragma unroll
      for (int u = 0; u < RR; ++u)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int v = v0 + h2 * 32 + lane;
          raw[u][h2] = v < nv ? __ldg(reinterpret_cast<const uint4*>(W + (size_t)(row0 + u) * n_in) + v)
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int v = v0 + h2 * 32 + lane;
        if (v < nv) {
          float f[RR][8];
#pragma unroll
          for (int u = 0; u < RR; ++u) {
            const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&raw[u][h2]);
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const float2 ff = __bfloat1622float2(hh[q2]);
              f[u][2 * q2] = ff.x;
              f[u][2 * q2 + 1] = ff.y;
            }
          }
#pragma unroll
          for (int bi = 0; bi < kPB; ++bi) {
            const float4 xa = *reinterpret_cast<const float4*>(xin + bi * n_in + v * 8);
            const float4 xb = *reinterpret_cast<const float4*>(xin + bi * n_in + v * 8 + 4);
#pragma unroll
            for (int u = 0; u < RR; ++u) {
              float t = acc[u][bi];
              t = fmaf(f[u][0], xa.x, t); t = fmaf(f[u][1], xa.y, t);
              t = fmaf(f[u][2], xa.z, t); t = fmaf(f[u][3], xa.w, t);
              t = fmaf(f[u][4], xb.x, t); t = fmaf(f[u][5], xb.y, t);
              t = fmaf(f[u][6], xb.z, t); t = fmaf(f[u][7], xb.w, t);
              acc[u][bi] = t;
            }
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < RR; ++u)
#pragma unroll
      for (int bi = 0; bi < kPB; ++bi) {
        const float r = warp_sum(acc[u][bi]);
        if (lane == 0) xo[bi * H + row0 + u] = r;
      }
  }
  __syncthreads();
  // RMSNorm + rotary: warp bi takes sequence b0 + bi
  if (warp < nb) {
    const int b = b0 + warp;
    const int L = a.seqlens[b];
    if (seq_len_ok(L, a.capacity)) {
      const float* x = xo + warp * H;
      const float* w = part == 0 ? a.qnorm_w : a.knorm_w;
      const int pos = part == 0 ? L - 1 : ((L - 1) / kB) * kB;
      float ss = 0.f;
      for (int e = lane; e < H; e += 32) ss += x[e] * x[e];
      ss = warp_sum(ss);
      const float rn = sqrtf(ss / (float)H + a.eps);
      float* out = a.gq + (((size_t)b * a.Hs + sh) * 2 + part) * H;
      for (int e = lane; e < H / 2; e += 32) {
        const float u0 = x[e] / rn * w[e], u1 = x[e + H / 2] / rn * w[e + H / 2];
        const float cs = a.rc[(size_t)pos * (H / 2) + e], sn = a.rs[(size_t)pos * (H / 2) + e];
        out[e] = u0 * cs - u1 * sn;
        out[e + H / 2] = u1 * cs + u0 * sn;
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) atomicAdd(a.pflag + (size_t)chunk * a.Hs + sh, 1);
}

// Issue the bulk copies of chunk i (keys i*CK .. min(c, (i+1)*CK) - 1) of a gate row into ring
// slot `slot`. Warp 0 calls this (all lanes). Paged caches: one copy per key row; a page id out
// of range is not read (its row's score is discarded) and is reported through *bad.
template <int H>
__device__ void gate_chunk_issue(const FzArgs& a, uint8_t* sm, uint64_t* bar, int slot, int i, int c,
                                 int b, int kv, bool* bad) {
  using namespace dfz;
  constexpr int CK = kKV / (2 * H);
  const int lane = threadIdx.x & 31;
  const int j0 = i * CK, nk = min(CK, c - j0);
  const uint32_t dst = smem_u32(sm + OFF_STAGE + slot * kKV);
  if (a.pt == nullptr) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, (uint32_t)(nk * H * 2));
      const __nv_bfloat16* src = a.gkc + (((size_t)b * a.Hkv + kv) * (size_t)a.nbmax + j0) * H;
      bulk_g2s(dst, src, (uint32_t)(nk * H * 2), bar);
    }
  } else {   // one copy per key row; a row whose page id is out of range is not copied
    constexpr int PPL = CK / 32;   // rows per lane
    int pgs[PPL], nvalid = 0;
    bool my_bad = false;
#pragma unroll
    for (int k = 0; k < PPL; ++k) {
      const int r = lane + 32 * k;
      int pg = -1;
      if (r < nk) {
        pg = a.pt[(size_t)b * a.nbmax + j0 + r];
        if (pg < 0 || pg >= a.num_pages) {
          my_bad = true;
          pg = -1;
        }
      }
      pgs[k] = pg;
      nvalid += pg >= 0 ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) nvalid += __shfl_xor_sync(0xffffffffu, nvalid, o);
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nvalid * H * 2));
    __syncwarp();
#pragma unroll
    for (int k = 0; k < PPL; ++k)
      if (pgs[k] >= 0)
        bulk_g2s(dst + (lane + 32 * k) * H * 2, a.gkc + ((size_t)pgs[k] * a.Hkv + kv) * H, H * 2, bar);
    if (__any_sync(0xffffffffu, my_bad)) *bad = true;
  }
}

// ---------------------------------------------------------------------------------------------
// S item: scores of the row's cached block keys against q~, the current block's score from the
// pooled key, logsumexp and Top-K (decode_select_row).
// ---------------------------------------------------------------------------------------------
template <int H, int NPT>
__device__ void select_item(const FzArgs& a, uint8_t* sm, uint64_t* gfull, uint32_t& gk_n, int b, int sh,
                            volatile int* abort_flag) {
  using namespace dfz;
  constexpr int CK = kKV / (2 * H);   // keys per 32 KB chunk
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv = sh / a.R;
  const int L = a.seqlens[b];
  const size_t orow = ((size_t)b * a.Hs + sh) * (a.K + 1);
  float* s = reinterpret_cast<float*>(sm + OFF_GS);
  float* xq = reinterpret_cast<float*>(sm + OFF_GX);
  float* xk = xq + H;
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  int* cnt_red = reinterpret_cast<int*>(red + kDecWarps);
  int* misc = cnt_red + 2 * kDecWarps;   // [4], decode_select_row's; misc[4]: a page id out of range
  int* hist = reinterpret_cast<int*>(sm + OFF_BLK);
  volatile bool* bad = reinterpret_cast<volatile bool*>(misc + 4);
  if (seq_len_ok(L, a.capacity)) {
    const int c = (L - 1) / kB;
    const int nchunk = (c + CK - 1) / CK;
    if (tid == 0) {
      *bad = false;
      if (a.pt != nullptr) {   // the current block's page too (its keys are read by the attention)
        const int pg = a.pt[(size_t)b * a.nbmax + c];
        if (pg < 0 || pg >= a.num_pages) *bad = true;
      }
    }
    __syncthreads();
    int issued = min(nchunk, kSlots);   // chunk copies issued (the same count in every thread)
    if (warp == 0)
      for (int i = 0; i < issued; ++i)
        gate_chunk_issue<H>(a, sm, gfull + (gk_n + i) % kSlots, (gk_n + i) % kSlots, i, c, b, kv,
                            const_cast<bool*>(bad));
    if (tid == 0) {
      const int* f = a.pflag + (size_t)(b / kPB) * a.Hs + sh;
      if (!wait_flag(f, 2, a.hdr + kHdrAbort)) fz_fail(a, 84, abort_flag);
    }
    bool ok = __syncthreads_and(!*abort_flag);
    if (ok) {
      const float* g = a.gq + ((size_t)b * a.Hs + sh) * 2 * H;
      for (int e = tid; e < 2 * H; e += kThreads) xq[e] = __ldcg(g + e);   // xk follows xq
    }
    __syncthreads();
    const float sqrt_h = sqrtf((float)H);
    constexpr int LPR = H / 8, RPW = 32 / LPR;   // lanes per key row (16 B each), rows per warp
    const int sub = lane % LPR, rsub = lane / LPR;
    float qv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) qv[u] = xq[sub * 8 + u];
    for (int i = 0; i < nchunk; ++i) {
      const uint32_t gc = gk_n + i, slot = gc % kSlots;
      if (ok && !warp_wait(gfull + slot, (gc / kSlots) & 1, abort_flag)) {
        if (lane == 0) fz_fail(a, 86, abort_flag);
        ok = false;
      }
      ok = __syncthreads_and(ok);   // the same decision in every warp
      if (ok) {
        const uint8_t* base = sm + OFF_STAGE + slot * kKV;
        const int j0 = i * CK, nk = min(CK, c - j0);
        constexpr int UNR = CK / (kDecWarps * RPW);
#pragma unroll
        for (int it = 0; it < UNR; ++it) {
          const int r = (it * kDecWarps + warp) * RPW + rsub;
          float acc = 0.f;
          if (r < nk) {
            const uint4 raw = *reinterpret_cast<const uint4*>(base + (size_t)r * H * 2 + sub * 16);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
              const float2 f = __bfloat1622float2(h2[w2]);
              acc = fmaf(qv[2 * w2], f.x, acc);
              acc = fmaf(qv[2 * w2 + 1], f.y, acc);
            }
          }
#pragma unroll
          for (int off = 1; off < LPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if (sub == 0 && r < nk) s[j0 + r] = acc / sqrt_h;
        }
      }
      __syncthreads();   // slot read by every warp: refill it
      if (ok && i + kSlots < nchunk) {
        if (warp == 0)
          gate_chunk_issue<H>(a, sm, gfull + slot, slot, i + kSlots, c, b, kv, const_cast<bool*>(bad));
        ++issued;
      }
    }
    if (!ok && tid == 0)   // copies possibly in flight (the last use of each slot): let them land
      for (int i = max(0, issued - kSlots); i < issued; ++i)
        mbar_wait_drain(gfull + (gk_n + i) % kSlots, ((gk_n + i) / kSlots) & 1);
    gk_n += issued;
    if (warp == 0) {
      float dot = 0.f;
      for (int e = lane; e < H; e += 32) dot += xq[e] * xk[e];
      dot = warp_sum(dot);
      if (lane == 0) s[c] = dot / sqrt_h;
    }
    const bool any_bad = __syncthreads_or(*bad);
    if (any_bad) {
      if (tid == 0) atomicCAS(a.hdr + kHdrErr, 0, 62);
      decode_select_empty(a.K, orow, a.sel_idx, a.sel_logg, a.idx_out, a.logg_out);
    } else if (ok) {
      decode_select_row<NPT>(s, c, a.K, a.ungated, orow, a.sel_idx, a.sel_logg, a.idx_out, a.logg_out,
                             DecSelScratch{red, cnt_red, misc, hist});
    }
  } else {
    decode_select_empty(a.K, orow, a.sel_idx, a.sel_logg, a.idx_out, a.logg_out);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) atomicExch(a.sflag + (size_t)b * a.Hs + sh, 1);
}

// ---------------------------------------------------------------------------------------------
// A item: the tensor-core split-K attention (same math as decode_attn_tc_kernel), then the merge
// of the row's splits by the last one to finish.
// ---------------------------------------------------------------------------------------------
struct RingCounters {
  uint32_t ring;   // K/V ring loads issued by earlier items
  uint32_t pair;   // pairs processed by earlier items (s_full, p_full, p_empty phases)
  uint32_t fin;    // attention items finished (final barrier phases)
};

__device__ void attn_item(const FzArgs& a, const CUtensorMap* tmK, const CUtensorMap* tmV, uint8_t* sm,
                          uint32_t tmem, RingCounters& rc, int b, int sh, int split,
                          volatile int* abort_flag) {
  using namespace dfz;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, K1 = a.K + 1;
  const int Lraw = a.seqlens[b];
  bool len_ok = seq_len_ok(Lraw, a.capacity);
  int own_page = 0;
  if (len_ok && a.pt != nullptr) {
    own_page = a.pt[(size_t)b * a.nbmax + (Lraw - 1) / kB];
    len_ok = own_page >= 0 && own_page < a.num_pages;
  }
  const bool seq_ok = len_ok;
  const int L = seq_ok ? Lraw : 0;
  const int per = (K1 + a.ns - 1) / a.ns;
  const int sl0 = split * per, sl1 = min(K1, sl0 + per);
  const size_t srow = ((size_t)b * a.Hs + sh) * K1;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + kSlots;
  uint64_t* s_full = bars + 2 * kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* p_empty = p_full + 2;
  uint64_t* final_bar = p_empty + 2;
  int* nblk_s = reinterpret_cast<int*>(sm + OFF_MISC + 8);
  int* last_s = reinterpret_cast<int*>(sm + OFF_MISC + 12);
  int* blk_j = reinterpret_cast<int*>(sm + OFF_BLK);
  float* blk_b = reinterpret_cast<float*>(sm + OFF_BLK + 128 * 4);
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  float* mref = reinterpret_cast<float*>(sm + OFF_MREF);

  if (tid == 0 && !wait_flag(a.sflag + (size_t)b * a.Hs + sh, 1, a.hdr + kHdrAbort)) fz_fail(a, 85, abort_flag);
  __syncthreads();
  if (*abort_flag) return;

  // K/V load i of this item (i even: K of pair i / 2, odd: V) into ring slot (ring + i) % 3,
  // once the slot's previous use has been released; warp 0 lane 0 only
  const int Hk = a.Hkv, kh = sh / a.R;
  auto load_kv = [&](int i, int nblk) -> bool {
    const uint32_t gi = rc.ring + i, slot = gi % kSlots;
    if (gi >= kSlots && !mbar_wait(empty + slot, ((gi / kSlots) - 1) & 1, abort_flag)) return false;
    const int n = i >> 1;
    const CUtensorMap* map = (i & 1) ? tmV : tmK;
    uint8_t* dst = sm + OFF_STAGE + slot * kKV;
    const int ja = blk_j[2 * n];
    const int jb = (2 * n + 1 < nblk) ? blk_j[2 * n + 1] : ja;   // odd count: masked copy
    int ya = ja * kB, yb = jb * kB, za = b * Hk + kh, zb = za;
    if (a.pt != nullptr) {   // pages range-checked by the S item (a bad one empties the row)
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
    return true;
  };
  int issued = 0;   // warp 0 lane 0: K/V loads issued so far

  // ---------------- setup ----------------
  if (warp == 0) {   // this split's kept blocks in slot order (valid ones only)
    int n = 0;
    for (int s0 = sl0; s0 < sl1; s0 += 32) {
      const int sl = s0 + lane;
      int j = -1;
      float lg = 0.f;
      if (sl < sl1 && seq_ok) {
        j = __ldcg(a.sel_idx + srow + sl);
        lg = __ldcg(a.sel_logg + srow + sl);
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
    __syncwarp();
    if (lane == 0) {
      *nblk_s = n;
      // the first loads go out now, while the other warps set up Q and the references
      const int first = min(2 * ((n + 1) >> 1), kSlots);
      for (; issued < first; ++issued)
        if (!load_kv(issued, n)) {
          fz_fail(a, 81, abort_flag);
          break;
        }
    }
  } else if (warp == 2 || warp == 3) {   // Q tile: rows h < G = q heads, rows >= G zero; P^T zero
    const int t = tid - 64;
    for (int e = t; e < kN * 16; e += 64) {
      const int h = e >> 4, c = e & 15;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (h < G && seq_ok)
        v = *reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + sh * G + h) * kD + c * 8);
      const uint32_t dst = smem_u32(sm + OFF_Q) + (c >> 3) * (kN * 128) + h * 128 + (((c & 7) ^ (h & 7)) << 4);
      st_shared_v4(dst, v.x, v.y, v.z, v.w);
    }
    for (int e = t; e < 2 * 2 * kN * 128 / 16; e += 64)
      st_shared_v4(smem_u32(sm + OFF_P) + e * 16, 0u, 0u, 0u, 0u);
  } else if (warp >= 4) {   // m_h = (q_h . k_own / sqrt(d) + log g_current) log2e + 32
    const int w4 = warp - 4;
    float lg_cur = 0.f;
    if (seq_ok) {   // the current block's slot (K, or c when c <= K)
      const int c = (L - 1) / kB;
      for (int s0 = 0; s0 < K1; s0 += 32) {
        const int s = s0 + lane;
        const bool hit = s < K1 && __ldcg(a.sel_idx + srow + s) == c;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
          const float v = hit ? __ldcg(a.sel_logg + srow + s) : 0.f;
          lg_cur = __shfl_sync(0xffffffffu, v, __ffs(m) - 1);
          break;
        }
      }
    }
    for (int h = w4; h < G; h += 4) {
      float dot = 0.f;
      if (seq_ok) {
        const int Hk = a.Hkv, kh = sh / a.R;
        const size_t own = a.pt != nullptr ? ((size_t)own_page * Hk + kh) * kB + (L - 1) % kB
                                           : ((size_t)b * Hk + kh) * a.capacity + (L - 1);
        const uint2 kr = *reinterpret_cast<const uint2*>(a.kc + own * kD + lane * 4);
        const uint2 qr = *reinterpret_cast<const uint2*>(a.q + ((size_t)b * a.Hq + sh * G + h) * kD + lane * 4);
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
  const int nblk = *nblk_s;
  const int npairs = (nblk + 1) >> 1;

  if (warp == 0) {
    // ---------------- K/V loads ----------------
    if (lane == 0) {
      for (; issued < 2 * npairs && !*abort_flag; ++issued)
        if (!load_kv(issued, nblk)) {
          fz_fail(a, 81, abort_flag);
          break;
        }
      for (int i = max(0, issued - kSlots); i < issued; ++i) {   // none in flight at exit
        const uint32_t gi = rc.ring + i;
        mbar_wait_drain(full + gi % kSlots, (gi / kSlots) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, kN, false, false);   // S^T = K Q^T
      constexpr uint32_t kIdO = idesc_bf16_f32(128, kN, true, false);    // O^T += V^T P
      const uint32_t q_addr = smem_u32(sm + OFF_Q);
      bool ok = true;
      auto pv = [&](int m) -> bool {
        const uint32_t gvi = rc.ring + 2 * m + 1, vslot = gvi % kSlots, gm = rc.pair + m;
        if (!mbar_wait(full + vslot, (gvi / kSlots) & 1, abort_flag)) return false;
        if (!mbar_wait(p_full + (gm & 1), (gm >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm + OFF_STAGE + vslot * kKV);
        const uint32_t p_addr = smem_u32(sm + OFF_P + (gm & 1) * 2 * kN * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kColO, sdesc_sw128(v_addr + kk * 2048, kHalfPair, 1024),
                      sdesc_sw128(p_addr + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024),
                      kIdO, (m > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty + vslot);
        tc_commit(p_empty + (gm & 1));
        return true;
      };
      for (int n = 0; n < npairs; ++n) {
        const uint32_t gn = rc.pair + n, st = gn & 1, gki = rc.ring + 2 * n, kslot = gki % kSlots;
        if (!mbar_wait(full + kslot, (gki / kSlots) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm + OFF_STAGE + kslot * kKV);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + kColS + st * kN,
                      sdesc_sw128(k_addr + (kk >> 2) * kHalfPair + (kk & 3) * 32, 16, 1024),
                      sdesc_sw128(q_addr + (kk >> 2) * (kN * 128) + (kk & 3) * 32, 16, 1024),
                      kIdS, kk > 0 ? 1u : 0u);
        tc_commit(s_full + st);
        tc_commit(empty + kslot);
        if (n >= 1 && !pv(n - 1)) { ok = false; break; }
      }
      if (ok && npairs >= 1 && !pv(npairs - 1)) ok = false;
      if (!ok) fz_fail(a, 82, abort_flag);
      tc_commit(final_bar);
      mbar_wait_drain(final_bar, rc.fin & 1);
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
      const uint32_t gn = rc.pair + n, st = gn & 1;
      if (!warp_wait(s_full + st, (gn >> 1) & 1, abort_flag)) { ok = false; break; }
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
      if (gn >= 2 && !warp_wait(p_empty + st, ((gn >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
      uint8_t* pb = sm + OFF_P + st * 2 * kN * 128 + (r >> 6) * (kN * 128);
      const int kk = r & 63;
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G)
          *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((((kk >> 3) ^ (h & 7)) << 4) | ((kk & 7) << 1))) =
              __float2bfloat16_rn(p[h]);
      const uint32_t gvi = rc.ring + 2 * n + 1, vslot = gvi % kSlots;
      if (__any_sync(0xffffffffu, !valid) && !warp_wait(full + vslot, (gvi / kSlots) & 1, abort_flag)) {
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
    if (!ok) fz_fail(a, 83, abort_flag);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float v = warp_sum(lsum[h]);
      if (lane == 0 && h < G) red[(warp - 4) * kN + h] = v;
    }
    const bool have = ok && npairs >= 1 && warp_wait(final_bar, rc.fin & 1, abort_flag);
    float o[kN];
    if (have) {
      tc_fence_after();
      tmem_ld16(tmem + lane_addr + kColO, o);
    }
    named_bar(1, 128);
    const size_t prow = (((size_t)b * a.Hs + sh) * a.ns + split) * G;
    for (int h = 0; h < G; ++h) a.part_acc[(prow + h) * kD + r] = have ? o[h] : 0.f;
    if (r < G) {
      const float l = red[r] + red[kN + r] + red[2 * kN + r] + red[3 * kN + r];
      const bool any = have && l > 0.f;
      a.part_ml[(prow + r) * 2] = any ? mref[r] : -INFINITY;
      a.part_ml[(prow + r) * 2 + 1] = any ? l : 0.f;
      if (any && !isfinite(l)) atomicCAS(a.hdr + kHdrErr, 0, 61);
    }
    __threadfence();
  }
  rc.ring += 2 * npairs;
  rc.pair += npairs;
  rc.fin += 1;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---------------- merge of the row's splits by the last one to finish ----------------
  if (tid == 0) {
    const int prev = atomicAdd(a.done + (size_t)b * a.Hs + sh, 1);
    *last_s = prev == a.ns - 1;
    __threadfence();
  }
  __syncthreads();
  if (*last_s) {
    for (int e = tid; e < G * kD; e += kThreads) {
      const int g = e / kD, ch = e - g * kD;
      const size_t r0 = ((size_t)b * a.Hs + sh) * a.ns;
      float M = -INFINITY;
      for (int sp = 0; sp < a.ns; ++sp) M = fmaxf(M, __ldcg(a.part_ml + ((r0 + sp) * G + g) * 2));
      float ls = 0.f, as = 0.f;
      for (int sp = 0; sp < a.ns; ++sp) {
        const size_t pr = (r0 + sp) * G + g;
        const float mm = __ldcg(a.part_ml + pr * 2);
        if (mm == -INFINITY) continue;
        const float f = exp2f(mm - M);
        ls += __ldcg(a.part_ml + pr * 2 + 1) * f;
        as += __ldcg(a.part_acc + pr * kD + ch) * f;
      }
      // a head outside the fixed reference's range (error 61: ls overflowed) is written as 0
      a.o[((size_t)b * a.Hq + sh * G + g) * kD + ch] =
          __float2bfloat16_rn(ls > 0.f && isfinite(ls) ? as / ls : 0.f);
    }
  }
}

}  // namespace

// 120 registers per thread: two 256-thread CTAs per SM (at 128 the occupancy calculation admits
// one, and the persistent grid would run at half the planned concurrency)
template <int H, int NPT>
__global__ void __maxnreg__(120)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const FzArgs a) {
  using namespace dfz;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* gfull = bars + 2 * kSlots + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  int* item_s = reinterpret_cast<int*>(sm + OFF_MISC + 16);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kNumBars; ++i)   // p_full counts the 128 P lanes, the rest one arrival
      mbar_init(bars + i, (i == 2 * kSlots + 2 || i == 2 * kSlots + 3) ? 128 : 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  RingCounters rc{0u, 0u, 0u};
  uint32_t gk_n = 0;
  const int total = a.nP + a.nS + a.nA;
  while (true) {
    if (tid == 0) *item_s = ld_volatile(a.hdr + kHdrAbort) ? total : atomicAdd(a.hdr + kHdrNext, 1);
    __syncthreads();
    const int it = *item_s;
    __syncthreads();
    if (it >= total || *abort_flag) break;
    if (it < a.nP) {   // (4-sequence chunk, gate head, part)
      const int part = it & 1, rest = it >> 1;
      proj_item<H>(a, sm, rest % a.Hs, part, rest / a.Hs);
    } else if (it < a.nP + a.nS) {
      const int s = it - a.nP;
      select_item<H, NPT>(a, sm, gfull, gk_n, s / a.Hs, s % a.Hs, abort_flag);
    } else {
      const int t = it - a.nP - a.nS;
      const int split = t % a.ns, rest = t / a.ns;
      attn_item(a, &tmK, &tmV, sm, tmem, rc, rest / a.Hs, rest % a.Hs, split, abort_flag);
    }
    fence_async_smem();   // generic writes of this item before any async-proxy write of the next
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
namespace {
struct FzLayout {
  size_t hdr, pflag, sflag, done, sel_idx, sel_logg, gq, part_ml, part_acc, total, clear_bytes;
  int ns, nchunk;
};

int fused_nsplit(const sas_decode_problem& p) {
  const int K1 = p.topk + 1;
  const long rows = (long)p.batch * gate_heads(p);
  int ns = (K1 + 15) / 16;                                    // about 8 pairs per split
  const int want = (int)((2 * 2 * 148 + rows - 1) / rows);    // at least two items per CTA
  if (ns < want) ns = want;
  const int cap = (K1 + 1) / 2;                               // at least one pair per split
  if (ns > cap) ns = cap;
  return ns < 1 ? 1 : ns;
}

FzLayout fused_layout(const sas_decode_problem& p) {
  FzLayout l;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const int Hs = gate_heads(p), G = p.num_q_heads / Hs;
  const size_t rows = (size_t)p.batch * Hs;
  l.ns = fused_nsplit(p);
  l.nchunk = (p.batch + dfz::kPB - 1) / dfz::kPB;
  size_t o = 0;
  l.hdr = o; o += 256;
  l.pflag = o; o += (size_t)l.nchunk * Hs * 4;
  l.sflag = o; o += rows * 4;
  l.done = o; o += rows * 4;
  o = al(o);
  l.clear_bytes = o;
  l.sel_idx = o; o += al(rows * (p.topk + 1) * 4);
  l.sel_logg = o; o += al(rows * (p.topk + 1) * 4);
  l.gq = o; o += al(rows * 2 * p.gate_hidden * 4);
  l.part_ml = o; o += al(rows * l.ns * G * 2 * 4);
  l.part_acc = o; o += al(rows * l.ns * G * 128 * 4);
  l.total = o;
  return l;
}
}  // namespace

bool decode_fused_supported(const sas_decode_problem& p) {
  const int Hs = gate_heads(p);
  const int G = p.num_q_heads / Hs;
  const int nbmax = (p.capacity + p.block - 1) / p.block;
  return tma_available() && p.dtype == SAS_BF16 && p.head_dim == 128 && p.block == 64 && G <= 8 &&
         p.topk + 1 <= 128 && (p.gate_hidden == 64 || p.gate_hidden == 128) && nbmax <= dfz::kMaxNB;
}

size_t decode_fused_workspace_bytes(const sas_decode_problem& p) { return fused_layout(p).total; }

template <int H, int NPT>
static sas_status launch_fused_hn(const CUtensorMap& tk, const CUtensorMap& tv, const FzArgs& a, cudaStream_t st) {
  static int grid = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(decode_fused_kernel<H, NPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         dfz::kSmemBytes);
    // two CTAs per SM need nearly all of the SM's shared memory: ask for the largest carveout
    cudaFuncSetAttribute(decode_fused_kernel<H, NPT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         100);
    // CTAs per SM from the SM's shared memory and registers (the occupancy query returns one
    // for this kernel, while two run side by side and halve the step time)
    int dev = 0, sms = 0, sm_smem = 0, reserved = 0, sm_regs = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaDeviceGetAttribute(&sm_regs, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    cudaFuncAttributes fa;
    cudaFuncGetAttributes(&fa, decode_fused_kernel<H, NPT>);
    const int by_smem = sm_smem / (dfz::kSmemBytes + reserved);
    const int by_regs = sm_regs / (fa.numRegs * dfz::kThreads);
    const int per_sm = by_smem < by_regs ? by_smem : by_regs;   // 2 (shared memory)
    grid = sms * (per_sm > 0 ? per_sm : 1);
  });
  const int total = a.nP + a.nS + a.nA;
  const int g = total < grid ? total : grid;
  decode_fused_kernel<H, NPT><<<g, dfz::kThreads, dfz::kSmemBytes, st>>>(tk, tv, a);
  return SAS_OK;
}

sas_status launch_decode_fused(const sas_decode_problem& p, const void* q, const void* q_nope,
                               const void* k_cache, const void* v_cache, const void* gkc,
                               const float* cur_pool, const void* wq, const float* qnorm_w,
                               const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                               float* logg_out, void* ws, const DecodePaging& pg, cudaStream_t st) {
  const FzLayout l = fused_layout(p);
  char* w = (char*)ws;
  // the header (word 0: this call's error code), the item counter and the flags start at zero
  if (cudaMemsetAsync(w, 0, l.clear_bytes, st) != cudaSuccess) {
    set_error("decode: clearing the workspace header failed");
    return SAS_ERR_CUDA;
  }
  CUtensorMap tk, tv;
  const uint64_t rows = pg.pt != nullptr ? (uint64_t)pg.num_pages * p.num_kv_heads
                                         : (uint64_t)p.batch * p.num_kv_heads;
  const uint64_t keys = pg.pt != nullptr ? (uint64_t)dfz::kB : (uint64_t)p.capacity;
  if (!make_tmap_bf16_3d(&tk, k_cache, 128, keys, rows, 64, 64, 1) ||
      !make_tmap_bf16_3d(&tv, v_cache, 128, keys, rows, 64, 64, 1)) {
    set_error("decode: TMA descriptor creation failed");
    return SAS_ERR_CUDA;
  }
  const int Hs = gate_heads(p);
  FzArgs a;
  a.q = (const __nv_bfloat16*)q;
  a.q_nope = (const __nv_bfloat16*)q_nope;
  a.kc = (const __nv_bfloat16*)k_cache;
  a.gkc = (const __nv_bfloat16*)gkc;
  a.cur_pool = cur_pool;
  a.wq = (const __nv_bfloat16*)wq;
  a.qnorm_w = qnorm_w;
  a.wk = (const __nv_bfloat16*)wk;
  a.knorm_w = knorm_w;
  a.seqlens = p.seqlens;
  a.rc = p.gate_rope_cos;
  a.rs = p.gate_rope_sin;
  a.pt = pg.pt;
  a.num_pages = pg.num_pages;
  a.o = (__nv_bfloat16*)o;
  a.idx_out = idx_out;
  a.logg_out = logg_out;
  a.hdr = (int*)(w + l.hdr);
  a.pflag = (int*)(w + l.pflag);
  a.sflag = (int*)(w + l.sflag);
  a.done = (int*)(w + l.done);
  a.sel_idx = (int32_t*)(w + l.sel_idx);
  a.sel_logg = (float*)(w + l.sel_logg);
  a.gq = (float*)(w + l.gq);
  a.part_ml = (float*)(w + l.part_ml);
  a.part_acc = (float*)(w + l.part_acc);
  a.batch = p.batch;
  a.Hq = p.num_q_heads;
  a.Hkv = p.num_kv_heads;
  a.Hs = Hs;
  a.G = p.num_q_heads / Hs;
  a.R = Hs / p.num_kv_heads;
  a.K = p.topk;
  a.capacity = p.capacity;
  a.nbmax = (p.capacity + p.block - 1) / p.block;
  a.ns = l.ns;
  a.ungated = p.ungated;
  a.nP = l.nchunk * Hs * 2;
  a.nS = p.batch * Hs;
  a.nA = p.batch * Hs * l.ns;
  a.eps = p.rms_eps;
  a.scale_log2 = kLog2e / sqrtf(128.f);
  const int nbmax = a.nbmax;
#define SAS_FZ(H)                                                      \
  {                                                                    \
    if (nbmax <= 256) return launch_fused_hn<H, 1>(tk, tv, a, st);     \
    if (nbmax <= 1024) return launch_fused_hn<H, 4>(tk, tv, a, st);    \
    return launch_fused_hn<H, 8>(tk, tv, a, st);                       \
  }
  if (p.gate_hidden == 64) SAS_FZ(64)
  SAS_FZ(128)
#undef SAS_FZ
}

}  // namespace sas
