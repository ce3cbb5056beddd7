// Construction of the inverted selection lists of the key-major attention passes (layout in
// sas_km.cuh). Five launches and a clear, no host synchronisation:
//   count  CTA per (window quarter, sequence, kv head): shared-memory histogram of the kept
//          blocks of 1024 tokens; per-quarter counts, entry totals by global atomics
//   scan   exclusive scan of the entry totals (per-chunk totals, a scan of those, per-chunk
//          writes), ascending list of non-empty entries
//   fill   CTA per (window quarter, sequence, kv head): every kept (token, block) pair placed
//          at its entry's offset + the counts of the window's earlier quarters + a per-entry
//          cursor, 64 tokens at a time staged in shared memory by block (order inside an
//          entry arbitrary)
#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_km.cuh"

namespace sas {

constexpr int kQuarters = 4;   // CTAs per window
constexpr int kQTok = km::kW / kQuarters;

// Histogram of the blocks kept by the tokens of quarter q of window w of sequence b, kv head
// kv: cnt_q[e][q] for every entry of the window (zeros included), cnt[e] += (cleared before).
__global__ void km_count_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cu,
                                int batch, int Hkv, int K, int P, int* __restrict__ cnt,
                                int* __restrict__ cnt_q) {
  __shared__ int hist[km::kMaxBins];
  const int w = blockIdx.x / kQuarters, qt = blockIdx.x - w * kQuarters;
  const int b = blockIdx.y, kv = blockIdx.z;
  const int nbins = km::kWB * (w + 1);
  for (int j = threadIdx.x; j < nbins; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int t0 = w * km::kW + qt * kQTok, t1 = min(L, t0 + kQTok);
  const int K1 = K + 1;
  for (int e = threadIdx.x; e < (t1 - t0) * K1; e += blockDim.x) {   // empty when t0 >= L
    const int tl = t0 + e / K1, s = e - (e / K1) * K1;
    const int j = idx[((size_t)(s0 + tl) * Hkv + kv) * K1 + s];
    if (j >= 0 && j < nbins) atomicAdd(&hist[j], 1);
  }
  __syncthreads();
  const int base = km::entry(kv, b, w, 0, batch, P);
  for (int j = threadIdx.x; j < nbins; j += blockDim.x) {
    const int h = hist[j];
    cnt_q[(size_t)(base + j) * kQuarters + qt] = h;
    if (h) atomicAdd(cnt + base + j, h);
  }
}

// Exclusive scan of the E entry counts in three launches (chunks of kScanChunk entries per CTA):
// per-chunk totals of the pairs and of the non-empty entries; one CTA scans the chunk totals;
// every chunk writes its entries' offsets and its non-empty entries, ascending, into `items`.
// ctl[0] = the number of non-empty entries; ctl[1] (the work counter of the main kernels) = 0.
constexpr int kScanThreads = 1024, kScanPer = 4, kScanChunk = kScanThreads * kScanPer;

// block-wide inclusive scan of (a, b) over kScanThreads threads; returns the block totals
__device__ __forceinline__ int2 block_scan2(int& a, int& b, int2* ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) { a += x; b += y; }
  }
  if (lane == 31) ws[warp] = make_int2(a, b);
  __syncthreads();
  if (warp == 0) {
    int2 v = ws[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, v.x, o), y = __shfl_up_sync(0xffffffffu, v.y, o);
      if (lane >= o) { v.x += x; v.y += y; }
    }
    ws[lane] = v;   // inclusive over warps
  }
  __syncthreads();
  if (warp > 0) { a += ws[warp - 1].x; b += ws[warp - 1].y; }
  const int2 tot = ws[31];
  __syncthreads();   // ws is reused by the caller's next scan
  return tot;
}

__global__ void __launch_bounds__(kScanThreads) km_scan_chunks_kernel(const int* __restrict__ cnt, int E,
                                                                     int2* __restrict__ chunk_tot) {
  __shared__ int2 ws[32];
  const int e0 = blockIdx.x * kScanChunk + threadIdx.x * kScanPer;
  int sc = 0, sn = 0;
#pragma unroll
  for (int u = 0; u < kScanPer; ++u) {
    const int c = e0 + u < E ? cnt[e0 + u] : 0;
    sc += c;
    sn += c > 0;
  }
  const int2 tot = block_scan2(sc, sn, ws);
  if (threadIdx.x == 0) chunk_tot[blockIdx.x] = tot;
}

// exclusive scan of the nchunk chunk totals in place (one CTA)
__global__ void __launch_bounds__(kScanThreads) km_scan_top_kernel(int2* __restrict__ chunk_tot, int nchunk,
                                                                  int* __restrict__ ctl) {
  __shared__ int2 ws[32];
  const int per = (nchunk + kScanThreads - 1) / kScanThreads;
  const int c0 = min(nchunk, (int)threadIdx.x * per), c1 = min(nchunk, c0 + per);
  int sc = 0, sn = 0;
  for (int c = c0; c < c1; ++c) { sc += chunk_tot[c].x; sn += chunk_tot[c].y; }
  int ic = sc, in = sn;
  const int2 tot = block_scan2(ic, in, ws);
  int rc = ic - sc, rn = in - sn;
  for (int c = c0; c < c1; ++c) {
    const int2 t = chunk_tot[c];
    chunk_tot[c] = make_int2(rc, rn);
    rc += t.x;
    rn += t.y;
  }
  if (threadIdx.x == 0) {
    ctl[0] = tot.y;
    ctl[1] = 0;
  }
}

__global__ void __launch_bounds__(kScanThreads) km_scan_write_kernel(const int* __restrict__ cnt, int E,
                                                                    const int2* __restrict__ chunk_off,
                                                                    int* __restrict__ off,
                                                                    int* __restrict__ items) {
  __shared__ int2 ws[32];
  const int e0 = blockIdx.x * kScanChunk + threadIdx.x * kScanPer;
  int c[kScanPer], sc = 0, sn = 0;
#pragma unroll
  for (int u = 0; u < kScanPer; ++u) {
    c[u] = e0 + u < E ? cnt[e0 + u] : 0;
    sc += c[u];
    sn += c[u] > 0;
  }
  int ic = sc, in = sn;
  block_scan2(ic, in, ws);
  const int2 base = chunk_off[blockIdx.x];
  int rc = base.x + ic - sc, rn = base.y + in - sn;
#pragma unroll
  for (int u = 0; u < kScanPer; ++u) {
    if (e0 + u < E) {
      off[e0 + u] = rc;
      if (c[u] > 0) items[rn++] = e0 + u;
    }
    rc += c[u];
  }
}

// Place every kept (token, block) pair of quarter q of window w at its entry's next free
// position: entry offset + the earlier quarters' counts + a cursor per entry. The quarter is
// taken 64 tokens at a time: the pairs are counted per block (their shared-atomic return value is
// their rank in the block), the counts scanned, the pairs staged in shared memory grouped by
// block and then written out in that order, so each block's pairs of the 64 tokens land in one
// contiguous run of the list instead of as scattered 8-byte stores.
constexpr int kFillThreads = 512;
constexpr int kFillTok = 64;                        // tokens per staging round
constexpr int kFillPer = kFillTok * 128 / kFillThreads;   // pairs per thread per round (K + 1 <= 128)
// shared memory: three per-block arrays, the staged pairs and their list positions (K + 1 per
// token), scan partials
static size_t fill_smem(int K1) { return (size_t)3 * km::kMaxBins * 4 + (size_t)kFillTok * K1 * 12 + 64; }

__global__ void __launch_bounds__(kFillThreads) km_fill_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ logg, const int32_t* __restrict__ cu,
    int batch, int Hkv, int K, int P, const int* __restrict__ off, const int* __restrict__ cnt_q,
    int2* __restrict__ list) {
  extern __shared__ int fsm[];
  int* cur = fsm;                          // [kMaxBins] next list position of each block
  int* lcnt = cur + km::kMaxBins;          // [kMaxBins] this round's pairs per block
  int* loff = lcnt + km::kMaxBins;         // [kMaxBins] their start in the staging buffer
  const int K1 = K + 1, cap = kFillTok * K1;
  int2* stage = reinterpret_cast<int2*>(loff + km::kMaxBins);   // [cap]
  int* gpos = reinterpret_cast<int*>(stage + cap);                // [cap] list position
  int* wsum = gpos + cap;                                         // [16] scan partials
  const int w = blockIdx.x / kQuarters, qt = blockIdx.x - w * kQuarters;
  const int b = blockIdx.y, kv = blockIdx.z;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int t0 = w * km::kW + qt * kQTok, t1 = min(L, t0 + kQTok);
  if (t0 >= L) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nbins = km::kWB * (w + 1);
  const int base = km::entry(kv, b, w, 0, batch, P);
  for (int j = tid; j < nbins; j += kFillThreads) {
    int o = off[base + j];
    for (int q = 0; q < qt; ++q) o += cnt_q[(size_t)(base + j) * kQuarters + q];
    cur[j] = o;
  }
  for (int r0 = t0; r0 < t1; r0 += kFillTok) {
    const int npair = (min(t1, r0 + kFillTok) - r0) * K1;
    for (int j = tid; j < nbins; j += kFillThreads) lcnt[j] = 0;
    __syncthreads();
    int jj[kFillPer], rk[kFillPer];
#pragma unroll
    for (int u = 0; u < kFillPer; ++u) {   // count, and the pair's rank within its block
      const int e = tid + u * kFillThreads;
      jj[u] = -1;
      if (e < npair) {
        const int tl = r0 + e / K1, sl = e - (e / K1) * K1;
        const int j = idx[((size_t)(s0 + tl) * Hkv + kv) * K1 + sl];
        if (j >= 0 && j < nbins) {
          jj[u] = j;
          rk[u] = atomicAdd(&lcnt[j], 1);
        }
      }
    }
    __syncthreads();
    {   // exclusive scan of lcnt[0..nbins) into loff (each thread 4 consecutive blocks)
      constexpr int kPerT = km::kMaxBins / kFillThreads;
      int v[kPerT], sum = 0;
#pragma unroll
      for (int u = 0; u < kPerT; ++u) {
        const int j = tid * kPerT + u;
        v[u] = j < nbins ? lcnt[j] : 0;
        sum += v[u];
      }
      int inc = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
      }
      if (lane == 31) wsum[warp] = inc;
      __syncthreads();
      int wbase = 0;
      for (int q = 0; q < warp; ++q) wbase += wsum[q];
      int run = wbase + inc - sum;
#pragma unroll
      for (int u = 0; u < kPerT; ++u) {
        const int j = tid * kPerT + u;
        if (j < nbins) loff[j] = run;
        run += v[u];
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kFillPer; ++u) {   // stage grouped by block
      if (jj[u] >= 0) {
        const int e = tid + u * kFillThreads;
        const int tl = r0 + e / K1, sl = e - (e / K1) * K1;
        const size_t gi = ((size_t)(s0 + tl) * Hkv + kv) * K1 + sl;
        const int slot = loff[jj[u]] + rk[u];
        stage[slot] = make_int2((s0 + tl) | (sl << 24), __float_as_int(logg[gi]));
        gpos[slot] = cur[jj[u]] + rk[u];
      }
    }
    __syncthreads();
    int nvalid = 0;   // = sum of lcnt: the last block's offset plus its count
    if (nbins > 0) nvalid = loff[nbins - 1] + lcnt[nbins - 1];
    for (int i = tid; i < nvalid; i += kFillThreads) list[gpos[i]] = stage[i];
    __syncthreads();
    for (int j = tid; j < nbins; j += kFillThreads) cur[j] += lcnt[j];
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------
static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

static void km_dims(const sas_problem& p, int* nW, int* P, int* E) {
  *nW = (p.max_seqlen + km::kW - 1) / km::kW;
  *P = km::kWB * (*nW * (*nW + 1) / 2);
  *E = gate_heads(p) * p.batch * *P;   // entries per gate head
}

bool km_supported(const sas_problem& p) {
  const int NBmax = (p.max_seqlen + p.block - 1) / p.block;
  return p.block == km::kB && p.max_seqlen <= km::kW * 32 && NBmax <= km::kMaxBins &&
         p.total_tokens < (1 << 24) && p.topk + 1 <= 128;
}

size_t km_lists_bytes(const sas_problem& p) {
  int nW, P, E;
  km_dims(p, &nW, &P, &E);
  const size_t nchunk = ((size_t)E + kScanChunk - 1) / kScanChunk;
  return 3 * al256((size_t)E * 4) + al256((size_t)E * kQuarters * 4) + 256 + al256(nchunk * 8) +
         al256((size_t)p.total_tokens * gate_heads(p) * (p.topk + 1) * 8);
}

KmLists km_lists_carve(const sas_problem& p, uint8_t* base) {
  KmLists L;
  km_dims(p, &L.nW, &L.P, &L.E);
  size_t o = 0;
  L.cnt = reinterpret_cast<int*>(base + o);   o += al256((size_t)L.E * 4);
  L.off = reinterpret_cast<int*>(base + o);   o += al256((size_t)L.E * 4);
  L.items = reinterpret_cast<int*>(base + o); o += al256((size_t)L.E * 4);
  L.cnt_q = reinterpret_cast<int*>(base + o); o += al256((size_t)L.E * kQuarters * 4);
  L.ctl = reinterpret_cast<int*>(base + o);   o += 256;
  L.chunk = reinterpret_cast<int2*>(base + o);
  o += al256((((size_t)L.E + kScanChunk - 1) / kScanChunk) * 8);
  L.list = reinterpret_cast<int2*>(base + o);
  return L;
}

sas_status launch_km_lists(const sas_problem& p, const int32_t* idx, const float* logg,
                           const KmLists& L, cudaStream_t st) {
  const dim3 wgrid(L.nW * kQuarters, p.batch, gate_heads(p));
  if (cudaMemsetAsync(L.cnt, 0, (size_t)L.E * 4, st) != cudaSuccess) {
    set_error("key-major lists: clearing the counts failed");
    return SAS_ERR_CUDA;
  }
  km_count_kernel<<<wgrid, 512, 0, st>>>(idx, p.cu_seqlens, p.batch, gate_heads(p), p.topk, L.P,
                                         L.cnt, L.cnt_q);
  const int nchunk = (L.E + kScanChunk - 1) / kScanChunk;
  km_scan_chunks_kernel<<<nchunk, kScanThreads, 0, st>>>(L.cnt, L.E, L.chunk);
  km_scan_top_kernel<<<1, kScanThreads, 0, st>>>(L.chunk, nchunk, L.ctl);
  km_scan_write_kernel<<<nchunk, kScanThreads, 0, st>>>(L.cnt, L.E, L.chunk, L.off, L.items);
  static std::once_flag fill_once;
  std::call_once(fill_once, [] {
    cudaFuncSetAttribute(km_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fill_smem(128));
  });
  km_fill_kernel<<<wgrid, kFillThreads, fill_smem(p.topk + 1), st>>>(idx, logg, p.cu_seqlens, p.batch, gate_heads(p),
                                                         p.topk, L.P, L.off, L.cnt_q, L.list);
  return launch_status("key-major selection lists", 5);
}

int sm_count() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  });
  return n;
}

}  // namespace sas
