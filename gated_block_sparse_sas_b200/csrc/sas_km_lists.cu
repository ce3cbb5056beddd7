// Construction of the inverted selection lists of the key-major attention passes (layout in
// sas_km.cuh). Three launches and a clear, no host synchronisation:
//   count  CTA per (window quarter, sequence, kv head): shared-memory histogram of the kept
//          blocks of 1024 tokens; per-quarter counts, entry totals by global atomics
//   scan   one CTA: exclusive scan of the entry totals, ascending list of non-empty entries
//   fill   CTA per (window quarter, sequence, kv head): every kept (token, block) pair placed
//          at its entry's offset + the counts of the window's earlier quarters + a shared
//          atomic cursor (order inside an entry arbitrary)
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

// Exclusive scan of the E counts (one CTA of 1024 threads); ascending list of the non-empty
// entries; ctl[0] = their number; ctl[1] (the work counter of the main kernels) = 0.
__global__ void __launch_bounds__(1024) km_scan_kernel(const int* __restrict__ cnt, int E,
                                                       int* __restrict__ off, int* __restrict__ items,
                                                       int* __restrict__ ctl) {
  __shared__ int ws_c[32], ws_n[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (E + 1023) / 1024;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int sc = 0, sn = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = cnt[e];
    sc += c;
    sn += c > 0;
  }
  int ic = sc, in = sn;   // inclusive warp scans
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ic, o), bb = __shfl_up_sync(0xffffffffu, in, o);
    if (lane >= o) { ic += a; in += bb; }
  }
  if (lane == 31) { ws_c[warp] = ic; ws_n[warp] = in; }
  __syncthreads();
  if (warp == 0) {
    int vc = ws_c[lane], vn = ws_n[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, vc, o), bb = __shfl_up_sync(0xffffffffu, vn, o);
      if (lane >= o) { vc += a; vn += bb; }
    }
    ws_c[lane] = vc;   // inclusive over warps
    ws_n[lane] = vn;
  }
  __syncthreads();
  int rc = ic - sc + (warp ? ws_c[warp - 1] : 0);
  int rn = in - sn + (warp ? ws_n[warp - 1] : 0);
  for (int e = e0; e < e1; ++e) {
    const int c = cnt[e];
    off[e] = rc;
    rc += c;
    if (c > 0) items[rn++] = e;
  }
  if (tid == 1023) {
    ctl[0] = ws_n[31];
    ctl[1] = 0;
  }
}

// Place every kept (token, block) pair of quarter q of window w at its entry's next free
// position: entry offset + the earlier quarters' counts + a shared atomic cursor.
__global__ void km_fill_kernel(const int32_t* __restrict__ idx, const float* __restrict__ logg,
                               const int32_t* __restrict__ cu, int batch, int Hkv, int K, int P,
                               const int* __restrict__ off, const int* __restrict__ cnt_q,
                               int2* __restrict__ list) {
  __shared__ int cur[km::kMaxBins];
  const int w = blockIdx.x / kQuarters, qt = blockIdx.x - w * kQuarters;
  const int b = blockIdx.y, kv = blockIdx.z;
  const int s0 = cu[b], L = cu[b + 1] - s0;
  const int t0 = w * km::kW + qt * kQTok, t1 = min(L, t0 + kQTok);
  if (t0 >= L) return;
  const int nbins = km::kWB * (w + 1);
  const int base = km::entry(kv, b, w, 0, batch, P);
  for (int j = threadIdx.x; j < nbins; j += blockDim.x) {
    int o = off[base + j];
    for (int q = 0; q < qt; ++q) o += cnt_q[(size_t)(base + j) * kQuarters + q];
    cur[j] = o;
  }
  __syncthreads();
  const int K1 = K + 1;
  for (int e = threadIdx.x; e < (t1 - t0) * K1; e += blockDim.x) {
    const int tl = t0 + e / K1, s = e - (e / K1) * K1;
    const size_t gi = ((size_t)(s0 + tl) * Hkv + kv) * K1 + s;
    const int j = idx[gi];
    if (j >= 0 && j < nbins) {
      const int pos = atomicAdd(&cur[j], 1);
      list[pos] = make_int2((s0 + tl) | (s << 24), __float_as_int(logg[gi]));
    }
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
  return 3 * al256((size_t)E * 4) + al256((size_t)E * kQuarters * 4) + 256 +
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
  km_scan_kernel<<<1, 1024, 0, st>>>(L.cnt, L.E, L.off, L.items, L.ctl);
  km_fill_kernel<<<wgrid, 512, 0, st>>>(idx, logg, p.cu_seqlens, p.batch, gate_heads(p), p.topk,
                                        L.P, L.off, L.cnt_q, L.list);
  return launch_status("key-major selection lists", 3);
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
