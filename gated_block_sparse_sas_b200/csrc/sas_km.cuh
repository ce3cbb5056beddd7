// Inverted selection lists shared by the key-major attention passes (forward and backward).
//
// The method keeps, per (token, kv head), K historical blocks plus the current block (README
// (b)). The key-major passes need the transpose: for a KV block j of a sequence, the tokens
// that kept it. Tokens are grouped into windows of 4096 so that the rows one pass touches at
// a time stay in L2. One entry per (kv head, sequence, window w, block j < 64 (w+1)):
//   e = (kv * batch + b) * P + 64 * w (w+1) / 2 + j,   P = 64 * nW (nW+1) / 2
// cnt[e] kept (token, block) pairs, off[e] their start in `list`; items = the non-empty
// entries in ascending order (so consecutive items share a window); list entries are
// (packed token index | slot << 24, log-gate bits).
#pragma once

#include "sas_common.cuh"

namespace sas {
namespace km {

constexpr int kB = 64;            // keys per block
constexpr int kW = 4096;          // tokens per window
constexpr int kWB = kW / kB;      // block steps per window (64)
constexpr int kMaxBins = 2048;    // blocks a window can see (max_seqlen <= 131072)

__host__ __device__ __forceinline__ int entry(int kv, int b, int w, int j, int batch, int P) {
  return (kv * batch + b) * P + kWB * (w * (w + 1) / 2) + j;
}

struct Item {
  int kv, b, w, j;
};

__device__ __forceinline__ Item decode(int e, int batch, int P) {
  Item it;
  const int kvb = e / P;
  const int rem = e - kvb * P;
  int w = 0;
  while (kWB * ((w + 1) * (w + 2) / 2) <= rem) ++w;
  it.w = w;
  it.j = rem - kWB * (w * (w + 1) / 2);
  it.kv = kvb / batch;
  it.b = kvb - it.kv * batch;
  return it;
}

}  // namespace km
}  // namespace sas
