// Internal launcher declarations (host side) shared by the C ABI implementation.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda.h>
#include <vector_types.h>

#include "sas.h"

namespace sas {

// Gate (selection) heads: one gate per KV head (default) or one per query head.
inline int gate_heads(const sas_problem& p) {
  return p.gate_heads > 0 ? p.gate_heads : p.num_kv_heads;
}
inline int gate_heads(const sas_decode_problem& p) {
  return p.gate_heads > 0 ? p.gate_heads : p.num_kv_heads;
}

sas_status launch_pool_keys(const sas_problem& p, const void* k_nope, float* pooled, cudaStream_t st);
sas_status launch_gate_keys(const sas_problem& p, const float* pooled, const void* wk,
                            const float* knorm_w, float* gkeys, cudaStream_t st);
size_t gate_scores_workspace_bytes(const sas_problem& p);
sas_status launch_gate_scores(const sas_problem& p, const void* q_nope, const void* k_nope,
                              const float* gkeys, const void* wq, const float* qnorm_w,
                              const void* wk, const float* knorm_w, float* scores, float* lse,
                              void* workspace, cudaStream_t st);
bool gate_select_fused(const sas_problem& p);
size_t gate_select_workspace_bytes(const sas_problem& p);
sas_status launch_gate_select(const sas_problem& p, const void* q_nope, const void* k_nope,
                              const float* gkeys, const void* wq, const float* qnorm_w,
                              const void* wk, const float* knorm_w, int32_t* idx, float* logg,
                              float* lse, void* workspace, cudaStream_t st);
sas_status launch_topk(const sas_problem& p, const float* scores, const float* lse, int32_t* idx,
                       float* logg, cudaStream_t st);
bool gate_bwd_supported(const sas_problem& p);
size_t gate_bwd_workspace_bytes(const sas_problem& p);
sas_status launch_gate_bwd(const sas_problem& p, const void* q_nope, const void* k_nope,
                           const float* pooled, const void* wq, const float* qnorm_w,
                           const void* wk, const float* knorm_w, const int32_t* idx,
                           const float* dlogg, float* dwq, float* dqnorm_w, float* dwk,
                           float* dknorm_w, void* workspace, cudaStream_t st);

sas_status launch_attn_fwd_simt(const sas_problem& p, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* logg, void* o, float* lse,
                                cudaStream_t st);
sas_status launch_attn_bwd_simt(const sas_problem& p, const void* q, const void* k, const void* v,
                                const void* o, const void* dout, const float* lse,
                                const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                                float* dlogg, float* drow, cudaStream_t st);

bool attn_tc_supported(const sas_problem& p);
int tc_rows_per_tile(int G);
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                       uint32_t b0, uint32_t b1, uint32_t b2);
bool make_tmap_f32_3d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                      uint32_t b0, uint32_t b1, uint32_t b2);
sas_status launch_rowdot(const sas_problem& p, const void* o, const void* dout, float* drow,
                         cudaStream_t st);

// inverted selection lists of the key-major passes (sas_km.cuh)
struct KmLists {
  int* cnt;
  int* off;
  int* items;
  int* cnt_q;    // per entry and window quarter
  int* ctl;      // [0] non-empty entries, [1] work counter
  int2* chunk;   // scan scratch: per-chunk totals, then offsets
  int2* list;
  int nW, P, E;
};
bool km_supported(const sas_problem& p);
size_t km_lists_bytes(const sas_problem& p);
KmLists km_lists_carve(const sas_problem& p, uint8_t* base);
sas_status launch_km_lists(const sas_problem& p, const int32_t* idx, const float* logg,
                           const KmLists& L, cudaStream_t st);
int sm_count();

bool attn_fwd_km_supported(const sas_problem& p);
size_t attn_fwd_km_workspace_bytes(const sas_problem& p);
sas_status launch_attn_fwd_km(const sas_problem& p, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* logg, void* o, float* lse,
                              void* workspace, cudaStream_t st);

bool attn_bwd_km_supported(const sas_problem& p);
size_t attn_bwd_km_workspace_bytes(const sas_problem& p);
sas_status launch_attn_bwd_km(const sas_problem& p, const void* q, const void* k, const void* v,
                              const void* o, const void* dout, const float* lse,
                              const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                              float* dlogg, void* workspace, cudaStream_t st);

bool tma_available();
bool make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t n0, uint64_t n1,
                       uint64_t row_bytes, uint32_t b0, uint32_t b1);
bool make_tmap_f32_sw128(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                         const uint32_t* box);
bool gate_tc_supported(const sas_problem& p);
size_t gate_tc_workspace_bytes(const sas_problem& p);
// Historical gate scores on the tensor cores (sas_gate_hist_tc.cu): q~ and the block keys split
// into tf32 hi + lo parts, three tf32 products per element (hi.hi + hi.lo + lo.hi).
bool gate_hist_tc_supported(const sas_problem& p);
size_t gate_hist_tc_workspace_bytes(const sas_problem& p);   // key splits (ghi, glo)
sas_status launch_gate_hist_tc(const sas_problem& p, const float* gkeys, const float* qproj,
                               const float* kproj, const float* qnorm_w, const float* knorm_w,
                               float* qhi, float* qlo, void* key_ws, float* scores, float* lse,
                               int* err, cudaStream_t st);
sas_status launch_gate_proj_tc(const sas_problem& p, const void* q_nope, const void* k_nope,
                               const void* wq, const void* wk, void* workspace, float** qproj,
                               float** kproj, cudaStream_t st,
                               const void** prefix_rows = nullptr);
// Paged decode caches: pt = page table [batch, ceil(capacity / B)] (page of block j of
// sequence b), pages of [Hkv, B, d] keys / values and [Hkv, h] gate keys; pt == nullptr for
// the contiguous [batch, Hkv, capacity, d] layout.
struct DecodePaging {
  const int32_t* pt = nullptr;
  int num_pages = 0;
};
bool decode_attn_tc_supported(const sas_decode_problem& p);
sas_status launch_decode_attn_tc(const sas_decode_problem& p, const void* q, const void* kc,
                                 const void* vc, const int32_t* sel_idx, const float* sel_logg,
                                 float* part_ml, float* part_acc, int* err, int ns,
                                 const DecodePaging& pg, cudaStream_t st);

// Fused persistent decode (sas_decode_fused.cu): gate, Top-K, attention and merge in one launch.
bool decode_fused_supported(const sas_decode_problem& p);
size_t decode_fused_workspace_bytes(const sas_decode_problem& p);
sas_status launch_decode_fused(const sas_decode_problem& p, const void* q, const void* q_nope,
                               const void* k_cache, const void* v_cache, const void* gkc,
                               const float* cur_pool, const void* wq, const float* qnorm_w,
                               const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                               float* logg_out, void* ws, const DecodePaging& pg, cudaStream_t st);
// Process-wide choice between the fused decode and the three-launch decode (default: fused
// where supported).
bool decode_fused_enabled();

int decode_nsplit(const sas_decode_problem& p);
size_t decode_workspace_bytes(const sas_decode_problem& p);
sas_status launch_decode(const sas_decode_problem& p, const void* q, const void* q_nope,
                         const void* k_cache, const void* v_cache, const void* gkc,
                         const float* cur_pool, const void* wq, const float* qnorm_w,
                         const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                         float* logg_out, void* ws, const DecodePaging& pg, cudaStream_t st);

}  // namespace sas
