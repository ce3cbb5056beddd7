// C ABI of the gated block-sparse attention library: argument checks, workspace sizes,
// kernel selection, stream-ordered launches. Declarations and the operator's definition
// are in include/sas.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <string>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {

static thread_local std::string g_err;
static thread_local uint64_t g_launches = 0;

void count_launches(int n) { g_launches += (uint64_t)n; }

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
}

sas_status launch_status(const char* what, int launches) {
  count_launches(launches);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: launch failed: %s", what, cudaGetErrorString(e));
    return SAS_ERR_CUDA;
  }
  return SAS_OK;
}

static bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

static int max_blocks(const sas_problem& p) { return (p.max_seqlen + p.block - 1) / p.block; }

// Shape checks common to every prefill entry point.
static sas_status check_problem(const sas_problem* p, bool needs_rope) {
  SAS_CHECK_ARG(p != nullptr, "problem is NULL");
  SAS_CHECK_ARG(p->batch >= 1, "batch must be >= 1 (got %d)", p->batch);
  SAS_CHECK_ARG(p->total_tokens >= 0, "total_tokens must be >= 0 (got %d)", p->total_tokens);
  SAS_CHECK_ARG(p->max_seqlen >= 1, "max_seqlen must be >= 1 (got %d)", p->max_seqlen);
  SAS_CHECK_ARG(p->num_kv_heads >= 1 && p->num_q_heads >= p->num_kv_heads &&
                    p->num_q_heads % p->num_kv_heads == 0,
                "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)", p->num_q_heads,
                p->num_kv_heads);
  const int G = p->num_q_heads / p->num_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 5 || G == 8)) {
    set_error("query heads per KV head must be 1, 2, 4, 5 or 8 (got %d)", G);
    return SAS_ERR_UNSUPPORTED;
  }
  if (!(p->head_dim == 64 || p->head_dim == 128)) {
    set_error("head_dim must be 64 or 128 (got %d)", p->head_dim);
    return SAS_ERR_UNSUPPORTED;
  }
  if (!(p->block == 16 || p->block == 32 || p->block == 64)) {
    set_error("block must be 16, 32 or 64 (got %d)", p->block);
    return SAS_ERR_UNSUPPORTED;
  }
  if (!(p->gate_hidden == 32 || p->gate_hidden == 64 || p->gate_hidden == 128)) {
    set_error("gate_hidden must be 32, 64 or 128 (got %d)", p->gate_hidden);
    return SAS_ERR_UNSUPPORTED;
  }
  SAS_CHECK_ARG(p->topk >= 1 && p->topk + 1 <= 128, "topk must be in 1..127 (got %d)", p->topk);
  SAS_CHECK_ARG(p->dtype == SAS_BF16 || p->dtype == SAS_FP32, "unknown dtype %d", (int)p->dtype);
  SAS_CHECK_ARG(p->rms_eps >= 0.f && isfinite(p->rms_eps), "rms_eps must be finite and >= 0");
  SAS_CHECK_ARG(p->gate_heads == 0 || p->gate_heads == p->num_kv_heads ||
                    p->gate_heads == p->num_q_heads,
                "gate_heads must be 0, num_kv_heads (%d) or num_q_heads (%d) (got %d)",
                p->num_kv_heads, p->num_q_heads, p->gate_heads);
  if (max_blocks(*p) > 2048) {
    set_error("max_seqlen / block must be <= 2048 blocks (got %d)", max_blocks(*p));
    return SAS_ERR_UNSUPPORTED;
  }
  SAS_CHECK_ARG(p->cu_seqlens != nullptr, "cu_seqlens is NULL");
  if (needs_rope)
    SAS_CHECK_ARG(p->gate_rope_cos != nullptr && p->gate_rope_sin != nullptr,
                  "gate rotary tables are NULL");
  return SAS_OK;
}

// Word 0 of a workspace is the call's pipeline error code: cleared (stream-ordered) before the
// call's kernels, so after the stream completes it holds this call's code and no earlier one.
static sas_status clear_error_word(void* workspace, cudaStream_t stream) {
  if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), stream) != cudaSuccess) {
    set_error("clearing the workspace error word failed");
    return SAS_ERR_CUDA;
  }
  return SAS_OK;
}

#define SAS_PTR(ptr)                                                        \
  do {                                                                      \
    SAS_CHECK_ARG((ptr) != nullptr, "%s is NULL", #ptr);                    \
    SAS_CHECK_ARG(aligned16(ptr), "%s is not 16-byte aligned", #ptr);       \
  } while (0)

}  // namespace sas

using namespace sas;

extern "C" {

const char* sas_last_error(void) { return g_err.c_str(); }

uint64_t sas_kernel_launches(void) { return g_launches; }

sas_status sas_rope_tables(int32_t positions, int32_t rot_dim, double base, float* cos_out,
                           float* sin_out) {
  SAS_CHECK_ARG(positions >= 1, "positions must be >= 1");
  SAS_CHECK_ARG(rot_dim >= 2 && rot_dim % 2 == 0, "rot_dim must be even and >= 2");
  SAS_CHECK_ARG(base > 0.0, "base must be > 0");
  SAS_CHECK_ARG(cos_out != nullptr && sin_out != nullptr, "output buffers are NULL");
  const int half = rot_dim / 2;
  for (int i = 0; i < half; ++i) {
    const double inv_freq = pow(base, -2.0 * i / rot_dim);
    for (int64_t pos = 0; pos < positions; ++pos) {
      const double th = (double)pos * inv_freq;
      cos_out[pos * half + i] = (float)cos(th);
      sin_out[pos * half + i] = (float)sin(th);
    }
  }
  return SAS_OK;
}

sas_status sas_pool_keys(const sas_problem* p, const void* k_nope, float* pooled,
                         cudaStream_t stream) {
  SAS_TRY(check_problem(p, false));
  SAS_PTR(k_nope);
  SAS_PTR(pooled);
  return launch_pool_keys(*p, k_nope, pooled, stream);
}

sas_status sas_gate_keys(const sas_problem* p, const float* pooled, const void* wk,
                         const float* knorm_w, float* gate_keys, cudaStream_t stream) {
  SAS_TRY(check_problem(p, true));
  SAS_PTR(pooled);
  SAS_PTR(wk);
  SAS_PTR(knorm_w);
  SAS_PTR(gate_keys);
  return launch_gate_keys(*p, pooled, wk, knorm_w, gate_keys, stream);
}

sas_status sas_gate_scores_workspace_size(const sas_problem* p, size_t* bytes) {
  SAS_TRY(check_problem(p, true));
  SAS_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  *bytes = gate_scores_workspace_bytes(*p);
  return SAS_OK;
}

sas_status sas_gate_scores(const sas_problem* p, const void* q_nope, const void* k_nope,
                           const float* gate_keys, const void* wq, const float* qnorm_w,
                           const void* wk, const float* knorm_w, float* scores, float* lse,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  SAS_TRY(check_problem(p, true));
  SAS_PTR(q_nope);
  SAS_PTR(k_nope);
  SAS_PTR(gate_keys);
  SAS_PTR(wq);
  SAS_PTR(qnorm_w);
  SAS_PTR(wk);
  SAS_PTR(knorm_w);
  SAS_PTR(scores);
  SAS_PTR(lse);
  if (p->total_tokens == 0) return SAS_OK;
  SAS_PTR(workspace);
  const size_t need = gate_scores_workspace_bytes(*p);
  if (workspace_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
    return SAS_ERR_WORKSPACE;
  }
  SAS_TRY(clear_error_word(workspace, stream));
  return launch_gate_scores(*p, q_nope, k_nope, gate_keys, wq, qnorm_w, wk, knorm_w, scores, lse,
                            workspace, stream);
}

sas_status sas_gate_select_workspace_size(const sas_problem* p, size_t* bytes) {
  SAS_TRY(check_problem(p, true));
  SAS_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  *bytes = gate_select_workspace_bytes(*p);
  return SAS_OK;
}

sas_status sas_gate_select(const sas_problem* p, const void* q_nope, const void* k_nope,
                           const float* gate_keys, const void* wq, const float* qnorm_w,
                           const void* wk, const float* knorm_w, int32_t* idx, float* logg,
                           float* lse, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  SAS_TRY(check_problem(p, true));
  SAS_PTR(q_nope);
  SAS_PTR(k_nope);
  SAS_PTR(gate_keys);
  SAS_PTR(wq);
  SAS_PTR(qnorm_w);
  SAS_PTR(wk);
  SAS_PTR(knorm_w);
  SAS_PTR(idx);
  SAS_PTR(logg);
  if (lse != nullptr) SAS_CHECK_ARG(aligned16(lse), "lse is not 16-byte aligned");
  if (p->total_tokens == 0) return SAS_OK;
  SAS_PTR(workspace);
  const size_t need = gate_select_workspace_bytes(*p);
  if (workspace_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
    return SAS_ERR_WORKSPACE;
  }
  SAS_TRY(clear_error_word(workspace, stream));
  return launch_gate_select(*p, q_nope, k_nope, gate_keys, wq, qnorm_w, wk, knorm_w, idx, logg,
                            lse, workspace, stream);
}

sas_status sas_gate_bwd_workspace_size(const sas_problem* p, size_t* bytes) {
  SAS_TRY(check_problem(p, true));
  SAS_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  if (!gate_bwd_supported(*p)) {
    set_error("gate_bwd: supported for bf16, head_dim 128, gate_hidden 128, block <= 128, one gate per KV group");
    return SAS_ERR_UNSUPPORTED;
  }
  *bytes = gate_bwd_workspace_bytes(*p);
  return SAS_OK;
}

sas_status sas_gate_bwd(const sas_problem* p, const void* q_nope, const void* k_nope,
                        const float* pooled, const void* wq, const float* qnorm_w, const void* wk,
                        const float* knorm_w, const int32_t* idx, const float* dlogg, float* dwq,
                        float* dqnorm_w, float* dwk, float* dknorm_w, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  SAS_TRY(check_problem(p, true));
  SAS_PTR(q_nope);
  SAS_PTR(k_nope);
  SAS_PTR(pooled);
  SAS_PTR(wq);
  SAS_PTR(qnorm_w);
  SAS_PTR(wk);
  SAS_PTR(knorm_w);
  SAS_PTR(idx);
  SAS_PTR(dlogg);
  SAS_PTR(dwq);
  SAS_PTR(dqnorm_w);
  SAS_PTR(dwk);
  SAS_PTR(dknorm_w);
  if (!gate_bwd_supported(*p)) {
    set_error("gate_bwd: supported for bf16, head_dim 128, gate_hidden 128, block <= 128, one gate per KV group");
    return SAS_ERR_UNSUPPORTED;
  }
  if (p->total_tokens == 0) {   // no rows: every gradient is zero
    const int G = p->num_q_heads / p->num_kv_heads, h = p->gate_hidden, d = p->head_dim;
    if (cudaMemsetAsync(dwq, 0, (size_t)p->num_kv_heads * h * G * d * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(dwk, 0, (size_t)p->num_kv_heads * h * 3 * d * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(dqnorm_w, 0, (size_t)h * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(dknorm_w, 0, (size_t)h * 4, stream) != cudaSuccess) {
      set_error("gate_bwd: clearing the outputs failed");
      return SAS_ERR_CUDA;
    }
    return SAS_OK;
  }
  SAS_PTR(workspace);
  const size_t need = gate_bwd_workspace_bytes(*p);
  if (workspace_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
    return SAS_ERR_WORKSPACE;
  }
  SAS_TRY(clear_error_word(workspace, stream));
  return launch_gate_bwd(*p, q_nope, k_nope, pooled, wq, qnorm_w, wk, knorm_w, idx, dlogg, dwq,
                         dqnorm_w, dwk, dknorm_w, workspace, stream);
}

sas_status sas_topk(const sas_problem* p, const float* scores, const float* lse, int32_t* idx,
                    float* logg, cudaStream_t stream) {
  SAS_TRY(check_problem(p, false));
  SAS_PTR(scores);
  SAS_PTR(lse);
  SAS_PTR(idx);
  SAS_PTR(logg);
  if (p->total_tokens == 0) return SAS_OK;
  return launch_topk(*p, scores, lse, idx, logg, stream);
}

sas_status sas_attn_fwd_workspace_size(const sas_problem* p, size_t* bytes) {
  SAS_TRY(check_problem(p, false));
  SAS_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  // word 0: pipeline error code of the tensor-core kernels (0 = none); the key-major path
  // adds its accumulators, per-row references and inverted selection lists
  *bytes = attn_fwd_km_supported(*p) ? attn_fwd_km_workspace_bytes(*p) : 256;
  return SAS_OK;
}

sas_status sas_attn_fwd(const sas_problem* p, const void* q, const void* k, const void* v,
                        const int32_t* idx, const float* logg, void* o, float* lse_attn,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  SAS_TRY(check_problem(p, false));
  SAS_PTR(q);
  SAS_PTR(k);
  SAS_PTR(v);
  SAS_PTR(idx);
  SAS_PTR(logg);
  SAS_PTR(o);
  SAS_PTR(lse_attn);
  SAS_PTR(workspace);
  if (p->total_tokens == 0) return SAS_OK;
  const size_t need = attn_fwd_km_supported(*p) ? attn_fwd_km_workspace_bytes(*p) : 256;
  if (workspace_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
    return SAS_ERR_WORKSPACE;
  }
  SAS_TRY(clear_error_word(workspace, stream));
  if (attn_fwd_km_supported(*p))
    return launch_attn_fwd_km(*p, q, k, v, idx, logg, o, lse_attn, workspace, stream);
  return launch_attn_fwd_simt(*p, q, k, v, idx, logg, o, lse_attn, stream);
}

sas_status sas_attn_bwd_workspace_size(const sas_problem* p, size_t* bytes) {
  SAS_TRY(check_problem(p, false));
  SAS_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  if (attn_bwd_km_supported(*p)) {   // key-major path: accumulators and selection lists
    *bytes = attn_bwd_km_workspace_bytes(*p);
    return SAS_OK;
  }
  // [256 B error word][D = rowsum(dO*O), fp32 T*Hq] (CUDA-core path)
  *bytes = 256 + ((((size_t)p->total_tokens * p->num_q_heads * sizeof(float)) + 255) & ~(size_t)255);
  return SAS_OK;
}

sas_status sas_attn_bwd(const sas_problem* p, const void* q, const void* k, const void* v,
                        const void* o, const void* dout, const float* lse_attn,
                        const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                        float* dlogg, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  SAS_TRY(check_problem(p, false));
  SAS_PTR(q);
  SAS_PTR(k);
  SAS_PTR(v);
  SAS_PTR(o);
  SAS_PTR(dout);
  SAS_PTR(lse_attn);
  SAS_PTR(idx);
  SAS_PTR(logg);
  SAS_PTR(dq);
  SAS_PTR(dk);
  SAS_PTR(dv);
  SAS_PTR(dlogg);
  size_t need = 0;
  sas_attn_bwd_workspace_size(p, &need);
  if (need > 0) {
    SAS_PTR(workspace);
    if (workspace_bytes < need) {
      set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
      return SAS_ERR_WORKSPACE;
    }
  }
  if (p->total_tokens == 0) return SAS_OK;
  SAS_TRY(clear_error_word(workspace, stream));
  if (attn_bwd_km_supported(*p))
    return launch_attn_bwd_km(*p, q, k, v, o, dout, lse_attn, idx, logg, dq, dk, dv, dlogg,
                              workspace, stream);
  float* drow = (float*)((char*)workspace + 256);
  return launch_attn_bwd_simt(*p, q, k, v, o, dout, lse_attn, idx, logg, dq, dk, dv, dlogg, drow,
                              stream);
}

static sas_status check_decode(const sas_decode_problem* p) {
  SAS_CHECK_ARG(p != nullptr, "problem is NULL");
  SAS_CHECK_ARG(p->batch >= 1, "batch must be >= 1 (got %d)", p->batch);
  SAS_CHECK_ARG(p->capacity >= 1, "capacity must be >= 1 (got %d)", p->capacity);
  SAS_CHECK_ARG(p->num_kv_heads >= 1 && p->num_q_heads >= p->num_kv_heads &&
                    p->num_q_heads % p->num_kv_heads == 0,
                "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)", p->num_q_heads,
                p->num_kv_heads);
  const int G = p->num_q_heads / p->num_kv_heads;
  if (!(G == 1 || G == 2 || G == 4 || G == 5 || G == 8)) {
    set_error("query heads per KV head must be 1, 2, 4, 5 or 8 (got %d)", G);
    return SAS_ERR_UNSUPPORTED;
  }
  if (!(p->head_dim == 64 || p->head_dim == 128)) {
    set_error("head_dim must be 64 or 128 (got %d)", p->head_dim);
    return SAS_ERR_UNSUPPORTED;
  }
  if (!(p->block == 16 || p->block == 32 || p->block == 64)) {
    set_error("block must be 16, 32 or 64 (got %d)", p->block);
    return SAS_ERR_UNSUPPORTED;
  }
  if (!(p->gate_hidden == 32 || p->gate_hidden == 64 || p->gate_hidden == 128)) {
    set_error("gate_hidden must be 32, 64 or 128 (got %d)", p->gate_hidden);
    return SAS_ERR_UNSUPPORTED;
  }
  SAS_CHECK_ARG(p->topk >= 1 && p->topk + 1 <= 128, "topk must be in 1..127 (got %d)", p->topk);
  SAS_CHECK_ARG(p->dtype == SAS_BF16 || p->dtype == SAS_FP32, "unknown dtype %d", (int)p->dtype);
  if ((p->capacity + p->block - 1) / p->block > 4096) {
    set_error("capacity / block must be <= 4096 blocks");
    return SAS_ERR_UNSUPPORTED;
  }
  SAS_CHECK_ARG(p->seqlens != nullptr, "seqlens is NULL");
  SAS_CHECK_ARG(p->gate_rope_cos != nullptr && p->gate_rope_sin != nullptr,
                "gate rotary tables are NULL");
  SAS_CHECK_ARG(p->ungated == 0 || p->ungated == 1, "ungated must be 0 or 1 (got %d)", p->ungated);
  SAS_CHECK_ARG(p->gate_heads == 0 || p->gate_heads == p->num_kv_heads ||
                    p->gate_heads == p->num_q_heads,
                "gate_heads must be 0, num_kv_heads (%d) or num_q_heads (%d) (got %d)",
                p->num_kv_heads, p->num_q_heads, p->gate_heads);
  return SAS_OK;
}

sas_status sas_decode_workspace_size(const sas_decode_problem* p, size_t* bytes) {
  SAS_TRY(check_decode(p));
  SAS_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  *bytes = decode_workspace_bytes(*p);
  return SAS_OK;
}

sas_status sas_decode(const sas_decode_problem* p, const void* q, const void* q_nope,
                      const void* k_cache, const void* v_cache, const void* gate_key_cache,
                      const float* cur_pool, const void* wq, const float* qnorm_w,
                      const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                      float* logg_out, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  SAS_TRY(check_decode(p));
  SAS_PTR(q);
  SAS_PTR(q_nope);
  SAS_PTR(k_cache);
  SAS_PTR(v_cache);
  SAS_PTR(gate_key_cache);
  SAS_PTR(cur_pool);
  SAS_PTR(wq);
  SAS_PTR(qnorm_w);
  SAS_PTR(wk);
  SAS_PTR(knorm_w);
  SAS_PTR(o);
  SAS_PTR(workspace);
  if (idx_out) SAS_CHECK_ARG(aligned16(idx_out), "idx_out is not 16-byte aligned");
  if (logg_out) SAS_CHECK_ARG(aligned16(logg_out), "logg_out is not 16-byte aligned");
  const size_t need = decode_workspace_bytes(*p);
  if (workspace_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
    return SAS_ERR_WORKSPACE;
  }
  return launch_decode(*p, q, q_nope, k_cache, v_cache, gate_key_cache, cur_pool, wq, qnorm_w, wk,
                       knorm_w, o, idx_out, logg_out, workspace, DecodePaging{}, stream);
}

sas_status sas_decode_paged(const sas_decode_problem* p, const int32_t* page_table,
                            int32_t num_pages, const void* q, const void* q_nope,
                            const void* k_pages, const void* v_pages, const void* gate_key_pages,
                            const float* cur_pool, const void* wq, const float* qnorm_w,
                            const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                            float* logg_out, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  SAS_TRY(check_decode(p));
  if (!decode_attn_tc_supported(*p)) {
    set_error("decode_paged: supported for bf16, head_dim 128, block 64 (one block per page)");
    return SAS_ERR_UNSUPPORTED;
  }
  SAS_CHECK_ARG(num_pages >= 1, "num_pages must be >= 1 (got %d)", num_pages);
  SAS_PTR(page_table);
  SAS_PTR(q);
  SAS_PTR(q_nope);
  SAS_PTR(k_pages);
  SAS_PTR(v_pages);
  SAS_PTR(gate_key_pages);
  SAS_PTR(cur_pool);
  SAS_PTR(wq);
  SAS_PTR(qnorm_w);
  SAS_PTR(wk);
  SAS_PTR(knorm_w);
  SAS_PTR(o);
  SAS_PTR(workspace);
  if (idx_out) SAS_CHECK_ARG(aligned16(idx_out), "idx_out is not 16-byte aligned");
  if (logg_out) SAS_CHECK_ARG(aligned16(logg_out), "logg_out is not 16-byte aligned");
  const size_t need = decode_workspace_bytes(*p);
  if (workspace_bytes < need) {
    set_error("workspace too small: %zu < %zu bytes", workspace_bytes, need);
    return SAS_ERR_WORKSPACE;
  }
  DecodePaging pg;
  pg.pt = page_table;
  pg.num_pages = num_pages;
  return launch_decode(*p, q, q_nope, k_pages, v_pages, gate_key_pages, cur_pool, wq, qnorm_w, wk,
                       knorm_w, o, idx_out, logg_out, workspace, pg, stream);
}

}  // extern "C"
