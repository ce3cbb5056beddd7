/*
 * sas.h -- C ABI of the B200 (sm_100a) gated block-sparse attention library.
 *
 * The operator is SAS gated sparse attention as described on the SAS pages:
 *   - project README "SAS: Simple Attention Sparsification via End-to-End
 *     Optimization of Context Ranking", intro items (a) and (b): discrete Top-K
 *     block selection, each selected block carrying a continuous gate that is
 *     added to the attention logits;
 *   - model card "tencent/Simple-Attention-Sparsification", table "Checkpoint
 *     configuration": KV block 64, Top-K 31 historical blocks, gate hidden 128,
 *     query projection Qproj, key-block pooling max + min + average, Q/K
 *     normalisation, gate RoPE; and its decode-budget paragraph (2,048 tokens,
 *     1,024 / 4,096 also usable);
 *   - the paper's abstract: gates inside the attention softmax in log form,
 *     normalised softmax gates that weigh history against the always-retained
 *     current block, FlashAttention-style memory-efficient kernel.
 *
 * Readings of points the pages leave open (the same ones the test oracle uses):
 *   one gate per (token, KV head), shared by the G = Hq/Hkv query heads; Qproj
 *   reads the G pre-rotary query heads concatenated (G*d -> h); pooled block key
 *   = concat(max, min, mean) (3d -> h); RMSNorm (eps, weight) after each
 *   projection, then rotate-half rotary over h at position t (query) or j*B
 *   (block start); score s = q~.k~/sqrt(h); softmax over every causally visible
 *   block j <= c_t (current block included), log g = s - logsumexp; the current
 *   block's key pools only tokens c_t*B..t; Top-K over historical blocks j < c_t
 *   (all if c_t <= K), ties to the lower index; attention logit
 *   z = q.k/sqrt(d) + log g(block of key) for selected blocks and keys <= t.
 *
 * Conventions (every entry point):
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or synchronises. Every launch is asynchronous on
 *     `stream`. Caller-provided workspace must be at least the size the matching
 *     *_workspace_size call reports and 256-byte aligned.
 *   - Tensors are dense, row-major, in the shapes written below; tokens of all
 *     sequences are packed back to back (cu_seqlens). Device pointers must be
 *     16-byte aligned.
 *   - T = total_tokens, Hq/Hkv = query/KV heads, G = Hq/Hkv, d = head_dim,
 *     B = block, K = topk, h = gate_hidden, NBmax = ceil(max_seqlen / B).
 *   - "dtype" tensors are bf16 (SAS_BF16) or fp32 (SAS_FP32); fp32 tensors are
 *     always fp32.
 *   - Errors: invalid or unsupported arguments are detected before any launch
 *     and return a negative status; sas_last_error() (thread-local) then holds
 *     the reason. A failed launch returns SAS_ERR_CUDA. Nothing is launched
 *     after the first error of a call.
 *   - Device-side errors: every entry point that takes a workspace uses its first
 *     int32 (word 0) as the call's error word. The call clears it on `stream`
 *     before its kernels run, and a kernel that meets a device-side failure
 *     writes a nonzero code there; read it once the stream has completed
 *     (0 = none). Codes: 41, 81-86 decode waits that gave up (bounded mbarrier
 *     or flag waits, about one second); 51-57 forward, 71-79 backward, 91-93 gate
 *     projection, 94-96 router weight-gradient, 97-99 tensor-core gate score waits
 *     that gave up; 60 forward / 61 decode: a row whose largest
 *     logit exceeds its own key's logit by more than ~97 nats (outside the fixed
 *     per-row reference's fp32 range; that row's output is 0 and its lse -inf);
 *     62 paged decode: a page id out of range.
 *     The outputs of a call with a nonzero code are not valid.
 *   - Supported: d in {64, 128}; B in {16, 32, 64}; 1 <= K <= 127;
 *     h in {32, 64, 128}; G in {1, 2, 4, 5, 8}; NBmax <= 2048 (prefill) or
 *     ceil(capacity / B) <= 4096 (decode). Anything else returns
 *     SAS_ERR_UNSUPPORTED.
 */
#ifndef SAS_H
#define SAS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sas_status {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = -1,
  SAS_ERR_UNSUPPORTED = -2,
  SAS_ERR_CUDA = -3,
  SAS_ERR_WORKSPACE = -4
} sas_status;

typedef enum sas_dtype { SAS_BF16 = 0, SAS_FP32 = 1 } sas_dtype;

/* A packed prefill / training problem. */
typedef struct sas_problem {
  int32_t batch;          /* number of sequences                                   */
  int32_t total_tokens;   /* T = cu_seqlens[batch]                                 */
  int32_t max_seqlen;     /* longest sequence                                      */
  int32_t num_q_heads;    /* Hq                                                    */
  int32_t num_kv_heads;   /* Hkv                                                   */
  int32_t head_dim;       /* d                                                     */
  int32_t block;          /* B, tokens per KV block                                */
  int32_t topk;           /* K, historical blocks kept per query                   */
  int32_t gate_hidden;    /* h                                                     */
  float rms_eps;          /* RMSNorm epsilon of the gate                           */
  sas_dtype dtype;        /* element type of Q/K/V/O/dO/dQ/dK/dV and gate weights  */
  const int32_t* cu_seqlens;   /* device [batch+1], cu_seqlens[0] = 0              */
  const float* gate_rope_cos;  /* device [max_seqlen, h/2] (sas_rope_tables)        */
  const float* gate_rope_sin;  /* device [max_seqlen, h/2]                          */
  /* Gate heads Hs. 0 or num_kv_heads: one gate per (token, KV head), shared by the G query
   * heads of the KV group (the default reading). num_q_heads: one gate per (token, query
   * head) -- the query projection reads that head alone (wq [Hq, h, d]), scores it against
   * its KV head's block keys, and every query head keeps its own blocks. Either way the
   * gate has Hq*d*h + Hkv*3d*h + 2h parameters. Tensors marked Hs below follow it; Gs =
   * Hq/Hs query heads share a selection. */
  int32_t gate_heads;
} sas_problem;

/* One decode step over a batch of contiguous KV caches. */
typedef struct sas_decode_problem {
  int32_t batch;
  int32_t capacity;       /* cache capacity in tokens, Lmax; NBmax = ceil(Lmax/B)  */
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block;
  int32_t topk;           /* budget = (K + 1) * B tokens                           */
  int32_t gate_hidden;
  float rms_eps;
  sas_dtype dtype;        /* q / caches / gate weights                              */
  const int32_t* seqlens;      /* device [batch]: L_b in 1..capacity, newest token at L_b-1 */
  const float* gate_rope_cos;  /* device [capacity, h/2]                           */
  const float* gate_rope_sin;
  /* 0 (default): the kept blocks' log-gates are added to the attention logits, as in the
   * prefill operator. 1: hard selection only -- the gate still picks the blocks (and
   * idx_out / logg_out still report them with their log-gates), but the attention is a plain
   * softmax over the kept keys, as a serving backend that uses the gate for selection alone
   * would compute it (Hugging Face card "tencent/Simple-Attention-Sparsification", SGLang
   * seer_attn backend section). */
  int32_t ungated;
  /* Gate heads Hs as in sas_problem (0 or num_kv_heads: per KV group; num_q_heads: per query
   * head, wq [Hq, h, d], selections [batch, Hq, K+1]). */
  int32_t gate_heads;
} sas_decode_problem;

/* Reason for the last non-OK status returned on this thread ("" if none). */
const char* sas_last_error(void);

/* Diagnostic: number of kernels this library has launched from the calling thread
 * since the library was loaded (every entry point adds the launches it issued). */
uint64_t sas_kernel_launches(void);

/* Host helper: cos/sin tables of the gate's rotate-half rotary embedding,
 * theta(p, i) = p * base^(-2i/rot_dim), computed in double and rounded once to
 * float. cos_out/sin_out are HOST buffers of positions * rot_dim/2 floats,
 * row p = position p. Model card "Checkpoint configuration": Gate RoPE enabled. */
sas_status sas_rope_tables(int32_t positions, int32_t rot_dim, double base,
                           float* cos_out, float* sin_out);

/* A1 -- key-block pooling (model card "Checkpoint configuration": key block pooling
 * max + min + average). k_nope: dtype [T, Hkv, d], keys before the backbone's
 * rotary embedding. pooled: fp32 [batch, NBmax, Hkv, 3d] = (max | min | mean) over
 * each block's tokens (a sequence's last block may be partial); blocks past a
 * sequence's end are written as 0. */
sas_status sas_pool_keys(const sas_problem* p, const void* k_nope, float* pooled,
                         cudaStream_t stream);

/* A2 -- gate block keys (model card: Q/K normalization, Gate RoPE).
 * k~_j = rope(RMSNorm(Wk . pooled_j) * knorm_w, pos = j*B).
 * pooled fp32 [batch, NBmax, Hkv, 3d]; wk dtype [Hkv, h, 3d]; knorm_w fp32 [h];
 * gate_keys fp32 [batch, NBmax, Hkv, h] (0 past a sequence's end). */
sas_status sas_gate_keys(const sas_problem* p, const float* pooled, const void* wk,
                         const float* knorm_w, float* gate_keys, cudaStream_t stream);

/* A3 -- gate scores (model card: Query projection Qproj; abstract: normalised
 * softmax gates calibrated against the always-retained current block).
 * q~_t,s = rope(RMSNorm(Wq[s] . concat_g q_nope[t, s*Gs+g]) * qnorm_w, pos = t) for gate
 * head s; s[t, s, j] = q~_t,s . k~_j / sqrt(h) with the block keys of KV head
 * kv = s*Gs/G: for j < c_t from gate_keys, and for j = c_t the current block's key pooled
 * over its tokens c_t*B..t (computed here from k_nope, wk, knorm_w); s = -inf for j > c_t.
 * lse[t, s] = logsumexp_{j<=c_t} s.
 * q_nope dtype [T, Hq, d]; k_nope dtype [T, Hkv, d]; gate_keys fp32 [batch, NBmax,
 * Hkv, h]; wq dtype [Hs, h, Gs*d]; wk dtype [Hkv, h, 3d]; qnorm_w, knorm_w fp32 [h];
 * scores fp32 [T, Hs, NBmax]; lse fp32 [T, Hs].
 * Workspace (size from sas_gate_scores_workspace_size): for bf16, d = 128, h = 128 the two
 * projections run as tensor-core GEMMs and the workspace holds their inputs and outputs
 * (per token and kv head: the current block's prefix max, min and mean as exact bf16 parts,
 * 1280 B, and the two projections, 1024 B); the historical scores then also run on the
 * tensor cores, from q~ and the block keys split into tf32 hi + lo parts (three tf32
 * products per element, hi.hi + hi.lo + lo.hi, fp32 accumulation: within a few fp32
 * roundings of the exact dot product), and the workspace holds the splits (per token and
 * gate head 1024 B, per cached block key 1024 B). Otherwise 256 B suffice. Word 0 is the
 * call's error word (codes 91-93, 97-99). */
sas_status sas_gate_scores_workspace_size(const sas_problem* p, size_t* bytes);
sas_status sas_gate_scores(const sas_problem* p, const void* q_nope, const void* k_nope,
                           const float* gate_keys, const void* wq, const float* qnorm_w,
                           const void* wk, const float* knorm_w, float* scores, float* lse,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* A3 + A4 fused -- gate scores and Top-K selection in one pass (paper abstract: Top-K keeps
 * the computation sparse; model card: Qproj, Q/K normalisation, gate RoPE, Top-K).
 * Same inputs as sas_gate_scores, same results as sas_gate_scores followed by sas_topk:
 * idx int32 / logg fp32 [T, Hs, K+1] (ids ascending, current block last, -1 padding),
 * and, if lse is not NULL, the gate logsumexp fp32 [T, Hs]. For bf16, d = 128, h = 128
 * and NBmax <= 1024 the scores live only in shared memory (one kernel holds a tile's score
 * rows, selects and writes the kept ids). Its historical products are fp32 FMA chains, where
 * sas_gate_scores uses tf32 hi/lo products on the tensor cores; both are within a few fp32
 * roundings of the exact scores, so the ids agree except at near-ties (both are then a
 * correct Top-K) and the log-gates to about 1e-5. Other shapes run the two unfused kernels through the workspace, which
 * then also holds the scores. Workspace (sas_gate_select_workspace_size): word 0 is the
 * call's error word (codes 91-93). */
sas_status sas_gate_select_workspace_size(const sas_problem* p, size_t* bytes);
sas_status sas_gate_select(const sas_problem* p, const void* q_nope, const void* k_nope,
                           const float* gate_keys, const void* wq, const float* qnorm_w,
                           const void* wk, const float* knorm_w, int32_t* idx, float* logg,
                           float* lse, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* Router backward (README intro item (b): the loss reaches the selector; paper abstract:
 * end-to-end optimisation of the context ranking) -- gradients of one layer's gate
 * parameters through the log-gates of the kept blocks, the selection held fixed:
 * dL/ds[t, kv, idx[t, kv, slot]] = dlogg[t, kv, slot], then back through
 * s = q~.k~/sqrt(h), the gate rotary, the RMSNorm and the two projections (the historical
 * block keys from `pooled`, the current block's key from its visible prefix of k_nope).
 * The softmax term of the gate (- softmax_j * the row sum of dlogg) is left out: it is zero
 * for the dlogg returned by sas_attn_bwd, whose row sums vanish because the attention does
 * not change when all log-gates of a row move by one constant.
 * Inputs as sas_gate_scores, plus pooled fp32 [batch, NBmax, Hkv, 3d] (sas_pool_keys),
 * idx int32 / dlogg fp32 [T, Hkv, K+1]. Outputs (overwritten, fp32): dwq [Hkv, h, G*d],
 * dqnorm_w [h], dwk [Hkv, h, 3d], dknorm_w [h]; sums of floating-point atomics, so their low
 * bits can change from run to run. Supported: bf16, head_dim 128, gate_hidden 128,
 * block <= 128, one gate per KV group (SAS_ERR_UNSUPPORTED otherwise). Workspace (sas_gate_bwd_workspace_size):
 * word 0 is the call's error word (the tensor-core projections' codes 91-93; 0 = none). */
sas_status sas_gate_bwd_workspace_size(const sas_problem* p, size_t* bytes);
sas_status sas_gate_bwd(const sas_problem* p, const void* q_nope, const void* k_nope,
                        const float* pooled, const void* wq, const float* qnorm_w, const void* wk,
                        const float* knorm_w, const int32_t* idx, const float* dlogg, float* dwq,
                        float* dqnorm_w, float* dwk, float* dknorm_w, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/* A4 -- Top-K selection (README (b); model card: Training Top-K 31 historical blocks).
 * Per (t, gate head s): the min(K, c_t) historical blocks with the highest score (ties to
 * the lower index), ascending, then the current block c_t, then -1 padding.
 * idx int32 [T, Hs, K+1]; logg fp32 [T, Hs, K+1] = s - lse on kept slots, 0 on
 * padding. Bit-exact given the scores. */
sas_status sas_topk(const sas_problem* p, const float* scores, const float* lse,
                    int32_t* idx, float* logg, cudaStream_t stream);

/* A5 -- gated sparse attention forward (README (b); abstract: gate in the softmax in
 * log form, FlashAttention-style). For query head hq (KV head kv = hq / G, gate head
 * s = hq / Gs), token t:
 * z_i = q_t.k_i/sqrt(d) + logg[t, s, slot] for keys i <= t of block idx[t, s, slot];
 * O_t = softmax(z) V; lse_attn = natural-log logsumexp of z.
 * q dtype [T, Hq, d]; k, v dtype [T, Hkv, d] (rotated); idx/logg as from sas_topk
 * (any valid selection: ascending historical, current block, -1 padding);
 * o dtype [T, Hq, d]; lse_attn fp32 [T, Hq].
 * Workspace: word 0 is the call's error word (cleared by the call; 0 = none; read by the
 * caller after the stream completes). For bf16, d = 128, B = 64 the workspace also holds fp32 output
 * accumulators [T, Hq, d + 1], per-row reference logits and the inverted selection lists
 * (blocks -> kept tokens), about T*Hq*520 + T*Hkv*(K+1)*8 bytes. In that configuration the
 * per-block partial sums are added with L2 reductions, so the low bits of o and lse_attn
 * can change from run to run; a row whose largest logit exceeds the logit of its own key
 * by more than ~97 nats sets error code 60 (its o is 0, lse_attn -inf). */
sas_status sas_attn_fwd_workspace_size(const sas_problem* p, size_t* bytes);
sas_status sas_attn_fwd(const sas_problem* p, const void* q, const void* k, const void* v,
                        const int32_t* idx, const float* logg, void* o, float* lse_attn,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* A6 -- backward of A5 with the selection held fixed (abstract: the loss reaches the
 * selector through standard backpropagation). Inputs as A5 plus o, dout (dtype
 * [T, Hq, d]) and lse_attn. Outputs dq dtype [T, Hq, d]; dk, dv dtype [T, Hkv, d];
 * dlogg fp32 [T, Hs, K+1] = sum over the gate head's Gs query heads and the keys of block
 * idx[t, s, slot] of P (dP - D), 0 on padding. */
sas_status sas_attn_bwd_workspace_size(const sas_problem* p, size_t* bytes);
sas_status sas_attn_bwd(const sas_problem* p, const void* q, const void* k, const void* v,
                        const void* o, const void* dout, const float* lse_attn,
                        const int32_t* idx, const float* logg, void* dq, void* dk, void* dv,
                        float* dlogg, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* A7 -- one sparse decode step (model card: sparse decode budget; Chinese guide caveat
 * 3: the budget caps the tokens each query attends to). For sequence b with L_b
 * cached tokens (newest at L_b-1, c = (L_b-1)/B): gate query at position L_b-1;
 * historical block keys read from gate_key_cache; the current block's key from the
 * running pool state (max, min, sum/n, n = L_b - c*B) at position c*B; softmax
 * gates, Top-K, then the gated attention of the gate head's query heads over its kept
 * blocks (gate heads as sas_problem's: per KV group, or per query head).
 * q dtype [batch, Hq, d] (rotated); q_nope dtype [batch, Hq, d];
 * k_cache, v_cache dtype [batch, Hkv, capacity, d]; gate_key_cache bf16
 * [batch, Hkv, NBmax, h] (entries j < c read); cur_pool fp32 [batch, Hkv, 3, d]
 * (max, min, sum over tokens c*B..L_b-1); wq, wk, qnorm_w, knorm_w as A3;
 * o dtype [batch, Hq, d]; idx_out int32 / logg_out fp32 [batch, Hs, K+1] may be NULL.
 * Workspace (sas_decode_workspace_size): word 0 is the call's error word (cleared by the
 * call; 41 / 81-86 a bounded wait gave up, 61 a row outside the fixed reference's range).
 * Implementation: where supported (bf16, d 128, B 64, G <= 8, h in {64, 128},
 * ceil(capacity / B) <= 2048) one persistent launch runs the gate, Top-K, attention and the
 * merge of the attention's splits (sas_decode_set_fused); otherwise three launches. */
sas_status sas_decode_workspace_size(const sas_decode_problem* p, size_t* bytes);
sas_status sas_decode(const sas_decode_problem* p, const void* q, const void* q_nope,
                      const void* k_cache, const void* v_cache, const void* gate_key_cache,
                      const float* cur_pool, const void* wq, const float* qnorm_w,
                      const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                      float* logg_out, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream);

/* Decode implementation switch (no counterpart in the SAS pages; a tuning and diagnostic
 * control). enable != 0 (the default): sas_decode, sas_decode_paged and sas_decode_noalloc use
 * the single persistent launch where it supports the shapes; 0: they always use the
 * three-launch decode (gate + Top-K; split-K attention; merge). Both select the same blocks
 * (the gate arithmetic is the same, in the same order); O agrees up to fp32 summation order
 * when the two choose different split counts. Process-wide: set it between calls, not while
 * another thread is issuing decode calls. Always returns SAS_OK. */
sas_status sas_decode_set_fused(int enable);

/* A7 over paged caches -- the decode step of sas_decode with the KV cache in fixed-size pages
 * (one KV block per page), as a paged serving backend holds it (README "Acknowledgements":
 * the SGLang block-sparse fork; model card, SGLang seer_attn launch section). Same operator,
 * same results as sas_decode on the same cached values (bit-identical: the same kernels read
 * the same numbers in the same order). Layout: page_table int32 [batch, ceil(capacity / B)],
 * entry (b, j) = the page holding block j of sequence b (entries j <= (L_b - 1) / B are read);
 * k_pages, v_pages dtype [num_pages, Hkv, B, d]; gate_key_pages bf16 [num_pages, Hkv, h] (the
 * cached gate key of the page's block, read for complete blocks). Other arguments and the
 * workspace (sas_decode_workspace_size) as sas_decode. A page id outside [0, num_pages) sets
 * error code 62 in workspace word 0; that sequence's output is 0 and nothing is read through
 * the bad entry. Supported: bf16, head_dim 128, B = 64 (the tensor-core decode);
 * SAS_ERR_UNSUPPORTED otherwise. */
sas_status sas_decode_paged(const sas_decode_problem* p, const int32_t* page_table,
                            int32_t num_pages, const void* q, const void* q_nope,
                            const void* k_pages, const void* v_pages, const void* gate_key_pages,
                            const float* cur_pool, const void* wq, const float* qnorm_w,
                            const void* wk, const float* knorm_w, void* o, int32_t* idx_out,
                            float* logg_out, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/* Allocation-free variant of sas_decode (no counterpart in the SAS pages; a library
 * convenience). For callers that cannot allocate device memory around a decode step --
 * a runtime whose pool has already reserved the device, a plugin inside another
 * framework's step, a latency-critical loop that must not touch an allocator. Same
 * arguments and results as sas_decode minus the workspace: the scratch is a fixed 8 MiB
 * array inside the library, held on every GPU that loads the library until the process
 * exits. Problems needing more scratch than that (sas_decode_workspace_size) return
 * SAS_ERR_UNSUPPORTED. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture. The stream must
 * belong to the current device; a cudaDeviceReset while the library stays loaded is not
 * supported (the cached address would be stale). Calls whose kernels overlap on the GPU
 * share the one array and race: serialise them. The only scratch word that must start at
 * zero, the error word (word 0, as sas_decode's workspace word 0), is cleared by each call
 * on its stream; sas_decode_noalloc_error_word gives its address. Allocates nothing (no
 * cudaMalloc/cudaFree). */
sas_status sas_decode_noalloc(const sas_decode_problem* p, const void* q, const void* q_nope,
                              const void* k_cache, const void* v_cache,
                              const void* gate_key_cache, const float* cur_pool,
                              const void* wq, const float* qnorm_w, const void* wk,
                              const float* knorm_w, void* o, int32_t* idx_out,
                              float* logg_out, cudaStream_t stream);

/* Device address of sas_decode_noalloc's error word on the current device (no counterpart
 * in the SAS pages). The word is the first int32 of the built-in scratch: each
 * sas_decode_noalloc call clears it on its stream and its kernels write a nonzero code on a
 * device-side failure (the codes of sas_decode's workspace word 0). Read it after the call
 * with a stream-ordered copy on the same stream, e.g. cudaMemcpyAsync into a host int32 and
 * a stream synchronise. Like the decode call, the first use on a device looks the address
 * up. Allocates nothing. */
sas_status sas_decode_noalloc_error_word(const int32_t** word);

#ifdef __cplusplus
}
#endif
#endif /* SAS_H */
