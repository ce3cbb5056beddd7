"""CPU oracle for SAS gated block-sparse causal attention -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import or
run this module. The CUDA library never calls it and shares no code with it.

Plain fp64 numpy, slow on purpose, written so that each step can be checked against
the method's description by eye. Sources (web pages on SAS):

  [README]   "SAS: Simple Attention Sparsification via End-to-End Optimization of
             Context Ranking", project README, intro items (a) and (b).
  [CARD]     "tencent/Simple-Attention-Sparsification" model card, "Checkpoint
             configuration" table (KV block 64, Top-K 31 historical blocks, gate
             hidden 128, query projection Qproj, key pooling max + min + average,
             Q/K normalisation on, gate RoPE on) and "Released checkpoints" table.
  [ABSTRACT] the paper's abstract (kipquest page "The abstract"): continuous selector
             scores injected into the attention logits; the gate sits inside the
             attention softmax in log form; normalised softmax gates calibrate
             historical context against the always-retained current block; Top-K
             keeps sparse computation; FlashAttention-style kernel.
  [GUIDE]    Chinese guide page, caveat 3: the budget caps the tokens each query
             attends to, it is not a KV-cache size.

Where the pages leave a step open, the reading used here is stated at that step:

  R1  selection is per query token; one gate per (token, KV head), shared by the G
      query heads of that KV group; Qproj reads the G pre-rotary query heads
      concatenated (G*d -> h). Variant (one gate per query head): Qproj reads each
      query head alone (d -> h, Wq [Hq, h, d]), the head's query is scored against its
      KV head's block keys, and every query head keeps its own blocks. The number of
      gate ("selection") heads Hs is read off Wq's first axis (Hs = Hkv or Hq) and off
      idx's second axis; query head hq uses selection head hq // (Hq/Hs) and KV head
      hq // (Hq/Hkv).
  R2  the gate reads pre-rotary Q and K and applies its own rotary embedding
      (rotate-half over h, base 1e6) at position t (query) and jB (block start).
  R3  pooled block key = concat[max, min, mean] over the block's tokens (3d);
      Kproj maps 3d -> h; no biases. (This shape reproduces the released gate
      parameter counts, 33.0M / 42.0M; see tests.)
  R4  Q/K normalisation = RMSNorm over h (eps 1e-6, learnable weight) after the
      projection and before the rotary embedding.
  R5  score s = q~ . k~ / sqrt(h).
  R6  gate softmax over all causally visible blocks j <= c_t (current block
      included); log g = s - logsumexp.
  R7  the current block's gate key pools only its visible prefix (tokens c_t*B..t),
      which is also what decode sees for a partial last block.
  R8  Top-K over historical blocks j < c_t (all of them if c_t <= K); ties go to the
      lower block index; output ascending, current block after the historical
      ones, -1 padding (padding log-gate 0).
  R9  logits z = q.k/sqrt(d) + log g(block of key) for selected blocks and keys
      i <= t; -inf elsewhere; no other scale.
  R10 gradients are those of the attention w.r.t. Q, K, V and log g with the
      selection held fixed (Top-K is piecewise constant).
  R11 decode is the same operator evaluated for the newest token; cached gate keys
      are inputs as given.
  R13 router backward: gradients of the gate parameters through the kept blocks'
      log-gates with the selection fixed (see gate_backward).

Parity pins live in tests/test_oracle_*.py and tests/test_gate_second_impl.py. The
gate's composition (R1-R7) has no worked example on the pages; besides the properties of
its parts (rotary relative position, RMSNorm scale invariance, prefix/full-block pooling
agreement, the parameter-count arithmetic) it is pinned by a second, independently
structured implementation of the same readings (torch fp64, explicit per-head and
per-block loops, complex-exponential rotary) on several sequences with non-unit norm
weights. The readings themselves (concatenation order, norm before rotary, the 1/sqrt(h)
scale, the prefix-pooled current key) remain readings of the pages.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
NEG_INF = -np.inf


def as64(x) -> np.ndarray:
    """Any tensor/array to a fresh fp64 numpy array (bf16 torch tensors go via fp32)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float32 if x.dtype == torch.bfloat16 else x.dtype) \
                .numpy().astype(F64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=F64).copy()


def seq_ranges(cu_seqlens):
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return [(int(cu[b]), int(cu[b + 1])) for b in range(len(cu) - 1)]


# ------------------------------------------------------------------------------------------
# gate building blocks  [CARD: Q/K normalization, Gate RoPE]  (R2, R4)
# ------------------------------------------------------------------------------------------

def rope_rotate(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate-half rotary embedding of the last axis of x at position(s) pos.

    x: [..., r] with r even; pos broadcast against x[..., 0].
    theta_i = pos * base^(-2i/r); out[i] = x[i]cos - x[i+r/2]sin, out[i+r/2] = x[i+r/2]cos + x[i]sin.
    """
    r = x.shape[-1]
    i = np.arange(r // 2, dtype=F64)
    theta = np.asarray(pos, dtype=F64)[..., None] * base ** (-2.0 * i / r)
    c, s = np.cos(theta), np.sin(theta)
    a, b = x[..., : r // 2], x[..., r // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w


def pool_tokens(k_nope_tokens: np.ndarray) -> np.ndarray:
    """[n, Hkv, d] -> [Hkv, 3d] = concat(max, min, mean) over the n tokens.  [CARD: max + min + average] (R3)"""
    return np.concatenate([k_nope_tokens.max(axis=0), k_nope_tokens.min(axis=0),
                           k_nope_tokens.mean(axis=0)], axis=-1)


def pool_keys(k_nope, cu_seqlens, block: int, max_blocks: int) -> np.ndarray:
    """A1: pooled block keys [batch, NBmax, Hkv, 3d]; blocks past a sequence's end are 0."""
    k = as64(k_nope)
    T, Hkv, d = k.shape
    seqs = seq_ranges(cu_seqlens)
    out = np.zeros((len(seqs), max_blocks, Hkv, 3 * d), dtype=F64)
    for b, (s0, s1) in enumerate(seqs):
        L = s1 - s0
        for j in range((L + block - 1) // block):
            out[b, j] = pool_tokens(k[s0 + j * block: s0 + min(L, (j + 1) * block)])
    return out


def project_key(pooled: np.ndarray, wk: np.ndarray, knorm_w, eps: float, pos, base: float):
    """Kproj -> RMSNorm -> gate rotary at pos.  pooled [..., Hkv, 3d], wk [Hkv, h, 3d]."""
    kh = np.einsum("khc,...kc->...kh", wk, pooled)
    return rope_rotate(rms_norm(kh, knorm_w, eps), pos, base)


def gate_keys(pooled, wk, knorm_w, block: int, eps: float, base: float, lengths=None):
    """A2: k~_j = rope(RMSNorm(Wk . P_j), pos = j*B)  -> [batch, NBmax, Hkv, h].

    Blocks past a sequence's end (given `lengths`) are left at 0.
    """
    P = as64(pooled)
    batch, nbm, Hkv, _ = P.shape
    pos = (np.arange(nbm, dtype=F64) * block)[None, :, None]          # broadcast over batch, Hkv
    out = project_key(P, as64(wk), as64(knorm_w), eps, pos, base)
    if lengths is not None:
        for b, L in enumerate(lengths):
            out[b, (L + block - 1) // block:] = 0.0
    return out


def gate_query(q_nope_rows: np.ndarray, wq: np.ndarray, qnorm_w, eps: float, pos, base: float):
    """q~ = rope(RMSNorm(Wq . concat_g Q_nope[t, s*Gs+g]), pos = t)  (R1, R2, R4).

    q_nope_rows [n, Hq, d], wq [Hs, h, Gs*d] -> [n, Hs, h] (Hs gate heads of Gs query heads).
    """
    n, Hq, d = q_nope_rows.shape
    Hkv = wq.shape[0]
    qcat = q_nope_rows.reshape(n, Hkv, (Hq // Hkv) * d)
    qh = np.einsum("khc,nkc->nkh", wq, qcat)
    return rope_rotate(rms_norm(qh, qnorm_w, eps), np.asarray(pos, dtype=F64)[:, None], base)


def current_block_key(k_nope_seq: np.ndarray, t: int, block: int, wk, knorm_w, eps, base):
    """k~ of the current block of in-sequence token t: pool tokens c*B..t only (R7)."""
    c = t // block
    P = pool_tokens(k_nope_seq[c * block: t + 1])
    return project_key(P, wk, knorm_w, eps, float(c * block), base)


def gate_scores(q_nope, k_nope, gkeys, wq, qnorm_w, wk, knorm_w, cu_seqlens, block, eps, base,
                rows=None):
    """A3: scores s[t, s, j] = q~_t,s . k~_j / sqrt(h) over visible blocks j <= c_t, and lse[t, s].

    k~_j for j < c_t comes from `gkeys` [batch, NBmax, Hkv, h] (of the gate head's KV head);
    the current block uses the prefix key (R7). Entries j > c_t are -inf. `rows` (packed
    token indices) restricts the rows computed; returns (s [n, Hs, NBmax], lse [n, Hs], rows).
    """
    q = as64(q_nope)
    k = as64(k_nope)
    gk = as64(gkeys)
    wq_, wk_ = as64(wq), as64(wk)
    qw, kw = as64(qnorm_w), as64(knorm_w)
    seqs = seq_ranges(cu_seqlens)
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    nbm, Hkv, h = gk.shape[1], gk.shape[2], gk.shape[3]
    Hs = wq_.shape[0]                       # gate heads: Hkv (per KV group) or Hq (per query head)
    kv_of = np.arange(Hs) // (Hs // Hkv)    # KV head whose block keys gate head s scores against
    s = np.full((len(rows), Hs, nbm), NEG_INF, dtype=F64)
    lse = np.empty((len(rows), Hs), dtype=F64)
    starts = np.array([a for a, _ in seqs])
    for r, tg in enumerate(rows):
        b = int(np.searchsorted(starts, tg, side="right") - 1)
        s0 = seqs[b][0]
        t = int(tg - s0)
        c = t // block
        qt = gate_query(q[tg:tg + 1], wq_, qw, eps, [t], base)[0]                # [Hs, h]
        kc = current_block_key(k[s0:seqs[b][1]], t, block, wk_, kw, eps, base)   # [Hkv, h]
        keys = np.concatenate([gk[b, :c], kc[None]], axis=0)[:, kv_of]          # [c+1, Hs, h]
        s[r, :, : c + 1] = np.einsum("kh,jkh->kj", qt, keys) / np.sqrt(h)
        m = s[r, :, : c + 1].max(axis=1, keepdims=True)
        lse[r] = (m + np.log(np.exp(s[r, :, : c + 1] - m).sum(axis=1, keepdims=True)))[:, 0]
    return s, lse, rows


# ------------------------------------------------------------------------------------------
# A4: Top-K selection  [README (b); CARD: Training Top-K 31 historical blocks]  (R6, R8)
# ------------------------------------------------------------------------------------------

def select_row(s_row: np.ndarray, c: int, K: int):
    """Block ids kept for one (token, kv head) row, ascending, current block last.

    Historical candidates are 0..c-1; keep the K highest scores (all if c <= K), ties to
    the lower index. Returns (ids, margin) where margin = s_(K) - s_(K+1) of the sorted
    historical scores (inf when no block is dropped).
    """
    cand = np.arange(c)
    if c <= K:
        return np.append(cand, c), np.inf
    order = np.lexsort((cand, -s_row[:c]))            # primary: score desc, secondary: index asc
    keep = np.sort(order[:K])
    margin = s_row[order[K - 1]] - s_row[order[K]]
    return np.append(keep, c), float(margin)


def topk(s, lse, positions, block: int, K: int):
    """Selection + log-gates for rows of `s` [n, Hkv, NBmax] at in-sequence `positions`.

    Returns idx [n, Hkv, K+1] int32 (-1 padded), logg [n, Hkv, K+1] (s - lse, 0 on padding),
    margin [n, Hkv].
    """
    n, Hkv, _ = s.shape
    idx = np.full((n, Hkv, K + 1), -1, dtype=np.int32)
    logg = np.zeros((n, Hkv, K + 1), dtype=F64)
    margin = np.empty((n, Hkv), dtype=F64)
    for r in range(n):
        c = int(positions[r]) // block
        for kv in range(Hkv):
            ids, mg = select_row(s[r, kv], c, K)
            idx[r, kv, : len(ids)] = ids
            logg[r, kv, : len(ids)] = s[r, kv, ids] - lse[r, kv]
            margin[r, kv] = mg
    return idx, logg, margin


# ------------------------------------------------------------------------------------------
# A5/A6: gated sparse attention  [README (b); ABSTRACT: gate inside the softmax in log form]
# ------------------------------------------------------------------------------------------

def logit_bias(idx_seq: np.ndarray, logg_seq: np.ndarray, block: int, rows) -> np.ndarray:
    """Bias [len(rows), L] for one sequence and one kv head: log g on the keys of selected
    blocks with key <= query, -inf elsewhere (R9)."""
    L = idx_seq.shape[0]
    bias = np.full((len(rows), L), NEG_INF, dtype=F64)
    for r, t in enumerate(rows):
        for j, lg in zip(idx_seq[t], logg_seq[t]):
            if j < 0:
                continue
            lo, hi = j * block, min((j + 1) * block, t + 1)
            if lo < hi:
                bias[r, lo:hi] = lg
    return bias


def attention_fwd(q, k, v, idx, logg, cu_seqlens, block: int, rows=None):
    """O and LSE of gated sparse causal attention.

    q [T, Hq, d], k/v [T, Hkv, d] (rotated), idx/logg [T, Hs, K+1] (Hs gate heads: Hkv, or
    Hq for one gate per query head). For head hq (gate head hq // (Hq/Hs), kv = hq // G)
    and token t: z_i = q_t . k_i / sqrt(d) + bias(t, i); O_t = softmax(z) V; LSE natural log.
    `rows` (packed token indices) restricts the rows computed. Returns (O [n, Hq, d],
    LSE [n, Hq], rows).
    """
    q, k, v = as64(q), as64(k), as64(v)
    idx = np.asarray(idx)
    logg = as64(logg)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    Hs = idx.shape[1]
    Gs = Hq // Hs
    rows = np.arange(T) if rows is None else np.asarray(rows)
    O = np.zeros((len(rows), Hq, d), dtype=F64)
    LSE = np.zeros((len(rows), Hq), dtype=F64)
    for (s0, s1) in seq_ranges(cu_seqlens):
        sel = np.nonzero((rows >= s0) & (rows < s1))[0]
        if len(sel) == 0:
            continue
        loc = rows[sel] - s0
        for sh in range(Hs):
            bias = logit_bias(idx[s0:s1, sh], logg[s0:s1, sh], block, loc)
            for g in range(Gs):
                hq = sh * Gs + g
                kv = hq // G
                z = q[s0 + loc, hq] @ k[s0:s1, kv].T / np.sqrt(d) + bias
                m = z.max(axis=1, keepdims=True)
                p = np.exp(z - m)
                l = p.sum(axis=1, keepdims=True)
                O[sel, hq] = (p / l) @ v[s0:s1, kv]
                LSE[sel, hq] = (m + np.log(l))[:, 0]
    return O, LSE, rows


def attention_bwd(q, k, v, dout, idx, logg, cu_seqlens, block: int):
    """Gradients of the gated sparse attention (R10), full problem.

    With P = softmax(z): D_t = sum_i P_ti dP_ti = dO_t . O_t, dP = dO V^T,
    dS = P (dP - D), dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d), dV = P^T dO,
    dlogg[t, s, slot] = sum over the query heads of gate head s and the keys of block
    idx[t, s, slot] of dS.
    Returns dq [T, Hq, d], dk, dv [T, Hkv, d], dlogg [T, Hs, K+1].
    """
    q, k, v, do = as64(q), as64(k), as64(v), as64(dout)
    idx = np.asarray(idx)
    logg = as64(logg)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    Hs = idx.shape[1]
    Gs = Hq // Hs
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dlogg = np.zeros(logg.shape, dtype=F64)
    for (s0, s1) in seq_ranges(cu_seqlens):
        L = s1 - s0
        loc = np.arange(L)
        for sh in range(Hs):
            bias = logit_bias(idx[s0:s1, sh], logg[s0:s1, sh], block, loc)
            dbias = np.zeros((L, L), dtype=F64)
            for g in range(Gs):
                hq = sh * Gs + g
                kv = hq // G
                z = q[s0:s1, hq] @ k[s0:s1, kv].T / np.sqrt(d) + bias
                m = z.max(axis=1, keepdims=True)
                p = np.exp(z - m)
                p /= p.sum(axis=1, keepdims=True)
                o = p @ v[s0:s1, kv]
                dp = do[s0:s1, hq] @ v[s0:s1, kv].T
                D = (do[s0:s1, hq] * o).sum(axis=1, keepdims=True)
                ds = p * (dp - D)
                dq[s0:s1, hq] = ds @ k[s0:s1, kv] / np.sqrt(d)
                dk[s0:s1, kv] += ds.T @ q[s0:s1, hq] / np.sqrt(d)
                dv[s0:s1, kv] += p.T @ do[s0:s1, hq]
                dbias += ds
            for t in range(L):
                for slot, j in enumerate(idx[s0 + t, sh]):
                    if j >= 0:
                        dlogg[s0 + t, sh, slot] = dbias[t, j * block: min((j + 1) * block, t + 1)].sum()
    return dq, dk, dv, dlogg


def attention_bwd_rows(q, k, v, dout, idx, logg, cu_seqlens, block: int, rows):
    """dQ and dlogg for some query rows only (each depends on its own row alone)."""
    q, k, v, do = as64(q), as64(k), as64(v), as64(dout)
    idx = np.asarray(idx)
    logg = as64(logg)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    Hs = idx.shape[1]
    Gs = Hq // Hs
    rows = np.asarray(rows)
    dq = np.zeros((len(rows), Hq, d), dtype=F64)
    dlogg = np.zeros((len(rows), Hs, idx.shape[2]), dtype=F64)
    for (s0, s1) in seq_ranges(cu_seqlens):
        sel = np.nonzero((rows >= s0) & (rows < s1))[0]
        if len(sel) == 0:
            continue
        loc = rows[sel] - s0
        for sh in range(Hs):
            bias = logit_bias(idx[s0:s1, sh], logg[s0:s1, sh], block, loc)
            dbias = np.zeros_like(bias)
            for g in range(Gs):
                hq = sh * Gs + g
                kv = hq // G
                z = q[s0 + loc, hq] @ k[s0:s1, kv].T / np.sqrt(d) + bias
                m = z.max(axis=1, keepdims=True)
                p = np.exp(z - m)
                p /= p.sum(axis=1, keepdims=True)
                o = p @ v[s0:s1, kv]
                dp = do[s0 + loc, hq] @ v[s0:s1, kv].T
                D = (do[s0 + loc, hq] * o).sum(axis=1, keepdims=True)
                ds = p * (dp - D)
                dq[sel, hq] = ds @ k[s0:s1, kv] / np.sqrt(d)
                dbias += ds
            for r, t in enumerate(loc):
                for slot, j in enumerate(idx[s0 + t, sh]):
                    if j >= 0:
                        dlogg[sel[r], sh, slot] = dbias[r, j * block: min((j + 1) * block, t + 1)].sum()
    return dq, dlogg


def attention_bwd_keys(q, k, v, dout, idx, logg, cu_seqlens, block: int, seq: int, kv: int,
                       key_lo: int, key_hi: int):
    """dK and dV for the keys key_lo..key_hi-1 (in-sequence) of one sequence and kv head.

    Every query row whose selection reaches one of those keys contributes; each such row's
    softmax is computed over its full selection, as in attention_bwd.
    """
    q, k, v, do = as64(q), as64(k), as64(v), as64(dout)
    idx = np.asarray(idx)
    logg = as64(logg)
    Hq, d = q.shape[1], q.shape[2]
    Hkv = k.shape[1]
    G = Hq // Hkv
    Hs = idx.shape[1]
    Gs = Hq // Hs
    s0, s1 = seq_ranges(cu_seqlens)[seq]
    L = s1 - s0
    jlo, jhi = key_lo // block, (key_hi - 1) // block
    dk = np.zeros((key_hi - key_lo, d), dtype=F64)
    dv = np.zeros((key_hi - key_lo, d), dtype=F64)
    cand = np.arange(key_lo, L)
    for sh in range(Hs):
        if (sh * Gs) // G != kv:          # gate heads whose query heads read this KV head
            continue
        hit = np.any((idx[s0 + cand, sh, :, None] >= jlo) & (idx[s0 + cand, sh, :, None] <= jhi),
                     axis=(1, 2))
        loc = cand[hit]
        if len(loc) == 0:
            continue
        _keys_grad_one_gate_head(q, k, v, do, idx, logg, block, s0, s1, sh, Gs, kv, key_lo,
                                 key_hi, loc, dk, dv)
    return dk, dv


def _keys_grad_one_gate_head(q, k, v, do, idx, logg, block, s0, s1, sh, Gs, kv, key_lo, key_hi,
                             loc, dk, dv):
    """Adds to dk, dv the contribution of the query heads of gate head sh (rows `loc`)."""
    d = q.shape[2]
    bias = logit_bias(idx[s0:s1, sh], logg[s0:s1, sh], block, loc)
    for g in range(Gs):
        hq = sh * Gs + g
        z = q[s0 + loc, hq] @ k[s0:s1, kv].T / np.sqrt(d) + bias
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v[s0:s1, kv]
        dp = do[s0 + loc, hq] @ v[s0:s1, kv].T
        D = (do[s0 + loc, hq] * o).sum(axis=1, keepdims=True)
        ds = p * (dp - D)
        dk += ds[:, key_lo:key_hi].T @ q[s0 + loc, hq] / np.sqrt(d)
        dv += p[:, key_lo:key_hi].T @ do[s0 + loc, hq]


# ------------------------------------------------------------------------------------------
# full prefill pipeline (A1..A5) -- convenience for the tests
# ------------------------------------------------------------------------------------------

def prefill_selection(q_nope, k_nope, wq, qnorm_w, wk, knorm_w, cu_seqlens, block, K, eps, base,
                      rows=None):
    """A1..A4 for (some) rows: returns dict(idx, logg, margin, scores, lse, rows, gate_keys)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lengths = np.diff(cu)
    nbm = int((lengths.max() + block - 1) // block)
    pooled = pool_keys(k_nope, cu, block, nbm)
    gk = gate_keys(pooled, wk, knorm_w, block, eps, base, lengths)
    s, lse, rows = gate_scores(q_nope, k_nope, gk, wq, qnorm_w, wk, knorm_w, cu, block, eps, base,
                               rows)
    starts = cu[:-1]
    pos = np.array([r - starts[np.searchsorted(starts, r, side="right") - 1] for r in rows])
    idx, logg, margin = topk(s, lse, pos, block, K)
    return dict(idx=idx, logg=logg, margin=margin, scores=s, lse=lse, rows=rows, pooled=pooled,
                gate_keys=gk)


# ------------------------------------------------------------------------------------------
# Router backward  [README (b): the loss reaches the selector; ABSTRACT: end-to-end
# optimisation of the context ranking]  (R13)
# ------------------------------------------------------------------------------------------
#
# R13 the gate parameters (Wq, Wk and the two RMSNorm weights) get the gradient of the
#     loss through the log-gates of the kept blocks, with the selection held fixed:
#     dL/ds[t, j] = sum over the slots holding j of dlogg - softmax_j(s[t, :c_t+1]) * sum of
#     all dlogg of the row, then back through s = q~.k~/sqrt(h), the rotary, the RMSNorm and
#     the projections (historical block keys from the pooled blocks, the current block's key
#     from its visible prefix).

def rms_norm_backward(x: np.ndarray, w: np.ndarray, eps: float, dy: np.ndarray):
    """Gradients of y = x / r * w, r = sqrt(mean(x^2) + eps), over the last axis.

    Returns (dx, dw) with dw summed over the leading axes."""
    H = x.shape[-1]
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    u = x / r
    dw = (dy * u).reshape(-1, H).sum(axis=0)
    du = dy * w
    dx = du / r - x * np.sum(du * x, axis=-1, keepdims=True) / (H * r ** 3)
    return dx, dw


def gate_backward(q_nope, k_nope, wq, qnorm_w, wk, knorm_w, idx, dlogg, cu_seqlens, block: int,
                  eps: float, base: float):
    """Router parameter gradients (R13) for the full problem.

    idx, dlogg [T, Hkv, K+1] (the forward's selection and the loss gradient of its
    log-gates). Returns dict(dwq [Hkv, h, G*d], dqnorm_w [h], dwk [Hkv, h, 3d], dknorm_w [h]).
    """
    q, k = as64(q_nope), as64(k_nope)
    wq_, wk_, qw, kw = as64(wq), as64(wk), as64(qnorm_w), as64(knorm_w)
    idx = np.asarray(idx)
    dl = as64(dlogg)
    T, Hq, d = q.shape
    Hkv, h = wq_.shape[0], wq_.shape[1]
    if wk_.shape[0] != Hkv:
        raise NotImplementedError("router backward: one gate per KV group only")
    G = Hq // Hkv
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    seqs = seq_ranges(cu)
    dwq = np.zeros_like(wq_)
    dwk = np.zeros_like(wk_)
    dqw = np.zeros(h)
    dkw = np.zeros(h)
    sq = np.sqrt(h)
    for s0, s1 in seqs:
        L = s1 - s0
        nb = (L + block - 1) // block
        # historical block keys of this sequence: pre-norm projections and final keys
        P = np.stack([pool_tokens(k[s0 + j * block: s0 + min(L, (j + 1) * block)])
                      for j in range(nb)])                                      # [nb, Hkv, 3d]
        xk = np.einsum("khc,jkc->jkh", wk_, P)                                  # [nb, Hkv, h]
        kt = rope_rotate(rms_norm(xk, kw, eps), (np.arange(nb) * block)[:, None], base)
        dkt = np.zeros_like(kt)                                                 # dL/dk~_j
        for t in range(L):
            tg = s0 + t
            c = t // block
            a = q[tg].reshape(Hkv, G * d)
            xq = np.einsum("khc,kc->kh", wq_, a)                                # [Hkv, h]
            qt = rope_rotate(rms_norm(xq, qw, eps), float(t), base)
            Pc = pool_tokens(k[s0 + c * block: tg + 1])                         # prefix (R7)
            xc = np.einsum("khc,kc->kh", wk_, Pc)
            kc = rope_rotate(rms_norm(xc, kw, eps), float(c * block), base)
            keys = np.concatenate([kt[:c], kc[None]], axis=0)                   # [c+1, Hkv, h]
            sc = np.einsum("kh,jkh->kj", qt, keys) / sq                         # [Hkv, c+1]
            p = np.exp(sc - sc.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            ds = -p * dl[tg].sum(axis=1, keepdims=True)                         # LSE term
            for kv in range(Hkv):
                for sl in range(idx.shape[2]):
                    j = int(idx[tg, kv, sl])
                    if j >= 0:
                        ds[kv, j] += dl[tg, kv, sl]
            dqt = np.einsum("kj,jkh->kh", ds, keys) / sq
            dkeys = np.einsum("kj,kh->jkh", ds, qt) / sq
            dkt[:c] += dkeys[:c]
            # current block key: rotary back (rotation by -angle), RMSNorm, Kproj
            dxc, dw_ = rms_norm_backward(xc, kw, eps, rope_rotate(dkeys[c], -float(c * block), base))
            dkw += dw_
            dwk += np.einsum("kh,kc->khc", dxc, Pc)
            dxq, dw_ = rms_norm_backward(xq, qw, eps, rope_rotate(dqt, -float(t), base))
            dqw += dw_
            dwq += np.einsum("kh,kc->khc", dxq, a)
        dxk, dw_ = rms_norm_backward(xk, kw, eps,
                                     rope_rotate(dkt, -(np.arange(nb) * block)[:, None].astype(F64), base))
        dkw += dw_
        dwk += np.einsum("jkh,jkc->khc", dxk, P)
    return dict(dwq=dwq, dqnorm_w=dqw, dwk=dwk, dknorm_w=dkw)


# ------------------------------------------------------------------------------------------
# A7: decode  [CARD: sparse decode budget; GUIDE caveat 3]  (R11)
# ------------------------------------------------------------------------------------------

def decode(q, q_nope, k_cache, v_cache, lengths, gate_key_cache, cur_pool, wq, qnorm_w, wk, knorm_w,
           block: int, K: int, eps: float, base: float, rows=None, gated: bool = True,
           selection=None):
    """One decode step for (some) sequences.

    Sequence b has L_b tokens cached, the newest at position L_b-1 with c = (L_b-1)//B.
    Gate: q~ at position L_b-1; historical keys k~_j (j < c) read from the cache; the current
    block key from the running pool state (max, min, sum/n), n = L_b - c*B, at position c*B.
    Then the same softmax gates, Top-K and gated attention as the prefill row L_b-1.
    gated=False keeps the selection but drops the log-gate from the attention logits (hard
    selection, as a serving backend that uses the gate only to pick blocks computes it;
    Hugging Face card "tencent/Simple-Attention-Sparsification", SGLang seer_attn section).
    `selection` = (idx, logg) [n, Hkv, K+1] replaces the gate's own Top-K in the attention:
    at a near-tie two selections are both correct, and the attention is then evaluated on
    the one given (the gate's own selection is still returned).
    Returns O [n, Hq, d], idx [n, Hkv, K+1], logg [n, Hkv, K+1], margin [n, Hkv].
    """
    q, qn = as64(q), as64(q_nope)
    gkc = as64(gate_key_cache) if not isinstance(gate_key_cache, np.ndarray) else gate_key_cache
    cp = as64(cur_pool)
    wq_, wk_, qw, kw = as64(wq), as64(wk), as64(qnorm_w), as64(knorm_w)
    lengths = np.asarray(lengths, dtype=np.int64)
    nb_all, Hq, d = q.shape
    Hs, h = wq_.shape[0], wq_.shape[1]          # gate heads: Hkv, or Hq (one per query head)
    Hkv = wk_.shape[0]
    G, Gs = Hq // Hkv, Hq // Hs
    rows = np.arange(nb_all) if rows is None else np.asarray(rows)
    O = np.zeros((len(rows), Hq, d))
    idx = np.full((len(rows), Hs, K + 1), -1, dtype=np.int32)
    logg = np.zeros((len(rows), Hs, K + 1))
    margin = np.zeros((len(rows), Hs))
    for r, b in enumerate(rows):
        L = int(lengths[b])
        t = L - 1
        c = t // block
        n = L - c * block
        qt = gate_query(qn[b:b + 1], wq_, qw, eps, [t], base)[0]                   # [Hs, h]
        P = np.concatenate([cp[b, :, 0], cp[b, :, 1], cp[b, :, 2] / n], axis=-1)   # [Hkv, 3d]
        kc = project_key(P, wk_, kw, eps, float(c * block), base)                   # [Hkv, h]
        kcache = as64(k_cache[b]) if not isinstance(k_cache, np.ndarray) else k_cache[b]
        vcache = as64(v_cache[b]) if not isinstance(v_cache, np.ndarray) else v_cache[b]
        for sh in range(Hs):
            kv = (sh * Gs) // G
            keys = np.concatenate([as64(gkc[b, kv, :c]), kc[kv][None]], axis=0)    # [c+1, h]
            s = keys @ qt[sh] / np.sqrt(h)
            m = s.max()
            lse = m + np.log(np.exp(s - m).sum())
            ids, mg = select_row(s, c, K)
            idx[r, sh, : len(ids)] = ids
            logg[r, sh, : len(ids)] = s[ids] - lse
            margin[r, sh] = mg
            if selection is None:
                use_ids, use_lg = ids, s[ids] - lse
            else:
                keep = np.asarray(selection[0][r, sh]) >= 0
                use_ids = np.asarray(selection[0][r, sh])[keep]
                use_lg = as64(selection[1][r, sh])[keep]
            bias = np.full(L, NEG_INF)
            for j, lg in zip(use_ids, use_lg):
                bias[j * block: min((j + 1) * block, L)] = lg if gated else 0.0
            kk, vv = kcache[kv, :L], vcache[kv, :L]
            for g in range(Gs):
                hq = sh * Gs + g
                z = kk @ q[b, hq] / np.sqrt(d) + bias
                zm = z.max()
                p = np.exp(z - zm)
                O[r, hq] = (p / p.sum()) @ vv
    return O, idx, logg, margin


# ------------------------------------------------------------------------------------------
# algorithmic work (attended pairs) -- used by the harness for FLOP counts
# ------------------------------------------------------------------------------------------

def attended_pairs(idx, cu_seqlens, block: int) -> int:
    """Number of (token, kv head, key) pairs with a finite logit."""
    idx = np.asarray(idx)
    total = 0
    for (s0, s1) in seq_ranges(cu_seqlens):
        t = np.arange(s1 - s0)
        j = idx[s0:s1].astype(np.int64)                          # [L, Hkv, K+1]
        lo = j * block
        hi = np.minimum((j + 1) * block, t[:, None, None] + 1)
        total += int(np.where(j >= 0, np.maximum(hi - lo, 0), 0).sum())
    return total
