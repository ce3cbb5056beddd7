"""Pins for the oracle's gated sparse attention (forward and backward).

Each test checks the oracle against something other than itself: PyTorch's
scaled_dot_product_attention (a library routine) with an independently built
float mask, closed-form identities, and finite differences.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import sas_inputs as si
from oracle import sas_oracle as orc


def _problem(lengths, Hq=4, Hkv=2, d=16, B=8, K=3, seed=5, gate_heads=None):
    shape = si.Shape(list(lengths), Hq, Hkv, d, B, K, 8, "fp32", seed=seed, gate_heads=gate_heads)
    inp = si.prefill_inputs(shape, with_dout=True)
    idx, logg = si.random_selection(shape)
    return shape, inp, idx, logg


def _mask_from_selection(idx_seq, logg_seq, B):
    """Float mask [Hkv, L, L] built by block-id comparison (independent of the oracle's loops)."""
    L, Hkv, S = idx_seq.shape
    key_blk = np.arange(L) // B
    mask = np.full((Hkv, L, L), -np.inf)
    causal = np.arange(L)[None, :] <= np.arange(L)[:, None]
    for kv in range(Hkv):
        hit = idx_seq[:, kv, :, None] == key_blk[None, None, :]          # [L, S, L]
        val = np.where(hit, logg_seq[:, kv, :, None].astype(np.float64), 0.0).sum(axis=1)
        sel = hit.any(axis=1) & causal
        mask[kv][sel] = val[sel]
    return mask


def _sdpa_reference(shape, inp, idx, logg):
    """Per sequence: SDPA (fp64) with the float mask; returns O, and grads incl. d(logg).
    The mask is built per gate head (KV head, or query head with one gate per query head)
    and repeated over that gate head's query heads."""
    G, B, Gs = shape.group, shape.block, shape.sel_group
    outs, grads = [], []
    for (s0, s1) in orc.seq_ranges(shape.cu_seqlens):
        q = inp["q"][s0:s1].double().transpose(0, 1).requires_grad_(True)          # [Hq, L, d]
        k = inp["k"][s0:s1].double().transpose(0, 1).requires_grad_(True)          # [Hkv, L, d]
        v = inp["v"][s0:s1].double().transpose(0, 1).requires_grad_(True)
        m = torch.from_numpy(_mask_from_selection(idx[s0:s1], logg[s0:s1], B)).requires_grad_(True)
        kk = k.repeat_interleave(G, 0)
        vv = v.repeat_interleave(G, 0)
        mm = m.repeat_interleave(Gs, 0)
        o = F.scaled_dot_product_attention(q[None], kk[None], vv[None], attn_mask=mm[None])[0]
        o.backward(inp["dout"][s0:s1].double().transpose(0, 1))
        # d(logg[t, s, slot]) = sum of d(mask) over the keys of that block (mask grad is
        # already summed over the gate head's query heads by repeat_interleave's backward)
        gm = m.grad.numpy()
        L = s1 - s0
        dl = np.zeros((L,) + idx.shape[1:])
        for t in range(L):
            for kv in range(shape.sel_heads):
                for sl, j in enumerate(idx[s0 + t, kv]):
                    if j >= 0:
                        dl[t, kv, sl] = gm[kv, t, j * B:(j + 1) * B][: max(0, t + 1 - j * B)].sum()
        outs.append(o.detach().transpose(0, 1).numpy())
        grads.append((q.grad.transpose(0, 1).numpy(), k.grad.transpose(0, 1).numpy(),
                      v.grad.transpose(0, 1).numpy(), dl))
    cat = lambda i: np.concatenate([g[i] for g in grads])
    return np.concatenate(outs), cat(0), cat(1), cat(2), cat(3)


@pytest.mark.parametrize("lengths,K,gate_heads", [([50], 2, None), ([37, 64, 9], 3, None),
                                                  ([130], 20, None), ([37, 64, 9], 3, 4),
                                                  ([90], 5, 4)])
def test_matches_sdpa_with_block_mask(lengths, K, gate_heads):
    """gate_heads = 4 = Hq: one gate, and so one selection, per query head."""
    shape, inp, idx, logg = _problem(lengths, K=K, gate_heads=gate_heads)
    O, LSE, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, shape.cu_seqlens, shape.block)
    dq, dk, dv, dl = orc.attention_bwd(inp["q"], inp["k"], inp["v"], inp["dout"], idx, logg,
                                       shape.cu_seqlens, shape.block)
    Or, dqr, dkr, dvr, dlr = _sdpa_reference(shape, inp, idx, logg)
    for a, b in [(O, Or), (dq, dqr), (dk, dkr), (dv, dvr), (dl, dlr)]:
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11)


def test_dense_reduction_equal_gates_all_blocks():
    """Equal gates with every block selected reduce to dense causal attention."""
    shape = si.Shape([96], 4, 2, 16, 8, 20, 8, "fp32", seed=7)
    inp = si.prefill_inputs(shape, with_dout=True)
    T, Hkv, K = 96, 2, 20
    idx = np.full((T, Hkv, K + 1), -1, np.int32)
    for t in range(T):
        c = t // 8
        idx[t, :, : c + 1] = np.arange(c + 1)
    logg = np.where(idx >= 0, -0.7, 0.0).astype(np.float32)
    O, _, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, shape.cu_seqlens, 8)
    q = inp["q"].double().transpose(0, 1)[None]
    k = inp["k"].double().transpose(0, 1).repeat_interleave(2, 0)[None]
    v = inp["v"].double().transpose(0, 1).repeat_interleave(2, 0)[None]
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True)[0].transpose(0, 1).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-10, atol=1e-12)


def test_log_gate_shift_invariance_and_gradient_sum():
    """A per-row constant added to the log-gates changes nothing; sum over slots of dlogg is 0."""
    shape, inp, idx, logg = _problem([70], K=3)
    args = (inp["q"], inp["k"], inp["v"], inp["dout"])
    base = orc.attention_bwd(*args, idx, logg, shape.cu_seqlens, shape.block)
    shift = np.random.default_rng(0).normal(size=logg.shape[:2])[..., None] * (idx >= 0)
    moved = orc.attention_bwd(*args, idx, logg + shift, shape.cu_seqlens, shape.block)
    for a, b in zip(base, moved):
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(base[3].sum(axis=2), 0.0, atol=1e-12)
    O0, _, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, shape.cu_seqlens, 8)
    O1, _, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg + shift, shape.cu_seqlens, 8)
    np.testing.assert_allclose(O0, O1, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("gate_heads", [None, 2])
def test_finite_differences(gate_heads):
    """Central differences of L = sum(O * W) against the analytic gradients (selection fixed);
    gate_heads = 2 = Hq: one selection per query head."""
    shape, inp, idx, logg = _problem([21], Hq=2, Hkv=1, d=4, B=4, K=2, seed=11,
                                     gate_heads=gate_heads)
    q, k, v = (orc.as64(inp[n]) for n in ("q", "k", "v"))
    w = orc.as64(inp["dout"])
    lg = logg.astype(np.float64)
    cu = shape.cu_seqlens

    def loss(q_, k_, v_, l_):
        return float((orc.attention_fwd(q_, k_, v_, idx, l_, cu, 4)[0] * w).sum())

    dq, dk, dv, dl = orc.attention_bwd(q, k, v, w, idx, lg, cu, 4)
    rng = np.random.default_rng(3)
    eps = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("logg", lg, dl)):
        flat = np.flatnonzero(idx >= 0) if name == "logg" else np.arange(arr.size)
        for e in rng.choice(flat, size=min(12, len(flat)), replace=False):
            plus, minus = arr.copy(), arr.copy()
            plus.flat[e] += eps
            minus.flat[e] -= eps
            a = {"q": (plus, k, v, lg), "k": (q, plus, v, lg), "v": (q, k, plus, lg),
                 "logg": (q, k, v, plus)}[name]
            b = {"q": (minus, k, v, lg), "k": (q, minus, v, lg), "v": (q, k, minus, lg),
                 "logg": (q, k, v, minus)}[name]
            fd = (loss(*a) - loss(*b)) / (2 * eps)
            assert abs(fd - grad.flat[e]) < 1e-6 * max(1.0, abs(fd)), (name, e, fd, grad.flat[e])


@pytest.mark.parametrize("gate_heads", [None, 4])
def test_row_and_key_subsets_match_full(gate_heads):
    shape, inp, idx, logg = _problem([45, 33], K=2, gate_heads=gate_heads)
    args = (inp["q"], inp["k"], inp["v"])
    O, LSE, _ = orc.attention_fwd(*args, idx, logg, shape.cu_seqlens, 8)
    rows = np.array([0, 7, 44, 45, 60, 77])
    Or, LSEr, _ = orc.attention_fwd(*args, idx, logg, shape.cu_seqlens, 8, rows=rows)
    np.testing.assert_allclose(Or, O[rows], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(LSEr, LSE[rows], rtol=1e-13)
    dq, dk, dv, dl = orc.attention_bwd(*args, inp["dout"], idx, logg, shape.cu_seqlens, 8)
    dqr, dlr = orc.attention_bwd_rows(*args, inp["dout"], idx, logg, shape.cu_seqlens, 8, rows)
    np.testing.assert_allclose(dqr, dq[rows], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dlr, dl[rows], rtol=1e-12, atol=1e-14)
    dk1, dv1 = orc.attention_bwd_keys(*args, inp["dout"], idx, logg, shape.cu_seqlens, 8, 1, 1, 8, 20)
    np.testing.assert_allclose(dk1, dk[45 + 8:45 + 20, 1], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv1, dv[45 + 8:45 + 20, 1], rtol=1e-12, atol=1e-14)


def test_attended_pairs_closed_form():
    """Pairs per (token, kv) = B*min(K, c_t) + (t mod B) + 1 for a full selection."""
    shape = si.Shape([300, 129], 4, 2, 16, 16, 5, 8, "fp32", seed=1)
    idx, _ = si.random_selection(shape)
    n = orc.attended_pairs(idx, shape.cu_seqlens, 16)
    expect = 0
    for L in shape.lengths:
        t = np.arange(L)
        expect += int((16 * np.minimum(5, t // 16) + t % 16 + 1).sum()) * 2
    assert n == expect
