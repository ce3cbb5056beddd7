"""A second, independently structured implementation of the SAS gate, to pin the oracle's
gate composition.

The pages (model card "tencent/Simple-Attention-Sparsification", table "Checkpoint
configuration": Qproj, key-block pooling max + min + average, Q/K normalisation, gate RoPE;
paper abstract: normalised softmax gates that weigh history against the always-retained
current block) name the gate's parts but print no worked example. This file restates the
gate from the written readings with a different structure from the oracle's, so that a
mistake in how the oracle composes the parts has to be made twice, in two different ways,
to go unnoticed:

  * plain torch fp64, one (sequence, token, kv head) at a time, explicit loops over the G
    query heads of a group, the blocks and the tokens of a block;
  * the gate rotary as a complex multiplication: channel pair (i, i + h/2) is the complex
    number x_i + i x_{i+h/2}, turned by exp(i * pos * base^(-2i/h));
  * RMSNorm with its learnable weight, applied before the rotary;
  * in-sequence positions from each sequence's own start;
  * the current block's key pooled over its visible prefix only;
  * Top-K by sorting (-score, block index).

Inputs carry random (non-unit) RMSNorm weights and several sequences, so a misplaced norm
weight, a packed instead of in-sequence position, another concatenation order, another score
scale or a full-block current key all change the result; the mutation test below shows that
each of those, made in this second implementation, is caught by the comparison.
"""
import math

import numpy as np
import pytest
import torch

import sas_inputs as si
from oracle import sas_oracle as orc

F64 = torch.float64


def _t(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float32 if x.dtype == torch.bfloat16 else x.dtype).to(F64)
    return torch.as_tensor(np.asarray(x), dtype=F64)


class SecondGate:
    """The gate of one packed problem, restated (see the module docstring)."""

    def __init__(self, inp, lengths, block, eps=1e-6, base=1e6, mutation=None):
        self.q = _t(inp["q_nope"])
        self.k = _t(inp["k_nope"])
        self.wq, self.wk = _t(inp["wq"]), _t(inp["wk"])
        self.qw, self.kw = _t(inp["qnorm_w"]), _t(inp["knorm_w"])
        self.lengths = list(lengths)
        self.starts = [int(x) for x in np.concatenate([[0], np.cumsum(lengths)[:-1]])]
        self.B, self.eps, self.base = block, eps, base
        self.Hs, self.h = self.wq.shape[0], self.wq.shape[1]      # gate heads
        self.Hkv = self.wk.shape[0]
        self.Gs = self.q.shape[1] // self.Hs                     # query heads per gate head
        self.G = self.q.shape[1] // self.Hkv                     # query heads per KV head
        self.mut = mutation
        self._block_keys = {}

    # -- parts -----------------------------------------------------------------------------
    def rotate(self, v, pos):
        half = self.h // 2
        z = torch.complex(v[:half], v[half:])
        freq = self.base ** (-2.0 * torch.arange(half, dtype=F64) / self.h)
        turn = torch.polar(torch.ones(half, dtype=F64), float(pos) * freq)
        r = z * turn
        return torch.cat([r.real, r.imag])

    def normalise_and_rotate(self, x, w, pos):
        if self.mut == "weight_after_rotary":
            y = self.rotate(x / torch.sqrt((x * x).mean() + self.eps), pos)
            return y * w
        y = x / torch.sqrt((x * x).mean() + self.eps) * w
        return self.rotate(y, pos)

    def pool(self, rows):
        """[n, d] token keys -> 3d: running max, running min and the mean, token by token."""
        mx = rows[0].clone()
        mn = rows[0].clone()
        sm = torch.zeros_like(rows[0])
        for r in rows:
            mx = torch.maximum(mx, r)
            mn = torch.minimum(mn, r)
            sm = sm + r
        return torch.cat([mx, mn, sm / rows.shape[0]])

    def key(self, pooled, kv, pos):
        return self.normalise_and_rotate(self.wk[kv] @ pooled, self.kw, pos)

    def query(self, tg, sh, pos):
        parts = [self.q[tg, sh * self.Gs + g] for g in range(self.Gs)]
        if self.mut == "concat_interleaved":
            qcat = torch.stack(parts, dim=1).reshape(-1)
        else:
            qcat = torch.cat(parts)
        return self.normalise_and_rotate(self.wq[sh] @ qcat, self.qw, pos)

    def kv_of(self, sh):
        """the KV head whose keys gate head sh's query heads read"""
        return (sh * self.Gs) // self.G

    def block_key(self, b, j, kv):
        if (b, j, kv) not in self._block_keys:
            s0, L = self.starts[b], self.lengths[b]
            rows = self.k[s0 + j * self.B: s0 + min(L, (j + 1) * self.B), kv]
            self._block_keys[(b, j, kv)] = self.key(self.pool(rows), kv, j * self.B)
        return self._block_keys[(b, j, kv)]

    # -- one row ---------------------------------------------------------------------------
    def row(self, b, t, sh, K):
        """Scores over blocks 0..c, logsumexp, kept ids and their log-gates for token t
        (in-sequence) of sequence b and gate head sh."""
        s0 = self.starts[b]
        c = t // self.B
        qpos = s0 + t if self.mut == "packed_positions" else t
        qt = self.query(s0 + t, sh, qpos)
        kv = self.kv_of(sh)
        keys = [self.block_key(b, j, kv) for j in range(c)]
        if self.mut == "full_block_current":
            keys.append(self.block_key(b, c, kv))
        else:
            rows = self.k[s0 + c * self.B: s0 + t + 1, kv]
            keys.append(self.key(self.pool(rows), kv, c * self.B))
        scale = self.h if self.mut == "scale_h" else math.sqrt(self.h)
        s = torch.stack([torch.dot(qt, kj) for kj in keys]) / scale
        lse = torch.logsumexp(s, dim=0)
        hist = sorted(range(c), key=lambda j: (-float(s[j]), j))[:K]
        ids = sorted(hist) + [c]
        return s, lse, ids, [float(s[j] - lse) for j in ids]


def _problem(lengths, Hq, Hkv, d, B, K, h, dtype, seed, gate_heads=None):
    shape = si.Shape(list(lengths), Hq, Hkv, d, B, K, h, dtype, seed=seed, gate_heads=gate_heads)
    return shape, si.prefill_inputs(shape)


CASES = {
    # several sequences (in-sequence positions), non-unit norm weights, G 2 and 5
    "fp32-G2-3seq": (([70, 33, 129], 4, 2, 8, 16, 3, 16, "fp32"), 11),
    "bf16-G5-2seq": (([90, 51], 10, 2, 16, 16, 2, 32, "bf16"), 12),
    # one gate per query head (gate_heads = Hq)
    "fp32-G2-per-head": (([70, 33], 4, 2, 8, 16, 3, 16, "fp32", 4), 14),
}


@pytest.mark.parametrize("name", list(CASES))
def test_oracle_gate_matches_second_implementation(name):
    args, seed = CASES[name]
    lengths, Hq, Hkv, d, B, K, h, dt = args[:8]
    shape, inp = _problem(lengths, Hq, Hkv, d, B, K, h, dt, seed, *args[8:])
    Hs = shape.sel_heads
    assert not torch.all(inp["qnorm_w"] == 1) and not torch.all(inp["knorm_w"] == 1)
    ref = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, B, K, 1e-6, 1e6)
    two = SecondGate(inp, lengths, B)
    n = 0
    for b, L in enumerate(lengths):
        s0 = two.starts[b]
        for j in range((L + B - 1) // B):            # A2: the historical block keys
            for kv in range(Hkv):
                np.testing.assert_allclose(ref["gate_keys"][b, j, kv], two.block_key(b, j, kv).numpy(),
                                           rtol=1e-11, atol=1e-12)
        for t in range(L):                           # A3/A4: every row
            c = t // B
            for sh in range(Hs):
                s, lse, ids, lg = two.row(b, t, sh, K)
                np.testing.assert_allclose(ref["scores"][s0 + t, sh, :c + 1], s.numpy(),
                                           rtol=1e-11, atol=1e-12)
                assert np.isneginf(ref["scores"][s0 + t, sh, c + 1:]).all()
                assert abs(ref["lse"][s0 + t, sh] - float(lse)) <= 1e-11
                kept = ref["idx"][s0 + t, sh]
                assert list(kept[kept >= 0]) == ids
                np.testing.assert_allclose(ref["logg"][s0 + t, sh, :len(ids)], lg, rtol=0, atol=1e-11)
                n += 1
    assert n == shape.total_tokens * Hs


@pytest.mark.parametrize("gate_heads", [None, 8])
def test_oracle_decode_gate_matches_second_implementation(gate_heads):
    """The decode gate (cached block keys + a running pool state for the current block) gives
    the second implementation's selection and log-gates for the newest token (gate_heads = 8
    = Hq: one gate per query head)."""
    lengths, Hq, Hkv, d, B, K, h = [77, 130, 16, 200], 8, 2, 16, 16, 4, 32
    shape, inp = _problem(lengths, Hq, Hkv, d, B, K, h, "fp32", 13, gate_heads)
    two = SecondGate(inp, lengths, B)
    nbm = shape.max_blocks
    cap = max(lengths)
    nb = len(lengths)
    gkc = np.zeros((nb, Hkv, nbm, h))
    pool = np.zeros((nb, Hkv, 3, d))
    qn = np.zeros((nb, Hq, d))
    kc = np.zeros((nb, Hkv, cap, d))
    k = orc.as64(inp["k_nope"])
    for b, L in enumerate(lengths):
        s0 = two.starts[b]
        c = (L - 1) // B
        qn[b] = orc.as64(inp["q_nope"][s0 + L - 1])
        for kv in range(Hkv):
            for j in range(c):
                gkc[b, kv, j] = two.block_key(b, j, kv).numpy()
            cur = k[s0 + c * B: s0 + L, kv]
            pool[b, kv] = np.stack([cur.max(0), cur.min(0), cur.sum(0)])
    _, idx, logg, _ = orc.decode(qn, qn, kc, kc, lengths, gkc, pool, inp["wq"], inp["qnorm_w"],
                                 inp["wk"], inp["knorm_w"], B, K, 1e-6, 1e6)
    for b, L in enumerate(lengths):
        for sh in range(shape.sel_heads):
            _, _, ids, lg = two.row(b, L - 1, sh, K)
            kept = idx[b, sh]
            assert list(kept[kept >= 0]) == ids
            np.testing.assert_allclose(logg[b, sh, :len(ids)], lg, rtol=0, atol=1e-11)


@pytest.mark.parametrize("mutation", ["weight_after_rotary", "packed_positions",
                                      "concat_interleaved", "scale_h", "full_block_current"])
def test_comparison_catches_plausible_composition_mistakes(mutation):
    """Each plausible composition mistake, made in the second implementation, makes it
    disagree with the oracle on these inputs (so the agreement above is not vacuous)."""
    (lengths, Hq, Hkv, d, B, K, h, dt), seed = CASES["fp32-G2-3seq"]
    shape, inp = _problem(lengths, Hq, Hkv, d, B, K, h, dt, seed)
    ref = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, B, K, 1e-6, 1e6)
    bad = SecondGate(inp, lengths, B, mutation=mutation)
    worst = 0.0
    for b, L in enumerate(lengths):
        s0 = bad.starts[b]
        for t in range(0, L, 5):
            s, _, _, _ = bad.row(b, t, 1, K)
            worst = max(worst, float(np.abs(ref["scores"][s0 + t, 1, :t // B + 1] - s.numpy()).max()))
    assert worst > 1e-3, f"{mutation} went unnoticed (max |score diff| {worst:.2e})"
