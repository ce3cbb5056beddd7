"""Pins for the oracle's gate router: pooling, projections, RMSNorm, gate rotary
embedding, softmax gates, Top-K selection and the parameter-count arithmetic."""
import json
import os

import numpy as np
import pytest
import torch

import sas_inputs as si
from oracle import sas_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sas_pages.json")


# ---- rotary embedding -------------------------------------------------------------------------

def test_rope_is_complex_rotation():
    """rotate-half rotary at position p == multiplying (x_i + i x_{i+r/2}) by exp(i p base^(-2i/r))."""
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 3, 32))
    pos = np.array([0, 1, 77, 4096, 131071], dtype=np.float64)
    out = orc.rope_rotate(x, pos[:, None], 1e6)
    z = x[..., :16] + 1j * x[..., 16:]
    w = np.exp(1j * pos[:, None, None] * 1e6 ** (-np.arange(16) / 16.0))
    ref = z * w
    np.testing.assert_allclose(out[..., :16], ref.real, atol=1e-12)
    np.testing.assert_allclose(out[..., 16:], ref.imag, atol=1e-12)


def test_rope_relative_position():
    rng = np.random.default_rng(1)
    q, k = rng.normal(size=(2, 64))
    a = orc.rope_rotate(q, 1000.0, 1e6) @ orc.rope_rotate(k, 960.0, 1e6)
    b = orc.rope_rotate(q, 40.0, 1e6) @ orc.rope_rotate(k, 0.0, 1e6)
    assert abs(a - b) < 1e-10
    np.testing.assert_allclose(orc.rope_rotate(q, 0.0, 1e6), q)


# ---- RMSNorm ----------------------------------------------------------------------------------

def test_rms_norm_properties():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(7, 128)) * 3.0
    y = orc.rms_norm(x, np.ones(128), 0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(axis=1)), 1.0, rtol=1e-13)
    np.testing.assert_allclose(orc.rms_norm(5.0 * x, np.ones(128), 0.0), y, rtol=1e-13)
    w = rng.normal(size=128)
    np.testing.assert_allclose(orc.rms_norm(x, w, 0.0), y * w, rtol=1e-13)
    np.testing.assert_allclose(orc.rms_norm(np.zeros((1, 8)), np.ones(8), 1e-6), 0.0)


# ---- pooling ----------------------------------------------------------------------------------

def test_pool_keys_brute_force():
    shape = si.Shape([37, 16, 5], 2, 2, 4, 16, 2, 8, "fp32", seed=3)
    inp = si.prefill_inputs(shape)
    k = inp["k_nope"].tolist()
    P = orc.pool_keys(inp["k_nope"], shape.cu_seqlens, 16, shape.max_blocks)
    base = 0
    for b, L in enumerate(shape.lengths):
        for j in range((L + 15) // 16):
            toks = range(base + 16 * j, base + min(L, 16 * j + 16))
            for kv in range(2):
                for c in range(4):
                    vals = [k[t][kv][c] for t in toks]
                    assert P[b, j, kv, c] == max(vals)
                    assert P[b, j, kv, 4 + c] == min(vals)
                    assert abs(P[b, j, kv, 8 + c] - sum(vals) / len(vals)) < 1e-12
        for j in range((L + 15) // 16, shape.max_blocks):
            assert not P[b, j].any()
        base += L


def test_prefix_key_at_block_end_equals_block_key():
    """The current-block prefix key of the last token of a full block is that block's key."""
    shape = si.Shape([200], 4, 2, 8, 16, 3, 16, "fp32", seed=4)
    inp = si.prefill_inputs(shape)
    P = orc.pool_keys(inp["k_nope"], shape.cu_seqlens, 16, shape.max_blocks)
    gk = orc.gate_keys(P, inp["wk"], inp["knorm_w"], 16, 1e-6, 1e6, shape.lengths)
    k = orc.as64(inp["k_nope"])
    for j in (0, 3, 11):
        t = 16 * j + 15
        kc = orc.current_block_key(k, t, 16, orc.as64(inp["wk"]), orc.as64(inp["knorm_w"]), 1e-6,
                                    1e6)
        np.testing.assert_allclose(kc, gk[0, j], rtol=1e-12, atol=1e-13)


# ---- gate scores and softmax gates -----------------------------------------------------------

def _gate(shape, inp, K=None, rows=None):
    return orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                 inp["knorm_w"], shape.cu_seqlens, shape.block,
                                 shape.topk if K is None else K, 1e-6, 1e6, rows)


def test_normalised_gates_sum_to_one_when_all_selected():
    shape = si.Shape([120, 50], 4, 2, 8, 16, 10, 16, "fp32", seed=6)
    inp = si.prefill_inputs(shape)
    r = _gate(shape, inp)
    g = np.exp(r["logg"]) * (r["idx"] >= 0)
    np.testing.assert_allclose(g.sum(axis=2), 1.0, rtol=1e-12)
    # the scores of visible blocks are finite, the others -inf
    pos = shape.positions()
    for n in range(len(pos)):
        c = pos[n] // 16
        assert np.isfinite(r["scores"][n, :, : c + 1]).all()
        assert np.isneginf(r["scores"][n, :, c + 1:]).all()


def test_zero_query_projection_gives_equal_gates():
    shape = si.Shape([80], 4, 2, 8, 16, 2, 16, "fp32", seed=8)
    inp = si.prefill_inputs(shape)
    inp["wq"] = torch.zeros_like(inp["wq"])
    r = _gate(shape, inp)
    pos = shape.positions()
    for n in range(80):
        c = pos[n] // 16
        n_sel = min(2, c) + 1
        np.testing.assert_allclose(r["logg"][n, :, :n_sel], -np.log(c + 1), rtol=1e-12)
        # all scores tie at 0: the lowest historical indices win
        np.testing.assert_array_equal(r["idx"][n, 0, :n_sel - 1], np.arange(n_sel - 1))


def test_scores_rows_subset_and_scaling():
    shape = si.Shape([70], 4, 1, 8, 16, 2, 16, "fp32", seed=9)
    inp = si.prefill_inputs(shape)
    full = _gate(shape, inp)
    rows = np.array([0, 15, 16, 69])
    part = _gate(shape, inp, rows=rows)
    np.testing.assert_array_equal(part["idx"], full["idx"][rows])
    np.testing.assert_allclose(part["scores"], full["scores"][rows])
    # doubling the key-norm weight doubles every score (s is bilinear in q~, k~)
    inp2 = dict(inp, knorm_w=inp["knorm_w"] * 2)
    twice = _gate(shape, inp2, rows=rows)
    np.testing.assert_allclose(twice["scores"][np.isfinite(part["scores"])],
                               2 * part["scores"][np.isfinite(part["scores"])], rtol=1e-12)


# ---- Top-K --------------------------------------------------------------------------------------

def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(10)
    for trial in range(200):
        c = int(rng.integers(0, 40))
        K = int(rng.integers(1, 12))
        s = np.round(rng.normal(size=c + 1), 1)          # rounding plants ties
        ids, margin = orc.select_row(s, c, K)
        ranked = sorted(range(c), key=lambda j: (-s[j], j))
        want = sorted(ranked[:K]) + [c]
        assert list(ids) == want
        if c > K:
            assert margin == s[ranked[K - 1]] - s[ranked[K]]


def test_topk_layout_and_padding():
    s = np.array([[[0.1, 0.5, -1.0, 0.5, 0.2, 9.0, -np.inf]]])
    lse = np.array([[np.log(np.exp(s[0, 0, :6]).sum())]])
    idx, logg, margin = orc.topk(s, lse, np.array([5 * 16 + 3]), 16, 3)
    np.testing.assert_array_equal(idx[0, 0], [1, 3, 4, 5])
    np.testing.assert_allclose(logg[0, 0], s[0, 0, [1, 3, 4, 5]] - lse[0, 0])
    idx, logg, _ = orc.topk(s, lse, np.array([1 * 16]), 16, 3)
    np.testing.assert_array_equal(idx[0, 0], [0, 1, -1, -1])
    assert logg[0, 0, 2] == 0 and logg[0, 0, 3] == 0


# ---- gate size arithmetic (reading R3) -----------------------------------------------------------

def test_gate_parameter_counts_match_released_checkpoints():
    """Qproj (G*d -> h per kv head) + Kproj (3d -> h per kv head) + two h-dim norm weights per
    layer reproduce the released gate sizes; summed pooling (d -> h) would not."""
    g = json.load(open(GOLDEN))
    h = g["checkpoint_configuration"]["gate_hidden"]
    for ck in g["released_checkpoints"]:
        Hq, Hkv, d, layers = ck["num_q_heads"], ck["num_kv_heads"], ck["head_dim"], ck["layers"]
        per_layer = Hq * d * h + Hkv * 3 * d * h + 2 * h
        params = per_layer * layers
        assert round(params / 1e6, 1) == ck["gate_params_millions"]
        assert abs(params * 2 / 2 ** 20 - ck["size_mib"]) <= 1.5       # bf16, plus file overhead
        summed = (Hq * d * h + Hkv * d * h + 2 * h) * layers
        assert round(summed / 1e6, 1) != ck["gate_params_millions"]
