"""Pin for the oracle's decode: one decode step equals the prefill row of the newest token
when its caches hold that prefill's own gate keys and running pool state."""
import numpy as np
import pytest

import sas_inputs as si
from oracle import sas_oracle as orc


@pytest.mark.parametrize("L,K,gate_heads", [(1, 3, None), (16, 3, None), (17, 3, None),
                                            (63, 3, None), (100, 3, None), (128, 3, None),
                                            (300, 15, None), (290, 7, None), (100, 3, 4),
                                            (290, 7, 4)])
def test_decode_equals_prefill_last_row(L, K, gate_heads):
    """gate_heads = 4 = Hq: one gate per query head."""
    B, h = 16, 16
    shape = si.Shape([L], 4, 2, 8, B, K, h, "fp32", seed=20 + L, gate_heads=gate_heads)
    inp = si.prefill_inputs(shape)
    sel = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, B, K, 1e-6, 1e6)
    O, _, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], sel["idx"], sel["logg"],
                                shape.cu_seqlens, B)
    # caches as a server would hold them after the prefill
    k = orc.as64(inp["k_nope"])
    c = (L - 1) // B
    cur = k[c * B: L]
    pool = np.stack([cur.max(0), cur.min(0), cur.sum(0)], axis=1)[None]          # [1, Hkv, 3, d]
    gkc = sel["gate_keys"].transpose(0, 2, 1, 3)                                   # [1, Hkv, NB, h]
    kc = orc.as64(inp["k"]).transpose(1, 0, 2)[None]
    vc = orc.as64(inp["v"]).transpose(1, 0, 2)[None]
    Od, idx, logg, _ = orc.decode(orc.as64(inp["q"])[L - 1:L], orc.as64(inp["q_nope"])[L - 1:L],
                                  kc, vc, [L], gkc, pool, inp["wq"], inp["qnorm_w"], inp["wk"],
                                  inp["knorm_w"], B, K, 1e-6, 1e6)
    np.testing.assert_array_equal(idx[0], sel["idx"][L - 1])
    np.testing.assert_allclose(logg[0], sel["logg"][L - 1], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Od[0], O[L - 1], rtol=1e-11, atol=1e-12)


def test_ungated_decode_is_softmax_over_kept_keys():
    """Hard selection (gated=False): same blocks, and O is a plain softmax attention over the
    kept keys -- checked against torch's scaled_dot_product_attention with a boolean mask
    built from the oracle's own selection (a library routine, independent of the oracle's
    softmax); the gated result differs whenever the kept log-gates differ."""
    import torch

    shp = si.DecodeShape([200, 37, 129], 256, 4, 2, 16, 16, 3, 16, seed=31, dtype="fp32")
    inp = si.decode_inputs(shp)
    args = (inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"], shp.lengths,
            inp["gate_key_cache"], inp["cur_pool"], inp["wq"], inp["qnorm_w"], inp["wk"],
            inp["knorm_w"], shp.block, shp.topk, 1e-6, 1e6)
    Og, idx_g, logg_g, _ = orc.decode(*args)
    Ou, idx_u, logg_u, _ = orc.decode(*args, gated=False)
    np.testing.assert_array_equal(idx_u, idx_g)
    np.testing.assert_array_equal(logg_u, logg_g)
    G = shp.num_q_heads // shp.num_kv_heads
    for b, L in enumerate(shp.lengths):
        for kv in range(shp.num_kv_heads):
            keep = np.zeros(L, dtype=bool)
            for j in idx_u[b, kv]:
                if j >= 0:
                    keep[j * shp.block: min((j + 1) * shp.block, L)] = True
            kk = torch.from_numpy(orc.as64(inp["k_cache"][b, kv, :L]))
            vv = torch.from_numpy(orc.as64(inp["v_cache"][b, kv, :L]))
            for g in range(G):
                hq = kv * G + g
                qq = torch.from_numpy(orc.as64(inp["q"][b, hq]))[None, None, None]
                ref = torch.nn.functional.scaled_dot_product_attention(
                    qq, kk[None, None], vv[None, None], attn_mask=torch.from_numpy(keep)[None, None, None])
                np.testing.assert_allclose(Ou[b, hq], ref[0, 0, 0].numpy(), rtol=1e-10, atol=1e-12)
    assert np.abs(Ou - Og).max() > 1e-6


def test_decode_on_a_given_selection_equals_prefill_row_on_it():
    """decode(selection=...) evaluates the newest token's attention on the selection given
    (a near-tie's other correct answer): it equals the prefill row's attention on that same
    selection, and on the gate's own selection it changes nothing."""
    L, B, K, h = 150, 16, 3, 16
    shape = si.Shape([L], 4, 2, 8, B, K, h, "fp32", seed=77)
    inp = si.prefill_inputs(shape)
    sel = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, B, K, 1e-6, 1e6)
    k = orc.as64(inp["k_nope"])
    c = (L - 1) // B
    cur = k[c * B: L]
    pool = np.stack([cur.max(0), cur.min(0), cur.sum(0)], axis=1)[None]
    gkc = sel["gate_keys"].transpose(0, 2, 1, 3)
    kc = orc.as64(inp["k"]).transpose(1, 0, 2)[None]
    vc = orc.as64(inp["v"]).transpose(1, 0, 2)[None]
    args = (orc.as64(inp["q"])[L - 1:L], orc.as64(inp["q_nope"])[L - 1:L], kc, vc, [L], gkc, pool,
            inp["wq"], inp["qnorm_w"], inp["wk"], inp["knorm_w"], B, K, 1e-6, 1e6)
    O0, idx0, logg0, _ = orc.decode(*args)
    O1, _, _, _ = orc.decode(*args, selection=(idx0, logg0))
    np.testing.assert_array_equal(O1, O0)
    # another valid selection: historical blocks 0, 2, 5 with arbitrary log-gates
    other = np.array([[[0, 2, 5, c]] * 2], dtype=np.int32)
    lg = np.array([[[-0.5, -1.5, -2.0, -0.7], [-3.0, -0.1, -0.2, -1.0]]])
    O2, idx2, _, _ = orc.decode(*args, selection=(other, lg))
    np.testing.assert_array_equal(idx2, idx0)          # the gate's own selection is still returned
    full_idx = np.full((L, 2, K + 1), -1, np.int32)
    full_lg = np.zeros((L, 2, K + 1))
    full_idx[L - 1], full_lg[L - 1] = other[0], lg[0]
    O, _, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], full_idx, full_lg, shape.cu_seqlens, B,
                                rows=np.array([L - 1]))
    np.testing.assert_allclose(O2, O, rtol=1e-11, atol=1e-12)
    assert np.abs(O2 - O0).max() > 1e-6
