"""Pin for the oracle's decode: one decode step equals the prefill row of the newest token
when its caches hold that prefill's own gate keys and running pool state."""
import numpy as np
import pytest

import sas_inputs as si
from oracle import sas_oracle as orc


@pytest.mark.parametrize("L", [1, 16, 17, 63, 100, 128])
def test_decode_equals_prefill_last_row(L):
    B, K, h = 16, 3, 16
    shape = si.Shape([L], 4, 2, 8, B, K, h, "fp32", seed=20 + L)
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
