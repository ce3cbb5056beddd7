"""Pin for the oracle's router backward (gate parameter gradients with the selection fixed):
central finite differences in fp64 of L = sum(dlogg * logg) through the oracle's forward
(pool -> gate keys -> gate scores -> log-gates gathered at the fixed selection)."""
import numpy as np
import pytest

import sas_inputs as si
from oracle import sas_oracle as orc


def _setup():
    shape = si.Shape([40, 23], 4, 2, 8, 8, 2, 8, "fp32", seed=77)
    inp = si.prefill_inputs(shape)
    cu = np.asarray(shape.cu_seqlens)
    sel = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"],
                                inp["wk"], inp["knorm_w"], cu, shape.block, shape.topk, 1e-6, 1e6)
    rng = np.random.default_rng(5)
    dlogg = rng.standard_normal(sel["idx"].shape) * (sel["idx"] >= 0)   # a generic dlogg
    return shape, inp, cu, sel["idx"], dlogg


def _loss(shape, inp, cu, idx, dlogg, wq, qw, wk, kw):
    lengths = np.diff(cu)
    nbm = int((lengths.max() + shape.block - 1) // shape.block)
    pooled = orc.pool_keys(inp["k_nope"], cu, shape.block, nbm)
    gk = orc.gate_keys(pooled, wk, kw, shape.block, 1e-6, 1e6, lengths)
    s, lse, _ = orc.gate_scores(inp["q_nope"], inp["k_nope"], gk, wq, qw, wk, kw, cu, shape.block,
                                1e-6, 1e6)
    T, Hkv, K1 = idx.shape
    tot = 0.0
    for t in range(T):
        for kv in range(Hkv):
            for sl in range(K1):
                j = idx[t, kv, sl]
                if j >= 0:
                    tot += dlogg[t, kv, sl] * (s[t, kv, j] - lse[t, kv])
    return tot


@pytest.mark.parametrize("param", ["wq", "qnorm_w", "wk", "knorm_w"])
def test_gate_backward_matches_finite_differences(param):
    shape, inp, cu, idx, dlogg = _setup()
    base = {n: orc.as64(inp[n]) for n in ("wq", "qnorm_w", "wk", "knorm_w")}
    grads = orc.gate_backward(inp["q_nope"], inp["k_nope"], base["wq"], base["qnorm_w"], base["wk"],
                              base["knorm_w"], idx, dlogg, cu, shape.block, 1e-6, 1e6)
    g = grads[{"wq": "dwq", "qnorm_w": "dqnorm_w", "wk": "dwk", "knorm_w": "dknorm_w"}[param]]
    rng = np.random.default_rng(11)
    flat = [tuple(int(v) for v in np.unravel_index(i, g.shape))
            for i in rng.choice(g.size, size=min(8, g.size), replace=False)]
    eps = 1e-6
    for ix in flat:
        plus = {n: v.copy() for n, v in base.items()}
        minus = {n: v.copy() for n, v in base.items()}
        plus[param][ix] += eps
        minus[param][ix] -= eps
        fd = (_loss(shape, inp, cu, idx, dlogg, plus["wq"], plus["qnorm_w"], plus["wk"], plus["knorm_w"])
              - _loss(shape, inp, cu, idx, dlogg, minus["wq"], minus["qnorm_w"], minus["wk"],
                      minus["knorm_w"])) / (2 * eps)
        assert abs(fd - g[ix]) <= 1e-6 * max(1.0, abs(fd)), (param, ix, fd, g[ix])

