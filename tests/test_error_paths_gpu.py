"""Device-side error reporting through the workspace error word (include/sas.h, "Device-side
errors"), on safe inputs built on the host.

The key-major forward and the tensor-core decode give every row one fixed softmax reference,
the logit of the row's own key (always kept: it sits in the current block) plus 32 in log2
units. A row whose largest logit exceeds its own key's logit by far more than that range
(here ~170 nats) cannot be represented; the kernels report it (code 60 forward, 61 decode),
write that row's output as 0 (and its lse as -inf) and leave every other row exact. The
inputs below plant one such row; nothing faults, the kernels only see large finite values.
"""
import numpy as np
import pytest
import torch

import sas_inputs as si
from oracle import sas_oracle as orc
from parity_utils import assert_out_close, to64

pytestmark = pytest.mark.gpu

BIG = 44.0        # q.k / sqrt(128) = 44^2 / 11.3 ~ 171 nats between the planted key and the own key


@pytest.fixture(scope="module")
def sas():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gated_block_sparse_sas_b200 as m
    return m


def _planted_prefill(seed=900):
    shape = si.Shape([300, 200], 8, 2, 128, 64, 3, 128, "bf16", seed=seed)
    inp = si.prefill_inputs(shape)
    idx, logg = si.random_selection(shape)
    t0, kv0, i0 = 250, 1, 10          # row 250 of sequence 0 keeps blocks 0..3 (c = 3 <= K)
    h0 = kv0 * shape.group + 1
    assert 0 in idx[t0, kv0]
    q, k = inp["q"].clone(), inp["k"].clone()
    q[t0, h0] = 0.0
    q[t0, h0, 0] = BIG
    k[i0, kv0] = 0.0
    k[i0, kv0, 0] = BIG
    k[t0, kv0] = 0.0                   # own key: logit 0
    inp["q"], inp["k"] = q, k
    return shape, inp, idx, logg, (t0, h0)


def test_forward_reports_a_row_beyond_the_reference(sas):
    shape, inp, idx, logg, (t0, h0) = _planted_prefill()
    dev = torch.device("cuda:0")
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=8, num_kv_heads=2, head_dim=128,
                                    block=64, topk=3, gate_hidden=128, dtype=torch.bfloat16)
    g = {k: v.to(dev) for k, v in inp.items()}
    ti, tl = torch.from_numpy(idx).to(dev), torch.from_numpy(logg).to(dev)
    ws = sas.attn_fwd_workspace(prob)
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], ti, tl, workspace=ws)
    torch.cuda.synchronize()
    assert sas.error_code(ws) == 60
    assert torch.count_nonzero(o[t0, h0]).item() == 0
    assert lse[t0, h0].item() == float("-inf")
    # every other row is untouched by the planted one
    O, LSE, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, shape.cu_seqlens, 64)
    keep = np.ones((shape.total_tokens, 8), dtype=bool)
    keep[t0, h0] = False
    assert_out_close(to64(o)[keep], O[keep], False, "O (other rows)")
    assert np.abs(to64(lse)[keep] - LSE[keep]).max() <= 2e-3
    with pytest.raises(sas.SasDeviceError, match="code 60"):
        sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], ti, tl, workspace=ws, check=True)
    # the next call on the same workspace clears the word: clean inputs report 0
    clean = si.prefill_inputs(shape)
    sas.sas_attn_fwd(prob, clean["q"].to(dev), clean["k"].to(dev), clean["v"].to(dev), ti, tl,
                     workspace=ws, check=True)
    assert sas.error_code(ws) == 0


def _planted_decode(seed=901):
    shp = si.DecodeShape([500, 300], 1024, 8, 2, 128, 64, 31, 128, seed=seed)
    inp = si.decode_inputs(shp)
    b0, kv0, i0 = 0, 0, 10            # 500 tokens: 8 blocks, all kept under K = 31
    h0 = kv0 * shp.group + 2
    L = shp.lengths[b0]
    q, kc = inp["q"].clone(), inp["k_cache"].clone()
    q[b0, h0] = 0.0
    q[b0, h0, 0] = BIG
    kc[b0, kv0, i0] = 0.0
    kc[b0, kv0, i0, 0] = BIG
    kc[b0, kv0, L - 1] = 0.0           # the newest token's own key: logit 0
    inp["q"], inp["k_cache"] = q, kc
    return shp, inp, (b0, h0)


def test_decode_reports_a_row_beyond_the_reference(sas):
    shp, inp, (b0, h0) = _planted_decode()
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=shp.capacity, num_q_heads=8,
                             num_kv_heads=2, head_dim=128, block=64, topk=31, gate_hidden=128,
                             dtype=torch.bfloat16)
    ws = sas._workspace(sas.lib_handle().sas_decode_workspace_size, prob.ref, prob.device)
    args = (prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"], g["gate_key_cache"],
            g["cur_pool"], g["wq"], g["qnorm_w"], g["wk"], g["knorm_w"])
    o = sas.sas_decode(*args, workspace=ws)
    torch.cuda.synchronize()
    assert sas.error_code(ws) == 61
    assert torch.count_nonzero(o[b0, h0]).item() == 0
    O, _, _, _ = orc.decode(inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"], shp.lengths,
                            inp["gate_key_cache"], inp["cur_pool"], inp["wq"], inp["qnorm_w"],
                            inp["wk"], inp["knorm_w"], 64, 31, 1e-6, 1e6)
    keep = np.ones((2, 8), dtype=bool)
    keep[b0, h0] = False
    assert_out_close(to64(o)[keep], O[keep], False, "O (other heads)")
    with pytest.raises(sas.SasDeviceError, match="code 61"):
        sas.sas_decode(*args, workspace=ws, check=True)
    clean = {k: v.cuda() for k, v in si.decode_inputs(shp).items()}
    sas.sas_decode(prob, clean["q"], clean["q_nope"], clean["k_cache"], clean["v_cache"],
                   clean["gate_key_cache"], clean["cur_pool"], clean["wq"], clean["qnorm_w"],
                   clean["wk"], clean["knorm_w"], workspace=ws, check=True)
    assert sas.error_code(ws) == 0
