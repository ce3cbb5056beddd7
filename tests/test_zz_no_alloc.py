"""sas_decode_noalloc: the decode step for callers that cannot allocate device memory.

It runs the same kernels as sas_decode with the scratch in a fixed array inside the
library. Checked here through the C ABI against sas_decode (caller workspace) on two calls
in a row, plus the size limit. This file is collected last on purpose."""
import ctypes

import pytest
import torch

import sas_inputs as si
from parity_utils import assert_out_close

pytestmark = pytest.mark.gpu


def test_decode_noalloc_matches_decode_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gated_block_sparse_sas_b200 as sas
    lib = sas.lib_handle()
    shp = si.DecodeShape([3000, 65, 1, 1777], 4096, 16, 4, 128, 64, 31, 128, seed=600)
    g = {k: v.cuda() for k, v in si.decode_inputs(shp).items()}
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=shp.capacity, num_q_heads=16,
                             num_kv_heads=4, head_dim=128, block=64, topk=31, gate_hidden=128,
                             dtype=torch.bfloat16)
    ref, ridx, _ = sas.sas_decode(prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"],
                                  g["gate_key_cache"], g["cur_pool"], g["wq"], g["qnorm_w"],
                                  g["wk"], g["knorm_w"], want_selection=True)
    args = [g[k].data_ptr() for k in ("q", "q_nope", "k_cache", "v_cache", "gate_key_cache",
                                      "cur_pool", "wq", "qnorm_w", "wk", "knorm_w")]
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(ref, float("nan"))
        idx = torch.full_like(ridx, -7)
        logg = torch.empty(ridx.shape, dtype=torch.float32, device="cuda")
        st = lib.sas_decode_noalloc(prob.ref, *args, o.data_ptr(), idx.data_ptr(), logg.data_ptr(),
                                    stream)
        assert st == 0, lib.sas_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(idx, ridx), f"call {call}: selection differs"
        assert_out_close(o, ref, False, f"O (call {call})")
        assert sas.decode_noalloc_error_code() == 0


def test_decode_noalloc_error_word_is_per_call():
    """A planted row beyond the decode's fixed softmax reference (a key whose logit exceeds the
    newest token's own-key logit by ~170 nats) sets error 61 in the built-in scratch's error
    word; the next, clean call clears it."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gated_block_sparse_sas_b200 as sas
    lib = sas.lib_handle()
    shp = si.DecodeShape([500, 300], 1024, 8, 2, 128, 64, 31, 128, seed=602)
    clean = {k: v.cuda() for k, v in si.decode_inputs(shp).items()}
    bad = {k: v.clone() for k, v in clean.items()}
    bad["q"][0, 2] = 0.0
    bad["q"][0, 2, 0] = 44.0
    bad["k_cache"][0, 0, 10] = 0.0
    bad["k_cache"][0, 0, 10, 0] = 44.0
    bad["k_cache"][0, 0, 499] = 0.0
    prob = sas.DecodeProblem(seqlens=clean["lengths"], capacity=shp.capacity, num_q_heads=8,
                             num_kv_heads=2, head_dim=128, block=64, topk=31, gate_hidden=128,
                             dtype=torch.bfloat16)
    stream = torch.cuda.current_stream().cuda_stream
    o = torch.empty((2, 8, 128), dtype=torch.bfloat16, device="cuda")
    for inp, want in ((bad, 61), (clean, 0), (bad, 61)):
        args = [inp[k].data_ptr() for k in ("q", "q_nope", "k_cache", "v_cache",
                                            "gate_key_cache", "cur_pool", "wq", "qnorm_w", "wk",
                                            "knorm_w")]
        st = lib.sas_decode_noalloc(prob.ref, *args, o.data_ptr(), None, None, stream)
        assert st == 0, lib.sas_last_error().decode()
        assert sas.decode_noalloc_error_code() == want


def test_decode_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gated_block_sparse_sas_b200 as sas
    lib = sas.lib_handle()
    lengths = torch.ones(4096, dtype=torch.int32, device="cuda")
    big = sas.DecodeProblem(seqlens=lengths, capacity=64, num_q_heads=64, num_kv_heads=8,
                            head_dim=128, block=64, topk=31, gate_hidden=128, dtype=torch.bfloat16)
    n = ctypes.c_size_t(0)
    assert lib.sas_decode_workspace_size(big.ref, ctypes.byref(n)) == 0
    assert n.value > 8 << 20
    st = lib.sas_decode_noalloc(big.ref, *([0x1000] * 13), None)
    assert st == sas.SAS_ERR_UNSUPPORTED
    assert "scratch" in lib.sas_last_error().decode()
