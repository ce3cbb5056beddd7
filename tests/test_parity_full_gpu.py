"""GPU parity at the benchmark's full sizes, in the launch configuration bench.py times.

The oracle computes sampled outputs one by one: Top-K rows, attention rows, dQ/dlogg rows
and dK/dV of sampled key blocks, decode steps of sampled sequences. Inputs are drawn on the
GPU by the seeded generator and copied to the host for the oracle (the generator's output,
identical to a host draw). Tolerances: tests/parity_utils.py."""
import numpy as np
import pytest
import torch

import sas_inputs as si
from oracle import sas_oracle as orc
from parity_utils import assert_grad_close, assert_out_close, compare_selection, to64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def sas():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gated_block_sparse_sas_b200 as m
    return m


def _problem(sas, shape, dev):
    return sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=shape.num_q_heads,
                                    num_kv_heads=shape.num_kv_heads, head_dim=shape.head_dim,
                                    block=shape.block, topk=shape.topk,
                                    gate_hidden=shape.gate_hidden, dtype=shape.torch_dtype)


def _rows(shape, n, seed):
    r = np.random.Generator(np.random.PCG64(seed))
    pick = list(r.choice(shape.total_tokens, size=n - 4, replace=False))
    ends = list(np.cumsum(shape.lengths) - 1)
    return np.unique(np.array(pick + [0, 63, 64] + ends[:1]))


@pytest.mark.parametrize("name", ["qwen3-4b-prefill-32k", "qwen3-14b-varlen-4seq"])
def test_prefill_full_size_sampled(sas, name):
    shape = si.workload(name)
    dev = torch.device("cuda:0")
    g = si.prefill_inputs(shape, device=dev)
    prob = _problem(sas, shape, dev)
    ws = sas.attn_fwd_workspace(prob)
    idx, logg = sas.prefill_selection(prob, g["q_nope"], g["k_nope"], g["wq"], g["qnorm_w"],
                                      g["wk"], g["knorm_w"])
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], idx, logg, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    cpu = {k: v.cpu() for k, v in g.items()}
    rows = _rows(shape, 28, 11)
    ref = orc.prefill_selection(cpu["q_nope"], cpu["k_nope"], cpu["wq"], cpu["qnorm_w"],
                                cpu["wk"], cpu["knorm_w"], shape.cu_seqlens, shape.block,
                                shape.topk, shape.rms_eps, shape.gate_rope_base, rows)
    ig = idx.cpu().numpy()[rows]
    compare_selection(ig, logg.cpu().numpy()[rows], ref["idx"], ref["logg"], ref["margin"])
    same = (ig == ref["idx"]).all(axis=-1).all(axis=-1)
    full_idx = np.full(idx.shape, -1, np.int32)
    full_lg = np.zeros(idx.shape)
    full_idx[rows], full_lg[rows] = ref["idx"], ref["logg"]
    O, LSE, _ = orc.attention_fwd(cpu["q"], cpu["k"], cpu["v"], full_idx, full_lg,
                                  shape.cu_seqlens, shape.block, rows=rows[same])
    assert_out_close(o.cpu()[rows[same]], O, False, "O")
    assert np.abs(to64(lse.cpu()[rows[same]]) - LSE).max() <= 2e-3


def test_train_full_size_backward_sampled(sas):
    shape = si.workload("qwen3-4b-train-32k")
    dev = torch.device("cuda:0")
    g = si.prefill_inputs(shape, device=dev, with_dout=True)
    prob = _problem(sas, shape, dev)
    idx, logg = si.random_selection(shape)
    ti, tl = torch.from_numpy(idx).to(dev), torch.from_numpy(logg).to(dev)
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], ti, tl)
    dq, dk, dv, dl = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o, g["dout"], lse, ti, tl)
    torch.cuda.synchronize()
    cpu = {k: v.cpu() for k, v in g.items()}
    rows = _rows(shape, 12, 12)
    dq_r, dl_r = orc.attention_bwd_rows(cpu["q"], cpu["k"], cpu["v"], cpu["dout"], idx, logg,
                                        shape.cu_seqlens, shape.block, rows)
    assert_grad_close(dq.cpu()[rows], dq_r, False, "dQ rows")
    assert_grad_close(dl.cpu()[rows], dl_r, False, "dlogg rows")
    for j, kv in ((3, 0), (300, 5)):
        dk_r, dv_r = orc.attention_bwd_keys(cpu["q"], cpu["k"], cpu["v"], cpu["dout"], idx, logg,
                                            shape.cu_seqlens, shape.block, 0, kv, j * 64,
                                            (j + 1) * 64)
        assert_grad_close(dk.cpu()[j * 64:(j + 1) * 64, kv], dk_r, False, f"dK block {j}")
        assert_grad_close(dv.cpu()[j * 64:(j + 1) * 64, kv], dv_r, False, f"dV block {j}")


def test_varlen_full_size_backward_sampled(sas):
    """The 14B varlen workload (4 packed sequences, G 5, K 63) forward + backward at full size
    on the gate's own selection, as bench.py runs it: dQ/dlogg rows and dK/dV of late blocks
    (few query rows reach them, so the oracle stays small) against the oracle."""
    shape = si.workload("qwen3-14b-varlen-4seq")
    dev = torch.device("cuda:0")
    g = si.prefill_inputs(shape, device=dev, with_dout=True)
    prob = _problem(sas, shape, dev)
    idx, logg = sas.prefill_selection(prob, g["q_nope"], g["k_nope"], g["wq"], g["qnorm_w"],
                                      g["wk"], g["knorm_w"])
    wsf, wsb = sas.attn_fwd_workspace(prob), sas.attn_bwd_workspace(prob)
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], idx, logg, workspace=wsf)
    dq, dk, dv, dl = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o, g["dout"], lse, idx, logg,
                                      workspace=wsb)
    torch.cuda.synchronize()
    assert sas.error_code(wsf) == 0 and sas.error_code(wsb) == 0
    cpu = {k: v.cpu() for k, v in g.items()}
    ig, lg = idx.cpu().numpy(), logg.cpu().numpy()
    rows = _rows(shape, 12, 13)
    dq_r, dl_r = orc.attention_bwd_rows(cpu["q"], cpu["k"], cpu["v"], cpu["dout"], ig, lg,
                                        shape.cu_seqlens, shape.block, rows)
    assert_grad_close(dq.cpu()[rows], dq_r, False, "dQ rows")
    assert_grad_close(dl.cpu()[rows], dl_r, False, "dlogg rows")
    b = int(np.argmin(shape.lengths))
    L, s0 = shape.lengths[b], int(shape.cu_seqlens[b])
    nb = (L + 63) // 64
    for j, kv in ((nb - 4, 0), (nb - 1, 7)):
        lo, hi = j * 64, min((j + 1) * 64, L)
        dk_r, dv_r = orc.attention_bwd_keys(cpu["q"], cpu["k"], cpu["v"], cpu["dout"], ig, lg,
                                            shape.cu_seqlens, shape.block, b, kv, lo, hi)
        assert_grad_close(dk.cpu()[s0 + lo:s0 + hi, kv], dk_r, False, f"dK block {j}")
        assert_grad_close(dv.cpu()[s0 + lo:s0 + hi, kv], dv_r, False, f"dV block {j}")


def test_decode_full_size_sampled(sas):
    shp = si.decode_workload("qwen3-8b-decode-b64")
    dev = torch.device("cuda:0")
    g = si.decode_inputs(shp, device=dev)
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=shp.capacity,
                             num_q_heads=shp.num_q_heads, num_kv_heads=shp.num_kv_heads,
                             head_dim=shp.head_dim, block=shp.block, topk=shp.topk,
                             gate_hidden=shp.gate_hidden, dtype=torch.bfloat16)
    o, idx, logg = sas.sas_decode(prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"],
                                  g["gate_key_cache"], g["cur_pool"], g["wq"], g["qnorm_w"],
                                  g["wk"], g["knorm_w"], want_selection=True)
    torch.cuda.synchronize()
    L = np.array(shp.lengths)
    pick = sorted({0, 17, 63, int(L.argmin()), int(L.argmax())} |
                  set(np.random.default_rng(14).choice(64, 8, replace=False).tolist()))
    for b in pick:
        sl = slice(b, b + 1)
        O, ridx, rlogg, margin = orc.decode(
            g["q"][sl].cpu(), g["q_nope"][sl].cpu(), g["k_cache"][sl].cpu(), g["v_cache"][sl].cpu(),
            [shp.lengths[b]], g["gate_key_cache"][sl].cpu(), g["cur_pool"][sl].cpu(), g["wq"].cpu(),
            g["qnorm_w"].cpu(), g["wk"].cpu(), g["knorm_w"].cpu(), shp.block, shp.topk,
            shp.rms_eps, shp.gate_rope_base)
        compare_selection(idx[sl].cpu().numpy(), logg[sl].cpu(), ridx, rlogg, margin)
        if (idx[sl].cpu().numpy() == ridx).all():
            assert_out_close(o[sl].cpu(), O, False, f"O seq {b}")
        else:   # a near-tie: the oracle's attention on the GPU's own selection
            Og, _, _, _ = orc.decode(
                g["q"][sl].cpu(), g["q_nope"][sl].cpu(), g["k_cache"][sl].cpu(),
                g["v_cache"][sl].cpu(), [shp.lengths[b]], g["gate_key_cache"][sl].cpu(),
                g["cur_pool"][sl].cpu(), g["wq"].cpu(), g["qnorm_w"].cpu(), g["wk"].cpu(),
                g["knorm_w"].cpu(), shp.block, shp.topk, shp.rms_eps, shp.gate_rope_base,
                selection=(idx[sl].cpu().numpy(), logg[sl].cpu().numpy()))
            assert_out_close(o[sl].cpu(), Og, False, f"O seq {b} (GPU selection)")
