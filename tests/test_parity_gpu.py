"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle, element by
element on the same seeded inputs. Small cases span several tiles and ragged tails;
tolerances are those stated in tests/parity_utils.py."""
import numpy as np
import pytest
import torch

import sas_inputs as si
from oracle import sas_oracle as orc
from parity_utils import (assert_grad_close, assert_out_close, assert_paths_agree,
                          compare_selection, rel_l2, to64, GATE_ABS, PATHS_GATE_ABS)

pytestmark = pytest.mark.gpu

CASES = {
    # lengths, Hq, Hkv, d, B, K, h, dtype
    "bf16-d128-B64-ragged": ([300, 64, 1, 130], 8, 2, 128, 64, 3, 128, "bf16"),
    "bf16-d128-B64-G5": ([513, 77], 10, 2, 128, 64, 4, 128, "bf16"),
    "bf16-d64-B32": ([257, 33], 8, 4, 64, 32, 5, 64, "bf16"),
    "fp32-d64-B16-tiny-shape": ([1024], 2, 1, 64, 16, 4, 32, "fp32"),
    "bf16-d128-B16-K-large": ([200], 4, 1, 128, 16, 20, 32, "bf16"),
}


@pytest.fixture(scope="module")
def sas():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gated_block_sparse_sas_b200 as m
    return m


def _setup(sas, name, seed=100):
    lengths, Hq, Hkv, d, B, K, h, dt = CASES[name]
    shape = si.Shape(list(lengths), Hq, Hkv, d, B, K, h, dt, seed=seed)
    inp = si.prefill_inputs(shape, with_dout=True)
    dev = torch.device("cuda:0")
    g = {k: v.to(dev) for k, v in inp.items()}
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=Hq, num_kv_heads=Hkv,
                                    head_dim=d, block=B, topk=K, gate_hidden=h,
                                    dtype=shape.torch_dtype)
    return shape, inp, g, prob


@pytest.mark.parametrize("name", list(CASES))
def test_gate_pipeline(sas, name):
    shape, inp, g, prob = _setup(sas, name)
    pooled = sas.sas_pool_keys(prob, g["k_nope"])
    gk = sas.sas_gate_keys(prob, pooled, g["wk"], g["knorm_w"])
    scores, lse = sas.sas_gate_scores(prob, g["q_nope"], g["k_nope"], gk, g["wq"], g["qnorm_w"],
                                      g["wk"], g["knorm_w"])
    idx, logg = sas.sas_topk(prob, scores, lse)
    torch.cuda.synchronize()
    ref = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, shape.block, shape.topk, 1e-6, 1e6)
    np.testing.assert_allclose(to64(pooled), ref["pooled"], rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(to64(gk), ref["gate_keys"], rtol=0, atol=GATE_ABS)
    s, sr = to64(scores), ref["scores"]
    assert (np.isneginf(s) == np.isneginf(sr)).all()
    fin = np.isfinite(sr)
    assert np.abs(s[fin] - sr[fin]).max() <= GATE_ABS
    assert np.abs(to64(lse) - ref["lse"]).max() <= GATE_ABS
    n, near, flips = compare_selection(idx.cpu().numpy(), logg, ref["idx"], ref["logg"], ref["margin"])
    assert near <= max(2, 0.01 * n)


@pytest.mark.parametrize("name", list(CASES))
def test_attention_forward(sas, name):
    shape, inp, g, prob = _setup(sas, name, seed=200)
    idx, logg = si.random_selection(shape)
    ws = sas.attn_fwd_workspace(prob)
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], torch.from_numpy(idx).cuda(),
                              torch.from_numpy(logg).cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "tensor-core pipeline reported a timeout"
    O, LSE, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, shape.cu_seqlens,
                                  shape.block)
    fp32 = shape.dtype == "fp32"
    assert_out_close(o, O, fp32, "O")
    assert np.abs(to64(lse) - LSE).max() <= (1e-4 if fp32 else 2e-3)


WINDOW_CASES = {
    # lengths, Hq, Hkv, K: several 4096-token windows of the key-major forward, ragged tails,
    # sequences shorter than a block, G = 4, 5, 8
    "windows-G4": ([9000, 4100, 70], 8, 2, 7),
    "windows-G5": ([4097, 5000, 1], 10, 2, 15),
    "windows-G8": ([8200, 300], 16, 2, 31),
    # the 14B varlen workload's group and budget: G = 5, K = 63 (4,096-token budget)
    "windows-G5-K63": ([9000, 4500, 130], 10, 2, 63),
}


@pytest.mark.parametrize("name", list(WINDOW_CASES))
def test_attention_forward_windows(sas, name):
    """Forward over several token windows; every row of the GPU output is computed, the
    oracle checks window edges, block edges, sequence ends and a random sample."""
    lengths, Hq, Hkv, K = WINDOW_CASES[name]
    shape = si.Shape(list(lengths), Hq, Hkv, 128, 64, K, 128, "bf16", seed=400)
    inp = si.prefill_inputs(shape, with_dout=False)
    dev = torch.device("cuda:0")
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=Hq, num_kv_heads=Hkv,
                                    head_dim=128, block=64, topk=K, gate_hidden=128,
                                    dtype=torch.bfloat16)
    idx, logg = si.random_selection(shape)
    ws = sas.attn_fwd_workspace(prob)
    o, lse = sas.sas_attn_fwd(prob, inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev),
                              torch.from_numpy(idx).to(dev), torch.from_numpy(logg).to(dev),
                              workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "tensor-core pipeline reported an error"
    o64, lse64 = to64(o), to64(lse)
    assert np.isfinite(o64).all() and np.isfinite(lse64).all()
    rng = np.random.default_rng(401)
    rows = set()
    for b, (s0, s1) in enumerate(zip(shape.cu_seqlens[:-1], shape.cu_seqlens[1:])):
        L = int(s1 - s0)
        for tl in (0, 1, 63, 64, 65, 4095, 4096, 4097, 8191, 8192, L - 2, L - 1):
            if 0 <= tl < L:
                rows.add(int(s0) + tl)
    rows |= set(rng.choice(shape.total_tokens, 120, replace=False).tolist())
    rows = np.array(sorted(rows))
    O, LSE, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, shape.cu_seqlens,
                                  shape.block, rows=rows)
    assert_out_close(o[torch.from_numpy(rows).to(dev)], O, False, "O")
    assert np.abs(lse64[rows] - LSE).max() <= 2e-3


@pytest.mark.parametrize("name", list(WINDOW_CASES))
def test_attention_backward_windows(sas, name):
    """Backward over several token windows: dQ/dlogg on window, block and sequence edges plus
    random rows; dK/dV on first, middle and last (ragged) blocks of every sequence."""
    lengths, Hq, Hkv, K = WINDOW_CASES[name]
    shape = si.Shape(list(lengths), Hq, Hkv, 128, 64, K, 128, "bf16", seed=500)
    inp = si.prefill_inputs(shape, with_dout=True)
    dev = torch.device("cuda:0")
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=Hq, num_kv_heads=Hkv,
                                    head_dim=128, block=64, topk=K, gate_hidden=128,
                                    dtype=torch.bfloat16)
    g = {k: v.to(dev) for k, v in inp.items()}
    idx, logg = si.random_selection(shape)
    ti, tl = torch.from_numpy(idx).to(dev), torch.from_numpy(logg).to(dev)
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], ti, tl)
    ws = sas.attn_bwd_workspace(prob)
    dq, dk, dv, dl = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o, g["dout"], lse, ti, tl,
                                      workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0, "tensor-core pipeline reported an error"
    rng = np.random.default_rng(501)
    rows = set()
    cu = shape.cu_seqlens
    for s0, s1 in zip(cu[:-1], cu[1:]):
        L = int(s1 - s0)
        for t in (0, 63, 64, 4095, 4096, 8191, 8192, L - 1):
            if 0 <= t < L:
                rows.add(int(s0) + t)
    rows |= set(rng.choice(shape.total_tokens, 40, replace=False).tolist())
    rows = np.array(sorted(rows))
    dq_r, dl_r = orc.attention_bwd_rows(inp["q"], inp["k"], inp["v"], inp["dout"], idx, logg,
                                        cu, shape.block, rows)
    assert_grad_close(dq.cpu()[rows], dq_r, False, "dQ rows")
    assert_grad_close(dl.cpu()[rows], dl_r, False, "dlogg rows")
    assert (to64(dl)[idx < 0] == 0).all()
    for b, (s0, s1) in enumerate(zip(cu[:-1], cu[1:])):
        L = int(s1 - s0)
        nb = (L + 63) // 64
        for j, kv in sorted({(0, 0), (nb // 2, Hkv - 1), (nb - 1, 0)}):
            lo, hi = j * 64, min((j + 1) * 64, L)
            dk_r, dv_r = orc.attention_bwd_keys(inp["q"], inp["k"], inp["v"], inp["dout"], idx,
                                                logg, cu, shape.block, b, kv, lo, hi)
            gk = dk.cpu()[int(s0) + lo:int(s0) + hi, kv]
            if np.linalg.norm(dk_r) < 1e-9:
                # a one-token sequence: P = 1, so dS = dP - D = 0 and dK = 0 in exact
                # arithmetic; only rounding noise of dP - D is left on the GPU
                assert np.abs(to64(gk)).max() <= 1e-4, f"dK seq {b} block {j} not ~0"
            else:
                assert_grad_close(gk, dk_r, False, f"dK seq {b} block {j}")
            assert_grad_close(dv.cpu()[int(s0) + lo:int(s0) + hi, kv], dv_r, False,
                              f"dV seq {b} block {j}")


@pytest.mark.parametrize("name", list(CASES))
def test_attention_backward(sas, name):
    shape, inp, g, prob = _setup(sas, name, seed=300)
    idx, logg = si.random_selection(shape)
    ti, tl = torch.from_numpy(idx).cuda(), torch.from_numpy(logg).cuda()
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], ti, tl)
    dq, dk, dv, dl = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o, g["dout"], lse, ti, tl)
    torch.cuda.synchronize()
    ref = orc.attention_bwd(inp["q"], inp["k"], inp["v"], inp["dout"], idx, logg, shape.cu_seqlens,
                            shape.block)
    fp32 = shape.dtype == "fp32"
    for gpu, r, nm in zip((dq, dk, dv, dl), ref, ("dQ", "dK", "dV", "dlogg")):
        assert_grad_close(gpu, r, fp32, nm)
    assert (to64(dl)[idx < 0] == 0).all()


def test_tiny_config_end_to_end(sas):
    """The tiny fp32 workload: gate -> Top-K -> attention fwd/bwd on the GPU against the oracle."""
    shape = si.workload("tiny-fp32-T1024")
    inp = si.prefill_inputs(shape, with_dout=True)
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.Problem.from_lengths(shape.lengths, torch.device("cuda:0"), num_q_heads=2,
                                    num_kv_heads=1, head_dim=64, block=16, topk=4, gate_hidden=32,
                                    dtype=torch.float32)
    idx, logg = sas.prefill_selection(prob, g["q_nope"], g["k_nope"], g["wq"], g["qnorm_w"],
                                      g["wk"], g["knorm_w"])
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], idx, logg)
    dq, dk, dv, dl = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o, g["dout"], lse, idx, logg)
    torch.cuda.synchronize()
    ref = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, 16, 4, 1e-6, 1e6)
    compare_selection(idx.cpu().numpy(), logg, ref["idx"], ref["logg"], ref["margin"])
    # attention against the oracle on the oracle's own selection (identical except near-ties)
    ri, rl = ref["idx"], ref["logg"].astype(np.float32)
    o2, lse2 = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], torch.from_numpy(ri).cuda(),
                                torch.from_numpy(rl).cuda())
    O, _, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], ri, rl, shape.cu_seqlens, 16)
    assert_out_close(o2, O, True, "O")
    grads = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o2, g["dout"], lse2,
                             torch.from_numpy(ri).cuda(), torch.from_numpy(rl).cuda())
    refg = orc.attention_bwd(inp["q"], inp["k"], inp["v"], inp["dout"], ri, rl, shape.cu_seqlens, 16)
    for gpu, r, nm in zip(grads, refg, ("dQ", "dK", "dV", "dlogg")):
        assert_grad_close(gpu, r, True, nm)


DEC_CASES = {
    "bf16-d128-B64": ([1, 64, 65, 700, 2048, 1500], 2048, 8, 2, 128, 64, 7, 128),
    "bf16-d128-B64-G4-K31": ([4000, 129, 2500], 4096, 16, 4, 128, 64, 31, 128),
    "bf16-d64-B16": ([30, 17, 300], 512, 4, 2, 64, 16, 5, 32),
    # the card's other decode budgets: 1,024 tokens (K 15) and 4,096 tokens (K 63)
    "bf16-budget1024-K15": ([3000, 1100, 70, 2048], 4096, 32, 8, 128, 64, 15, 128),
    "bf16-budget4096-K63": ([6000, 4200, 130, 5000], 8192, 16, 4, 128, 64, 63, 128),
    # 40 sequences x 8 KV heads of mixed lengths
    "bf16-batch40-mixed": (si.draw_lengths(41, 40, 1, 2500), 2560, 32, 8, 128, 64, 15, 128),
}


@pytest.mark.parametrize("name,gated", [(n, True) for n in DEC_CASES] +
                         [("bf16-d128-B64-G4-K31", False), ("bf16-d64-B16", False)])
def test_decode(sas, name, gated):
    lengths, cap, Hq, Hkv, d, B, K, h = DEC_CASES[name]
    shp = si.DecodeShape(list(lengths), cap, Hq, Hkv, d, B, K, h, seed=400)
    inp = si.decode_inputs(shp)
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=cap, num_q_heads=Hq, num_kv_heads=Hkv,
                             head_dim=d, block=B, topk=K, gate_hidden=h, dtype=torch.bfloat16,
                             gated=gated)
    o, idx, logg = sas.sas_decode(prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"],
                                  g["gate_key_cache"], g["cur_pool"], g["wq"], g["qnorm_w"], g["wk"],
                                  g["knorm_w"], want_selection=True)
    torch.cuda.synchronize()
    O, ridx, rlogg, margin = orc.decode(inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"],
                                        lengths, inp["gate_key_cache"], inp["cur_pool"], inp["wq"],
                                        inp["qnorm_w"], inp["wk"], inp["knorm_w"], B, K, 1e-6, 1e6,
                                        gated=gated)
    compare_selection(idx.cpu().numpy(), logg, ridx, rlogg, margin)
    same = (idx.cpu().numpy() == ridx).all(axis=-1).all(axis=-1)
    assert_out_close(o[torch.from_numpy(same)], O[same], False, "O")
    # near-tie rows: the oracle's attention evaluated on the GPU's own selection
    if not same.all():
        Og, _, _, _ = orc.decode(inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"], lengths,
                                 inp["gate_key_cache"], inp["cur_pool"], inp["wq"], inp["qnorm_w"],
                                 inp["wk"], inp["knorm_w"], B, K, 1e-6, 1e6, gated=gated,
                                 selection=(idx.cpu().numpy(), logg.cpu().numpy()))
        assert_out_close(o[torch.from_numpy(~same)], Og[~same], False, "O (near-tie rows)")


FUSED_CASES = {
    # (lengths, capacity, Hq, Hkv, d, B, K, h, gate_heads or None, gated, paged)
    "K31-G4": ([4000, 129, 2500, 1, 64, 65], 4096, 16, 4, 128, 64, 31, 128, None, True, False),
    "K63-G5": ([6000, 4200, 130, 5000], 8192, 20, 4, 128, 64, 63, 128, None, True, False),
    "K15-batch40": (si.draw_lengths(43, 40, 1, 2500), 2560, 32, 8, 128, 64, 15, 128, None, True, False),
    "K31-h64-ungated": ([3000, 700, 64], 4096, 16, 4, 128, 64, 31, 64, None, False, False),
    "K15-per-head": ([4200, 300, 65], 4224, 8, 2, 128, 64, 15, 128, 8, True, False),
    "K31-paged": ([3000, 65, 1, 1777, 4096], 4096, 16, 4, 128, 64, 31, 128, None, True, True),
}


@pytest.mark.parametrize("name", list(FUSED_CASES))
def test_decode_fused_equals_three_launch(sas, name):
    """The single persistent decode launch and the three-launch decode select the same blocks
    with the same log-gates (the gate arithmetic is the same, in the same order) and give the
    same O up to the split merge's summation order; both agree with the oracle."""
    lengths, cap, Hq, Hkv, d, B, K, h, gh, gated, paged = FUSED_CASES[name]
    shp = si.DecodeShape(list(lengths), cap, Hq, Hkv, d, B, K, h, seed=420,
                         **({} if gh is None else {"gate_heads": gh}))
    inp = si.decode_inputs(shp)
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=cap, num_q_heads=Hq, num_kv_heads=Hkv,
                             head_dim=d, block=B, topk=K, gate_hidden=h, dtype=torch.bfloat16,
                             gated=gated, **({} if gh is None else {"gate_heads": gh}))
    common = (g["cur_pool"], g["wq"], g["qnorm_w"], g["wk"], g["knorm_w"])
    if paged:
        pt, n_pages, kp, vp, gp = _paged_from_contiguous(inp, shp, 421)
        pt, kp, vp, gp = pt.cuda(), kp.cuda(), vp.cuda(), gp.cuda()
        run = lambda: sas.sas_decode_paged(prob, pt, n_pages, g["q"], g["q_nope"], kp, vp, gp,
                                           *common, want_selection=True, check=True)
    else:
        run = lambda: sas.sas_decode(prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"],
                                     g["gate_key_cache"], *common, want_selection=True, check=True)
    try:
        sas.sas_decode_set_fused(False)
        o3, i3, l3 = run()
        sas.sas_decode_set_fused(True)
        of, i_f, lf = run()
    finally:
        sas.sas_decode_set_fused(True)
    torch.cuda.synchronize()
    assert torch.equal(i_f, i3)
    assert torch.equal(lf, l3)
    assert_out_close(of, o3.float().cpu().numpy(), False, "O fused vs three-launch")
    O, ridx, rlogg, margin = orc.decode(inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"],
                                        lengths, inp["gate_key_cache"], inp["cur_pool"], inp["wq"],
                                        inp["qnorm_w"], inp["wk"], inp["knorm_w"], B, K, 1e-6, 1e6,
                                        gated=gated)
    compare_selection(i_f.cpu().numpy(), lf, ridx, rlogg, margin)
    same = (i_f.cpu().numpy() == ridx).all(axis=-1).all(axis=-1)
    assert_out_close(of[torch.from_numpy(same)], O[same], False, "O")


def test_decode_equals_prefill_row(sas):
    """A decode step over caches written from a prefill equals that prefill's last row."""
    L, B, K, h = 777, 64, 5, 128
    shape = si.Shape([L], 8, 2, 128, B, K, h, "bf16", seed=500)
    inp = si.prefill_inputs(shape)
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.Problem.from_lengths([L], torch.device("cuda:0"), num_q_heads=8, num_kv_heads=2,
                                    head_dim=128, block=B, topk=K, gate_hidden=h,
                                    dtype=torch.bfloat16)
    pooled = sas.sas_pool_keys(prob, g["k_nope"])
    gk = sas.sas_gate_keys(prob, pooled, g["wk"], g["knorm_w"])
    gk_bf = gk.to(torch.bfloat16)
    scores, lse = sas.sas_gate_scores(prob, g["q_nope"], g["k_nope"], gk_bf.float().contiguous(),
                                      g["wq"], g["qnorm_w"], g["wk"], g["knorm_w"])
    idx, logg = sas.sas_topk(prob, scores, lse)
    o, _ = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], idx, logg)
    c = (L - 1) // B
    cur = g["k_nope"][c * B:L].float()
    pool = torch.stack([cur.amax(0), cur.amin(0), cur.sum(0)], dim=1)[None].contiguous()
    dprob = sas.DecodeProblem(seqlens=torch.tensor([L], dtype=torch.int32, device="cuda"),
                              capacity=L, num_q_heads=8, num_kv_heads=2, head_dim=128, block=B,
                              topk=K, gate_hidden=h, dtype=torch.bfloat16)
    od, di, dl = sas.sas_decode(dprob, g["q"][L - 1:L].contiguous(), g["q_nope"][L - 1:L].contiguous(),
                                g["k"].transpose(0, 1)[None].contiguous(),
                                g["v"].transpose(0, 1)[None].contiguous(),
                                gk_bf[0].transpose(0, 1)[None].contiguous(), pool, g["wq"],
                                g["qnorm_w"], g["wk"], g["knorm_w"], want_selection=True)
    torch.cuda.synchronize()
    assert torch.equal(di[0], idx[L - 1])
    assert (dl[0] - logg[L - 1]).abs().max().item() <= GATE_ABS
    assert (od[0].float() - o[L - 1].float()).abs().max().item() <= 2e-2


GATE_BWD_CASES = {
    # lengths, Hq, Hkv, d, B, K, h (bf16; the router backward's supported shape)
    "bf16-G4-K7-ragged": ([700, 300, 64, 1], 16, 4, 128, 64, 7, 128),
    "bf16-G8-K3": ([1100, 129], 16, 2, 128, 64, 3, 128),
    "bf16-G5-K15-long": ([5000, 300], 10, 2, 128, 64, 15, 128),
}


@pytest.mark.parametrize("name", list(GATE_BWD_CASES))
def test_gate_backward(sas, name):
    """Router backward vs the oracle (both fed the GPU's selection): dWq, dWk and the two
    RMSNorm weight gradients, fp32, relative L2 <= 2e-3. dlogg is random with zero row sums
    over the kept slots, as the attention backward's own dlogg has."""
    lengths, Hq, Hkv, d, B, K, h = GATE_BWD_CASES[name]
    shape = si.Shape(list(lengths), Hq, Hkv, d, B, K, h, "bf16", seed=501)
    inp = si.prefill_inputs(shape)
    dev = torch.device("cuda:0")
    g = {k: v.to(dev) for k, v in inp.items() if isinstance(v, torch.Tensor)}
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=Hq, num_kv_heads=Hkv,
                                    head_dim=d, block=B, topk=K, gate_hidden=h,
                                    dtype=torch.bfloat16)
    idx, _ = sas.prefill_selection(prob, g["q_nope"], g["k_nope"], g["wq"], g["qnorm_w"], g["wk"],
                                   g["knorm_w"])
    pooled = sas.sas_pool_keys(prob, g["k_nope"])
    idx_np = idx.cpu().numpy()
    valid = idx_np >= 0
    rng = np.random.default_rng(3)
    dl = rng.standard_normal(idx_np.shape) * valid
    dl -= valid * (dl.sum(axis=2, keepdims=True) / np.maximum(valid.sum(axis=2, keepdims=True), 1))
    dlogg = torch.from_numpy(dl.astype(np.float32)).to(dev)
    dwq, dqn, dwk, dkn = sas.sas_gate_bwd(prob, g["q_nope"], g["k_nope"], pooled, g["wq"],
                                          g["qnorm_w"], g["wk"], g["knorm_w"], idx, dlogg)
    torch.cuda.synchronize()
    ref = orc.gate_backward(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                            inp["knorm_w"], idx_np, dlogg.cpu().numpy().astype(np.float64),
                            np.asarray(shape.cu_seqlens), B, 1e-6, 1e6)
    for gpu, key in ((dwq, "dwq"), (dqn, "dqnorm_w"), (dwk, "dwk"), (dkn, "dknorm_w")):
        e = rel_l2(gpu, ref[key])
        assert np.isfinite(to64(gpu)).all(), key
        assert e <= 2e-3, f"{key}: rel-L2 {e:.3e}"


SELECT_CASES = {
    # fused path, 64-token tiles (NBmax <= 512), ragged sequences, G 4 and 5
    "bf16-d128-B64-ragged": ([300, 64, 1, 130], 8, 2, 128, 64, 3, 128, "bf16"),
    "bf16-d128-B64-G5": ([513, 77, 4100], 10, 2, 128, 64, 31, 128, "bf16"),
    # fused path, 32-token tiles (512 < NBmax <= 1024), K 63 as the 14B varlen workload
    "bf16-G5-K63-40k": ([40000, 333], 10, 2, 128, 64, 63, 128, "bf16"),
    # shapes outside the fused kernel: the unfused kernels through the workspace
    "bf16-d64-B32": ([257, 33], 8, 4, 64, 32, 5, 64, "bf16"),
    "fp32-d64-B16-tiny-shape": ([1024], 2, 1, 64, 16, 4, 32, "fp32"),
}


@pytest.mark.parametrize("name", list(SELECT_CASES))
def test_gate_select_fused(sas, name):
    """sas_gate_select (scores + Top-K in one pass, scores kept on chip) against the unfused
    sas_gate_scores + sas_topk on the GPU (ids bit-identical, log-gates and logsumexp to fp32
    rounding) and against the oracle on window/block/sequence edges and random rows."""
    lengths, Hq, Hkv, d, B, K, h, dt = SELECT_CASES[name]
    shape = si.Shape(list(lengths), Hq, Hkv, d, B, K, h, dt, seed=700)
    inp = si.prefill_inputs(shape)
    dev = torch.device("cuda:0")
    g = {k: v.to(dev) for k, v in inp.items()}
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=Hq, num_kv_heads=Hkv,
                                    head_dim=d, block=B, topk=K, gate_hidden=h,
                                    dtype=shape.torch_dtype)
    pooled = sas.sas_pool_keys(prob, g["k_nope"])
    gk = sas.sas_gate_keys(prob, pooled, g["wk"], g["knorm_w"])
    ws = sas.gate_select_workspace(prob)
    idx, logg, lse = sas.sas_gate_select(prob, g["q_nope"], g["k_nope"], gk, g["wq"], g["qnorm_w"],
                                         g["wk"], g["knorm_w"], workspace=ws, want_lse=True)
    scores, lse_u = sas.sas_gate_scores(prob, g["q_nope"], g["k_nope"], gk, g["wq"], g["qnorm_w"],
                                        g["wk"], g["knorm_w"])
    idx_u, logg_u = sas.sas_topk(prob, scores, lse_u)
    torch.cuda.synchronize()
    assert sas.error_code(ws) == 0
    assert_paths_agree(idx.cpu().numpy(), idx_u.cpu().numpy(), scores.cpu(), K)
    same = torch.from_numpy((idx.cpu().numpy() == idx_u.cpu().numpy()).all(axis=-1))
    assert (logg - logg_u).abs()[same.to(logg.device)].max().item() <= PATHS_GATE_ABS
    assert (lse - lse_u).abs().max().item() <= PATHS_GATE_ABS
    rng = np.random.default_rng(701)
    rows = set()
    for s0, s1 in zip(shape.cu_seqlens[:-1], shape.cu_seqlens[1:]):
        L = int(s1 - s0)
        for t in (0, 63, 64, 2047, 4095, 4096, 32767, 32768, L - 1):
            if 0 <= t < L:
                rows.add(int(s0) + t)
    rows |= set(rng.choice(shape.total_tokens, 60, replace=False).tolist())
    rows = np.array(sorted(rows))
    ref = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, B, K, 1e-6, 1e6, rows)
    compare_selection(idx.cpu().numpy()[rows], logg.cpu().numpy()[rows], ref["idx"], ref["logg"],
                      ref["margin"])
    assert np.abs(to64(lse)[rows] - ref["lse"]).max() <= GATE_ABS


def _paged_from_contiguous(inp, shp, seed, spare=17):
    """Scatter contiguous decode caches into shuffled pages of one block each (plus unused
    pages full of large values that must never be read)."""
    NB = shp.capacity // shp.block
    nb = shp.batch
    n_pages = nb * NB + spare
    perm = np.random.default_rng(seed).permutation(n_pages)
    pt = perm[:nb * NB].reshape(nb, NB).astype(np.int32)
    Hkv, d, h, B = shp.num_kv_heads, shp.head_dim, shp.gate_hidden, shp.block
    kp = torch.full((n_pages, Hkv, B, d), 300.0, dtype=inp["k_cache"].dtype)
    vp = torch.full((n_pages, Hkv, B, d), -300.0, dtype=inp["v_cache"].dtype)
    gp = torch.full((n_pages, Hkv, h), 300.0, dtype=torch.bfloat16)
    for b in range(nb):
        for j in range(NB):
            kp[pt[b, j]] = inp["k_cache"][b, :, j * B:(j + 1) * B]
            vp[pt[b, j]] = inp["v_cache"][b, :, j * B:(j + 1) * B]
            gp[pt[b, j]] = inp["gate_key_cache"][b, :, j]
    return torch.from_numpy(pt), n_pages, kp, vp, gp


PAGED_CASES = {
    "budget2048-K31": ([3000, 65, 1, 1777, 4096], 4096, 16, 4, 128, 64, 31, 128),
    "budget4096-K63-G5": ([6000, 4200, 130, 64], 8192, 20, 4, 128, 64, 63, 128),
    "batch32-mixed": (si.draw_lengths(42, 32, 1, 1024), 1024, 32, 8, 128, 64, 7, 128),
}


@pytest.mark.parametrize("name", list(PAGED_CASES))
def test_decode_paged_equals_contiguous(sas, name):
    """sas_decode_paged over shuffled one-block pages gives exactly sas_decode's results on the
    same cached values (same kernels, same numbers, same order), and a page id out of range
    is reported (code 62) with that sequence's output 0 and the others unchanged."""
    lengths, cap, Hq, Hkv, d, B, K, h = PAGED_CASES[name]
    shp = si.DecodeShape(list(lengths), cap, Hq, Hkv, d, B, K, h, seed=410)
    inp = si.decode_inputs(shp)
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=cap, num_q_heads=Hq, num_kv_heads=Hkv,
                             head_dim=d, block=B, topk=K, gate_hidden=h, dtype=torch.bfloat16)
    common = (g["cur_pool"], g["wq"], g["qnorm_w"], g["wk"], g["knorm_w"])
    o_c, i_c, l_c = sas.sas_decode(prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"],
                                   g["gate_key_cache"], *common, want_selection=True, check=True)
    pt, n_pages, kp, vp, gp = _paged_from_contiguous(inp, shp, 411)
    pt, kp, vp, gp = pt.cuda(), kp.cuda(), vp.cuda(), gp.cuda()
    o_p, i_p, l_p = sas.sas_decode_paged(prob, pt, n_pages, g["q"], g["q_nope"], kp, vp, gp, *common,
                                         want_selection=True, check=True)
    torch.cuda.synchronize()
    assert torch.equal(i_p, i_c)
    assert torch.equal(l_p, l_c)
    assert torch.equal(o_p, o_c)
    # a bad page id in sequence 0's history
    bad = pt.clone()
    bad[0, 0] = n_pages + 5   # block 0 is read by every sequence
    ws = sas._workspace(sas.lib_handle().sas_decode_workspace_size, prob.ref, prob.device)
    o_b = sas.sas_decode_paged(prob, bad, n_pages, g["q"], g["q_nope"], kp, vp, gp, *common,
                               workspace=ws)
    torch.cuda.synchronize()
    assert sas.error_code(ws) == 62
    assert torch.count_nonzero(o_b[0]).item() == 0
    assert torch.equal(o_b[1:], o_c[1:])


PER_HEAD_CASES = {
    # one gate per query head (gate_heads = Hq): tensor-core paths (gate projections, fused
    # selection, key-major attention with 128 single-head rows per tile, tensor-core decode)
    "bf16-d128-B64-G4": ([4200, 300, 65], 8, 2, 128, 64, 15, 128, "bf16"),
    # CUDA-core paths (fp32, d 64)
    "fp32-d64-B16-G2": ([300, 77], 4, 2, 64, 16, 5, 32, "fp32"),
}


def _per_head(sas, name, seed):
    lengths, Hq, Hkv, d, B, K, h, dt = PER_HEAD_CASES[name]
    shape = si.Shape(list(lengths), Hq, Hkv, d, B, K, h, dt, seed=seed, gate_heads=Hq)
    inp = si.prefill_inputs(shape, with_dout=True)
    dev = torch.device("cuda:0")
    g = {k: v.to(dev) for k, v in inp.items()}
    prob = sas.Problem.from_lengths(shape.lengths, dev, num_q_heads=Hq, num_kv_heads=Hkv,
                                    head_dim=d, block=B, topk=K, gate_hidden=h,
                                    dtype=shape.torch_dtype, gate_heads=Hq)
    return shape, inp, g, prob


def _edge_rows(shape, n_random, seed):
    rows = set()
    for s0, s1 in zip(shape.cu_seqlens[:-1], shape.cu_seqlens[1:]):
        L = int(s1 - s0)
        for t in (0, 15, 16, 63, 64, 4095, 4096, L - 1):
            if 0 <= t < L:
                rows.add(int(s0) + t)
    rng = np.random.default_rng(seed)
    rows |= set(rng.choice(shape.total_tokens, n_random, replace=False).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", list(PER_HEAD_CASES))
def test_per_head_gate_selection(sas, name):
    """One gate per query head: the fused and the unfused selection agree bit for bit, and
    match the oracle (per-query-head Qproj, scored against the KV head's block keys)."""
    shape, inp, g, prob = _per_head(sas, name, 800)
    idx, logg = sas.prefill_selection(prob, g["q_nope"], g["k_nope"], g["wq"], g["qnorm_w"],
                                      g["wk"], g["knorm_w"])
    idx_u, logg_u = sas.prefill_selection(prob, g["q_nope"], g["k_nope"], g["wq"], g["qnorm_w"],
                                          g["wk"], g["knorm_w"], fused=False)
    torch.cuda.synchronize()
    assert idx.shape == (shape.total_tokens, shape.num_q_heads, shape.topk + 1)
    assert torch.equal(idx, idx_u)
    assert (logg - logg_u).abs().max().item() <= PATHS_GATE_ABS
    rows = _edge_rows(shape, 60, 801)
    ref = orc.prefill_selection(inp["q_nope"], inp["k_nope"], inp["wq"], inp["qnorm_w"], inp["wk"],
                                inp["knorm_w"], shape.cu_seqlens, shape.block, shape.topk, 1e-6,
                                1e6, rows)
    compare_selection(idx.cpu().numpy()[rows], logg.cpu().numpy()[rows], ref["idx"], ref["logg"],
                      ref["margin"])


@pytest.mark.parametrize("name", list(PER_HEAD_CASES))
def test_per_head_attention(sas, name):
    """Every query head on its own selection: forward rows, dQ / dlogg rows and dK / dV of
    first, middle and last blocks against the oracle."""
    shape, inp, g, prob = _per_head(sas, name, 810)
    idx, logg = si.random_selection(shape)
    ti, tl = torch.from_numpy(idx).cuda(), torch.from_numpy(logg).cuda()
    wsf, wsb = sas.attn_fwd_workspace(prob), sas.attn_bwd_workspace(prob)
    o, lse = sas.sas_attn_fwd(prob, g["q"], g["k"], g["v"], ti, tl, workspace=wsf)
    dq, dk, dv, dl = sas.sas_attn_bwd(prob, g["q"], g["k"], g["v"], o, g["dout"], lse, ti, tl,
                                      workspace=wsb)
    torch.cuda.synchronize()
    assert sas.error_code(wsf) == 0 and sas.error_code(wsb) == 0
    fp32 = shape.dtype == "fp32"
    cu = shape.cu_seqlens
    rows = _edge_rows(shape, 40, 811)
    O, LSE, _ = orc.attention_fwd(inp["q"], inp["k"], inp["v"], idx, logg, cu, shape.block,
                                  rows=rows)
    assert_out_close(o[torch.from_numpy(rows).cuda()], O, fp32, "O")
    assert np.abs(to64(lse)[rows] - LSE).max() <= (1e-4 if fp32 else 2e-3)
    dq_r, dl_r = orc.attention_bwd_rows(inp["q"], inp["k"], inp["v"], inp["dout"], idx, logg, cu,
                                        shape.block, rows)
    assert_grad_close(dq.cpu()[rows], dq_r, fp32, "dQ rows")
    assert_grad_close(dl.cpu()[rows], dl_r, fp32, "dlogg rows")
    assert (to64(dl)[idx < 0] == 0).all()
    B = shape.block
    for b, (s0, s1) in enumerate(zip(cu[:-1], cu[1:])):
        L = int(s1 - s0)
        nb = (L + B - 1) // B
        for j, kv in sorted({(0, 0), (nb // 2, shape.num_kv_heads - 1), (nb - 1, 0)}):
            lo, hi = j * B, min((j + 1) * B, L)
            dk_r, dv_r = orc.attention_bwd_keys(inp["q"], inp["k"], inp["v"], inp["dout"], idx,
                                                logg, cu, B, b, kv, lo, hi)
            if np.linalg.norm(dk_r) > 1e-9:
                assert_grad_close(dk.cpu()[int(s0) + lo:int(s0) + hi, kv], dk_r, fp32,
                                  f"dK seq {b} block {j}")
            assert_grad_close(dv.cpu()[int(s0) + lo:int(s0) + hi, kv], dv_r, fp32,
                              f"dV seq {b} block {j}")


@pytest.mark.parametrize("d,B,h,dt", [(128, 64, 128, "bf16"), (64, 16, 32, "bf16")])
def test_per_head_decode(sas, d, B, h, dt):
    """Decode with one gate per query head against the oracle (selection per query head)."""
    shp = si.DecodeShape([3000, 65, 1, 1777], 4096, 8, 2, d, B, 15, h, seed=820, dtype=dt,
                         gate_heads=8)
    inp = si.decode_inputs(shp)
    g = {k: v.cuda() for k, v in inp.items()}
    prob = sas.DecodeProblem(seqlens=g["lengths"], capacity=shp.capacity, num_q_heads=8,
                             num_kv_heads=2, head_dim=d, block=B, topk=15, gate_hidden=h,
                             dtype=torch.bfloat16, gate_heads=8)
    o, idx, logg = sas.sas_decode(prob, g["q"], g["q_nope"], g["k_cache"], g["v_cache"],
                                  g["gate_key_cache"], g["cur_pool"], g["wq"], g["qnorm_w"], g["wk"],
                                  g["knorm_w"], want_selection=True, check=True)
    torch.cuda.synchronize()
    assert idx.shape == (4, 8, 16)
    O, ridx, rlogg, margin = orc.decode(inp["q"], inp["q_nope"], inp["k_cache"], inp["v_cache"],
                                        shp.lengths, inp["gate_key_cache"], inp["cur_pool"],
                                        inp["wq"], inp["qnorm_w"], inp["wk"], inp["knorm_w"], B, 15,
                                        1e-6, 1e6, selection=(idx.cpu().numpy(), logg.cpu().numpy()))
    compare_selection(idx.cpu().numpy(), logg, ridx, rlogg, margin)
    assert_out_close(o, O, False, "O")
