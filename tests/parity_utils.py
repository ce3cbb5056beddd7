"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used by every parity test):
  * Top-K block ids: identical, except rows whose exact margin between the K-th and
    (K+1)-th historical score is below 1e-5 (near-ties, counted and reported).
  * bf16 outputs: max |diff| <= 2e-2 and mean |diff| <= 2e-3.
  * gradients: relative L2 error <= 5e-2.
  * fp32 inputs (CUDA-core path, fp32 arithmetic): max |diff| <= 1e-4, gradient
    relative L2 <= 1e-4.
  * fp32 gate quantities (scores, lse, log-gates): |diff| <= 5e-5 (fp32 accumulation of
    O(1) values over <= 1024 terms; the fp64 oracle is exact by comparison).
"""
import numpy as np
import torch

NEAR_TIE = 1e-5
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
GRAD_REL_L2 = 5e-2
FP32_MAX_ABS, FP32_GRAD_REL_L2 = 1e-4, 1e-4
GATE_ABS = 5e-5


def to64(t):
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            t = t.float()
        return t.numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def assert_out_close(gpu, ref, fp32: bool, what: str):
    a, b = to64(gpu), to64(ref)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    d = np.abs(a - b)
    assert np.isfinite(a).all(), f"{what}: non-finite GPU values"
    if fp32:
        assert d.max() <= FP32_MAX_ABS, f"{what}: max|diff| {d.max():.3e}"
    else:
        assert d.max() <= BF16_MAX_ABS, f"{what}: max|diff| {d.max():.3e}"
        assert d.mean() <= BF16_MEAN_ABS, f"{what}: mean|diff| {d.mean():.3e}"
    return float(d.max()), float(d.mean())


def rel_l2(gpu, ref) -> float:
    a, b = to64(gpu), to64(ref)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_grad_close(gpu, ref, fp32: bool, what: str):
    e = rel_l2(gpu, ref)
    assert np.isfinite(to64(gpu)).all(), f"{what}: non-finite GPU values"
    assert e <= (FP32_GRAD_REL_L2 if fp32 else GRAD_REL_L2), f"{what}: rel-L2 {e:.3e}"
    return e


# Two GPU selection paths (fused scores + Top-K against the separate kernels): the historical
# scores come from different arithmetic (tf32 hi/lo products on the tensor cores, fp32 FMA on
# the CUDA cores), each within GATE_ABS of the oracle, so their log-gates and logsumexps agree
# to a few fp32 roundings of the row's score range; 2e-5 bounds that with room.
PATHS_GATE_ABS = 2e-5


def assert_paths_agree(idx_a, idx_b, scores, K):
    """Selections of two GPU paths: identical ids except at rows whose K-th and (K+1)-th largest
    historical scores (from `scores` [T, Hs, NBmax], the unfused path's) are a near-tie, where
    both selections are correct. Returns the number of such rows."""
    a, b = np.asarray(idx_a), np.asarray(idx_b)
    diff = ~(a == b).all(axis=-1)
    if not diff.any():
        return 0
    s = to64(scores)
    for r, h in np.argwhere(diff):
        c = int(a[r, h, K])   # the current block, always in the last slot when c > K
        row = np.sort(s[r, h, :c])[::-1]
        assert c > K and row[K - 1] - row[K] < NEAR_TIE, \
            f"row {r} head {h}: selections differ with margin {row[K - 1] - row[K]:.3e}"
    return int(diff.sum())


def compare_selection(idx_gpu, logg_gpu, idx_ref, logg_ref, margin_ref):
    """Top-K parity: exact ids except near-ties; log-gates within GATE_ABS where ids agree.
    Returns (n_rows, n_near_tie, n_mismatch_near_tie)."""
    ig, ir = np.asarray(idx_gpu), np.asarray(idx_ref)
    lg, lr = to64(logg_gpu), to64(logg_ref)
    margin = np.asarray(margin_ref)
    same = (ig == ir).all(axis=-1)
    near = margin < NEAR_TIE
    bad = ~same & ~near
    assert not bad.any(), f"{int(bad.sum())} Top-K rows differ with margin >= {NEAR_TIE}: " \
        f"first at {np.argwhere(bad)[0]}"
    valid = same[..., None] & (ir >= 0)
    if valid.any():
        err = np.abs(lg - lr)[valid].max()
        assert err <= GATE_ABS, f"log-gate max|diff| {err:.3e}"
    assert (lg[ig < 0] == 0).all()
    return int(same.size), int(near.sum()), int((~same & near).sum())
