"""The seeded generator: numpy and torch paths agree bit for bit; slices equal the full draw."""
import numpy as np
import torch

import sas_inputs as si


def test_numpy_and_torch_paths_identical():
    for start in (0, 12345, (1 << 32) - 7, 3 * (1 << 32) + 11):
        a = si.normal_np(3, 7, start, 5000)
        b = si.normal_torch(3, 7, start, 5000, "cpu").numpy()
        assert a.dtype == np.float32
        np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))


def test_moments_and_independence():
    x = si.normal_np(1, 1, 0, 1 << 20).astype(np.float64)
    assert abs(x.mean()) < 5e-3 and abs(x.var() - 1) < 5e-3
    y = si.normal_np(1, 2, 0, 1 << 20).astype(np.float64)
    assert abs(np.corrcoef(x, y)[0, 1]) < 5e-3
    assert abs(np.corrcoef(x[:-1], x[1:])[0, 1]) < 5e-3


def test_slices_and_rounding():
    full = si.draw(9, "k_cache", (4, 3, 40, 8), dtype=torch.bfloat16)
    part = si.draw(9, "k_cache", (3, 40, 8), dtype=torch.bfloat16, offset=2 * 3 * 40 * 8)
    assert torch.equal(full[2], part)
    small = si.draw(9, "k_cache", (4, 3, 40, 8), dtype=torch.bfloat16, chunk=1000)
    assert torch.equal(full, small)


def test_decode_rows_match_full_draw():
    shp = si.DecodeShape([40, 70, 33], 128, 4, 2, 8, 16, 2, 8, seed=5)
    full = si.decode_inputs(shp)
    part = si.decode_inputs(shp, batch_rows=[2])
    for k in ("q", "q_nope", "k_cache", "v_cache", "gate_key_cache", "cur_pool", "lengths"):
        assert torch.equal(full[k][2:3], part[k]), k


def test_random_selection_structure():
    shp = si.Shape([200, 77], 4, 2, 8, 16, 4, 8, "bf16", seed=2)
    idx, logg = si.random_selection(shp)
    pos = shp.positions()
    for n in range(len(pos)):
        c = pos[n] // 16
        for kv in range(2):
            row = idx[n, kv]
            k = min(4, c)
            assert list(row[k + 1:]) == [-1] * (4 - k)
            assert row[k] == c
            assert len(set(row[:k])) == k and all(0 <= j < c for j in row[:k])
            assert list(row[:k]) == sorted(row[:k])
    assert (logg[idx >= 0] <= -1).all() and (logg[idx < 0] == 0).all()


def test_sequence_draw_matches_packed_draw():
    shp = si.Shape([40, 70, 33], 4, 2, 8, 16, 2, 8, "bf16", seed=6)
    full = si.prefill_inputs(shp, with_dout=True)
    one = si.prefill_inputs(shp, with_dout=True, sequence=1)
    for k in ("q_nope", "k_nope", "q", "k", "v", "dout"):
        assert torch.equal(full[k][40:110], one[k]), k
    for k in ("wq", "wk", "qnorm_w", "knorm_w"):
        assert torch.equal(full[k], one[k]), k
    assert one["cu_seqlens"].tolist() == [0, 70]
    assert si.sequence_shape(shp, 1).lengths == [70]
