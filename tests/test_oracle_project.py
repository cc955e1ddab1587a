"""Pins of oracle/project.py (the projection the quantize-on-write path codes)."""
import numpy as np
import torch

from oracle import project


def test_bf16_round_ties_and_neighbours():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7
    v = np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, -(1 + 2.0**-8), 3.0, 1 + 2.0**-8 + 2.0**-20, 0.0, 2.0**-130])
    want = np.array([1.0, 1 + 2.0**-6, -1.0, 3.0, 1 + 2.0**-7, 0.0, 2.0**-130])
    assert np.array_equal(project.bf16_round(v), want)


def test_bf16_round_matches_library_conversion():
    # float32 -> bfloat16 in torch rounds to nearest even: the same rule on float32 inputs
    r = np.random.default_rng(5)
    f = (r.standard_normal(20000) * np.exp(r.normal(0, 4, 20000))).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(project.bf16_round(f.astype(np.float64)), ref)


def test_projection_picks_weight_columns_and_orders_heads():
    # x rows are unit vectors e_i: head h, token t must give column i_t of head h's weight rows
    hidden, n_heads, d = 16, 2, 128
    r = np.random.default_rng(1)
    w = torch.from_numpy(r.standard_normal((n_heads * d, hidden)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    idx = [3, 0, 15]
    x = np.zeros((3, hidden), dtype=np.float32)
    x[np.arange(3), idx] = 1.0
    k = project.project(x, w, n_heads)
    for h in range(n_heads):
        for t, i in enumerate(idx):
            assert np.array_equal(k[h * 3 + t], w[h * d:(h + 1) * d, i])


def test_projection_rounds_the_exact_sum_once():
    # 1 + 2^-8 + 2^-9 (exact in float64) rounds up to 1 + 2^-7; rounding 1 + 2^-8 first would tie to 1
    x = np.array([[1.0, 2.0**-8, 2.0**-9]], dtype=np.float32)
    w = np.zeros((128, 3), dtype=np.float32)
    w[5] = 1.0
    k = project.project(x, w, 1)
    assert k[0, 5] == 1 + 2.0**-7
    assert np.all(np.delete(k[0], 5) == 0.0)


def test_tie_flags():
    s = np.array([1 + 2.0**-8, 1 + 2.0**-8 + 1e-3, 1.0])
    a = np.array([1.0, 1.0, 1.0])
    f = project.bf16_tie_flags(s, a, rel=2e-5)
    assert f.tolist() == [True, False, False]
