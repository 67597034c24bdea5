"""Pins of the fp64 oracle of the Gaussian-sketch global low-rank step (CPU)."""
import numpy as np
import pytest

from oracle import sketch


def _orth(rng, n, r):
    q, _ = np.linalg.qr(rng.standard_normal((n, r)))
    return q


def _to_bf16_bits(a):
    f = np.asarray(a, dtype=np.float32).view(np.uint32)
    return ((f + np.uint32(0x7FFF) + ((f >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def test_assemble_wbig_places_each_expert():
    M, N, d_out, d_in = 2, 3, 4, 5
    K = M * N
    grid = np.array([4, 0, 5, 2, 1, 3])
    # expert k holds the constant k+1 (exact in bf16)
    w = np.stack([np.full((d_out, d_in), k + 1.0, dtype=np.float32) for k in range(K)])
    big = sketch.assemble_wbig(_to_bf16_bits(w), grid, M, N)
    for k in range(K):
        m, n = divmod(int(grid[k]), N)
        blk = big[m * d_out:(m + 1) * d_out, n * d_in:(n + 1) * d_in]
        assert np.all(blk == k + 1.0)


@pytest.mark.parametrize("R,C,r,l", [(96, 80, 6, 6), (128, 64, 8, 14), (64, 200, 5, 12)])
def test_exact_recovery_of_rank_r(R, C, r, l):
    rng = np.random.default_rng(R * 7 + C)
    u0, v0 = _orth(rng, R, r), _orth(rng, C, r)
    s0 = np.sort(rng.uniform(0.5, 5.0, r))[::-1]
    w = (u0 * s0) @ v0.T
    omega = rng.standard_normal((C, l))
    u, s, v = sketch.sketch_lowrank(w, omega, r)
    np.testing.assert_allclose(s, s0, rtol=1e-10)
    np.testing.assert_allclose((u * s) @ v.T, w, atol=1e-10 * np.abs(w).max())
    np.testing.assert_allclose(u.T @ u, np.eye(r), atol=1e-10)
    np.testing.assert_allclose(v.T @ v, np.eye(r), atol=1e-10)
    # the factors span the planted subspaces
    np.testing.assert_allclose(np.abs(u0.T @ u), np.eye(r), atol=1e-8)


def test_full_rank_within_range_finder_bound():
    rng = np.random.default_rng(5)
    R, C, r, l = 120, 90, 10, 18
    n = min(R, C)
    s_all = 0.8 ** np.arange(n)
    w = (_orth(rng, R, n) * s_all) @ _orth(rng, C, n).T
    u, s, v = sketch.sketch_lowrank(w, rng.standard_normal((C, l)), r)
    err = np.linalg.norm(w - (u * s) @ v.T, 2)
    assert err <= sketch.range_finder_bound(s_all, r, l) + s_all[r]
    # and never better than the optimal rank-r error
    assert err >= s_all[r] * (1 - 1e-9)
    # the leading singular values are close to the true ones
    np.testing.assert_allclose(s[:3], s_all[:3], rtol=1e-3)


def test_sketch_rejects_too_narrow():
    with pytest.raises(ValueError):
        sketch.sketch_lowrank(np.eye(4), np.ones((4, 2)), 3)
