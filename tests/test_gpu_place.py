"""Expert placement (embeddings, K-Means biclustering, greedy 2D placement) on
the GPU against the fp64 oracle: ideal coordinates, grid_assign and the
iteration counts must be identical."""
import numpy as np
import pytest

import synth
from oracle import placement as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import os
    from tiled_rank_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from tiled_rank_b200 import build
        build.build()
    return torch


def run_place(torch, u, v, M, N, max_iter=100):
    from tiled_rank_b200 import _lib as L
    dev = torch.device("cuda:0")
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(dev)
    vd = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(dev)
    pin = L.place_in(ud, vd, M, N, max_iter)
    ws = torch.empty(L.tileq_place_workspace_size(pin), dtype=torch.uint8, device=dev)
    K = u.shape[0]
    grid = torch.full((K,), -1, dtype=torch.int32, device=dev)
    ideal = torch.full((K, 2), -1, dtype=torch.int32, device=dev)
    its = torch.zeros(2, dtype=torch.int32, device=dev)
    L.tileq_place_experts(pin, grid, ws, ideal, its)
    torch.cuda.synchronize()
    return grid.cpu().numpy(), ideal.cpu().numpy(), tuple(its.cpu().numpy().tolist())


def check(torch, u, v, M, N, max_iter=100, what=""):
    lm, ln, g, its = P.place_experts(u, v, M, N, max_iter)
    gg, gi, gits = run_place(torch, u, v, M, N, max_iter)
    assert np.array_equal(gi[:, 0], lm), f"{what}: row clusters"
    assert np.array_equal(gi[:, 1], ln), f"{what}: column clusters"
    assert np.array_equal(gg, g), f"{what}: grid_assign"
    assert gits == tuple(its), f"{what}: iterations {gits} vs {its}"
    return gg


# planted grids at the layers' shapes (left factor: d_ff rows, right: d_model rows), r0 = 16
@pytest.mark.parametrize("K,M,N,d_u,d_v,r0", [
    (8, 2, 4, 14336, 4096, 16),     # Mixtral-shaped, 8 experts on 2 x 4
    (60, 6, 10, 1408, 2048, 16),    # Qwen1.5-MoE-shaped, 60 experts on 6 x 10
    (64, 8, 8, 1536, 4096, 16),     # 64 experts on 8 x 8
])
def test_planted_full_shapes(torch_cuda, K, M, N, d_u, d_v, r0):
    u, v, cells = synth.planted_factors(K, M, N, d_u, d_v, r0, noise=0.1, seed=K)
    g = check(torch_cuda, u, v, M, N, what=f"planted {K}")
    assert len(set(g.tolist())) == K


@pytest.mark.parametrize("K,M,N,d_u,d_v,r0,seed", [
    (64, 8, 8, 96, 80, 4, 1),       # unstructured, high-dimensional: conflicts
    (60, 6, 10, 37, 53, 3, 2),      # ragged flattened lengths (111, 159: not multiples of 64)
    (33, 4, 9, 40, 24, 7, 3),       # K not a multiple of 4 (partial 4 x 4 Gram blocks)
    (5, 3, 3, 20, 30, 2, 4),        # fewer experts than cells
    (2, 4, 1, 16, 16, 5, 5),        # more grid rows than experts: min(M, K) clusters
    (1, 1, 1, 8, 8, 1, 6),          # one expert
    (12, 3, 4, 4, 2, 256, 7),       # the widest r0
    (16, 4, 4, 300, 200, 1, 8),     # r0 = 1
    # low-dimensional embeddings: several Lloyd updates before the assignment settles
    (64, 8, 8, 1, 1, 3, 9),
    (60, 6, 10, 2, 1, 2, 10),
])
def test_random_factors(torch_cuda, K, M, N, d_u, d_v, r0, seed):
    rng = np.random.default_rng([seed, 11])
    u = rng.standard_normal((K, d_u, r0)).astype(np.float32)
    v = rng.standard_normal((K, d_v, r0)).astype(np.float32)
    check(torch_cuda, u, v, M, N, what=f"random {K}x{M}x{N}")


def test_degenerate_factors(torch_cuda):
    """Sign ties (+a and -a in one column) and duplicate experts."""
    rng = np.random.default_rng(21)
    K, M, N, d, r0 = 12, 3, 4, 24, 4
    u = rng.standard_normal((K, d, r0)).astype(np.float32)
    v = rng.standard_normal((K, d, r0)).astype(np.float32)
    u[0, 3, 1], u[0, 7, 1] = -9.0, 9.0           # the first row decides: flip
    v[2, 0, 0], v[2, 5, 0] = 8.0, -8.0           # the first row decides: keep
    u[6] = u[5]                                  # duplicates: equal distances to everything
    v[6] = -v[5]                                 # the same embedding after the sign fix
    check(torch_cuda, u, v, M, N, what="degenerate")


def test_zero_factor(torch_cuda):
    """A zero factor embeds as the zero vector, at distance |c|^2 = 1 from every
    single-expert centre: the first assignment is an exact tie that rounding
    decides, so several results are correct.  Checked instead: the labels are a
    K-Means fixed point (each expert at a nearest centre, within rounding, of
    the means of the labelled experts) and grid_assign is the greedy placement
    of the returned ideal coordinates."""
    u, v, _ = synth.planted_factors(24, 4, 6, 64, 48, 4, noise=0.3, seed=41)
    u[7] = 0.0
    v[7] = 0.0
    g, ideal, _ = run_place(torch_cuda, u, v, 4, 6)
    for side, f, C in ((0, u, 4), (1, v, 6)):
        E = np.stack([P.embed(f[k]) for k in range(24)])
        lab = ideal[:, side]
        assert lab.min() >= 0 and lab.max() < C
        cen = np.stack([E[lab == j].mean(axis=0) for j in range(C) if np.any(lab == j)])
        used = [j for j in range(C) if np.any(lab == j)]
        d = ((E[:, None, :] - cen[None, :, :]) ** 2).sum(-1)
        mine = d[np.arange(24), [used.index(j) for j in lab]]
        assert np.all(mine <= d.min(axis=1) + 1e-9)
    assert np.array_equal(g, P.greedy_place(ideal[:, 0], ideal[:, 1], 4, 6))


def test_iteration_cap(torch_cuda):
    rng = np.random.default_rng(31)
    u = rng.standard_normal((64, 1, 3)).astype(np.float32)   # points on the sphere: 5 and 3 updates
    v = rng.standard_normal((64, 1, 3)).astype(np.float32)
    for cap in (1, 2):
        _, _, its = run_place(torch_cuda, u, v, 8, 8, cap)
        assert its == (cap, cap)
        check(torch_cuda, u, v, 8, 8, cap, what=f"cap {cap}")
