"""Pins of the expert-placement oracle (TileQ technical summary, section 2.1,
steps 2-4: embeddings, K-Means biclustering, greedy 2D placement)."""
import itertools

import numpy as np
import pytest

import synth
from oracle import placement as P


def test_embed_hand_case_and_sign_invariance():
    f = np.array([[1.0, -3.0], [-2.0, 1.0], [2.0, 3.0]])
    # column 0: |-2| and |2| tie -> the first (row 1, negative) decides: flip
    # column 1: |-3| and |3| tie -> row 0 (negative): flip
    want = np.array([-1.0, 3.0, 2.0, -1.0, -2.0, -3.0]) / np.sqrt(28.0)
    np.testing.assert_allclose(P.embed(f), want, rtol=1e-15)
    rng = np.random.default_rng(0)
    g = rng.standard_normal((50, 6))
    e = P.embed(g)
    assert abs(np.linalg.norm(e) - 1.0) < 1e-14
    for flips in itertools.product([-1.0, 1.0], repeat=3):
        s = np.ones(6)
        s[[0, 2, 5]] = flips
        np.testing.assert_array_equal(P.embed(g * s[None, :]), e)
    assert np.array_equal(P.embed(np.zeros((4, 2))), np.zeros(8))


def test_farthest_first_hand_case():
    E = np.array([[0.0], [1.0], [10.0], [11.0], [5.0]])
    # 0 -> farthest is 11 (index 3); then min distances: 1, 1, 10^2 vs 1^2 ... -> 5 (index 4, d=25)
    assert P.farthest_first(E, 3) == [0, 3, 4]
    # a tie: points 1 and 2 are both 1 away from their nearest centre -> the lower index
    assert P.farthest_first(np.array([[0.0], [1.0], [3.0], [4.0]]), 3) == [0, 3, 1]


def test_kmeans_hand_case():
    E = np.array([[0.0, 0.0], [0.0, 1.0], [10.0, 0.0], [10.0, 1.0], [0.0, 0.4]])
    lab, cen, it = P.kmeans(E, 2, 50)
    assert list(lab) == [0, 0, 1, 1, 0]
    np.testing.assert_allclose(cen, [[0.0, 1.4 / 3.0], [10.0, 0.5]], rtol=1e-15)
    assert it == 1
    # an exact tie in the assignment: the centres start at 0 and 4 (farthest
    # first), and 2 is 4 away (squared) from both -> the lower centre; the
    # centres then move to 1 and 4 and no label changes
    lab, cen, it = P.kmeans(np.array([[0.0], [4.0], [2.0]]), 2, 50)
    assert list(lab) == [0, 1, 0]
    np.testing.assert_array_equal(cen, [[1.0], [4.0]])
    assert it == 1


@pytest.mark.parametrize("P_,D,C,seed", [(30, 5, 4, 1), (64, 40, 8, 2), (60, 17, 6, 3), (9, 3, 9, 4)])
def test_kmeans_matches_sklearn_lloyd(P_, D, C, seed):
    """scikit-learn's Lloyd iterations from the same initial centres give the
    same labels; and the result is a fixed point of the algorithm."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(seed)
    E = rng.standard_normal((P_, D))
    lab, cen, it = P.kmeans(E, C, 300)
    init = E[P.farthest_first(E, C)]
    km = KMeans(n_clusters=C, init=init, n_init=1, max_iter=300, tol=0.0, algorithm="lloyd").fit(E)
    assert np.array_equal(lab, km.labels_)
    d = ((E[:, None, :] - cen[None, :, :]) ** 2).sum(-1)
    assert np.array_equal(lab, d.argmin(axis=1))
    for j in range(C):
        if np.any(lab == j):
            np.testing.assert_allclose(cen[j], E[lab == j].mean(axis=0), rtol=1e-12, atol=1e-15)


def test_kmeans_iteration_cap():
    rng = np.random.default_rng(7)
    E = rng.standard_normal((200, 4))
    lab1, _, it1 = P.kmeans(E, 8, 1)
    assert it1 == 1
    lab, _, it = P.kmeans(E, 8, 1000)
    assert it > 1


def test_greedy_place_hand_cases():
    # no conflict: every expert gets its ideal cell
    g = P.greedy_place([0, 1, 1, 0], [1, 0, 1, 0], 2, 2)
    assert list(g) == [1, 2, 3, 0]
    # experts 0, 1, 2 all want (0, 0) on a 2x2 grid; 3 wants (1, 1)
    # distance 0: (0,(0,0)) and (3,(1,1)); distance 1: expert 1 -> cell 1, expert 2 -> cell 2
    g = P.greedy_place([0, 0, 0, 1], [0, 0, 0, 1], 2, 2)
    assert list(g) == [0, 1, 2, 3]
    # 1x3 grid, all three want the middle: 0 takes it, 1 takes the left (lower cell), 2 the right
    g = P.greedy_place([0, 0, 0], [1, 1, 1], 1, 3)
    assert list(g) == [1, 0, 2]
    # 3x3 grid, two experts want the corner (0, 0): the second goes to (0, 1), not (1, 1)
    g = P.greedy_place([0, 0, 2], [0, 0, 2], 3, 3)
    assert list(g) == [0, 1, 8]


@pytest.mark.parametrize("K,M,N,seed", [(8, 2, 4, 0), (60, 6, 10, 1), (64, 8, 8, 2), (5, 3, 3, 3)])
def test_greedy_place_properties(K, M, N, seed):
    from scipy.optimize import linear_sum_assignment
    rng = np.random.default_rng(seed)
    im, inn = rng.integers(0, M, K), rng.integers(0, N, K)
    g = P.greedy_place(im, inn, M, N)
    assert len(set(g.tolist())) == K and g.min() >= 0 and g.max() < M * N
    wants = {}
    for k in range(K):
        wants.setdefault((im[k], inn[k]), []).append(k)
    for (m, n), ks in wants.items():
        assert g[ks[0]] == m * N + n            # the lowest index of the experts that want a cell gets it
    cost = np.array([[(c // N - im[k]) ** 2 + (c % N - inn[k]) ** 2 for c in range(M * N)] for k in range(K)])
    r, c = linear_sum_assignment(cost)
    assert cost[np.arange(K), g].sum() >= cost[r, c].sum()
    # without conflicts greedy is optimal (zero)
    cells = rng.permutation(M * N)[:K]
    g2 = P.greedy_place(cells // N, cells % N, M, N)
    assert np.array_equal(g2, cells)


def _same_partition(a, b):
    """a and b label the same partition (up to renaming the labels)."""
    return all((a[i] == a[j]) == (b[i] == b[j]) for i in range(len(a)) for j in range(len(a)))


@pytest.mark.parametrize("K,M,N,d_u,d_v,r0", [(8, 2, 4, 96, 64, 8), (24, 4, 6, 64, 80, 4),
                                              (16, 4, 4, 128, 128, 16)])
def test_place_experts_recovers_planted_grid(K, M, N, d_u, d_v, r0):
    u, v, cells = synth.planted_factors(K, M, N, d_u, d_v, r0, noise=0.05, seed=K)
    lm, ln, g, its = P.place_experts(u, v, M, N)
    assert _same_partition(lm, cells // N) and _same_partition(ln, cells % N)
    # a full grid of distinct (row, column) clusters: every expert gets its ideal cell
    assert np.array_equal(g, lm * N + ln)
    assert all(1 <= i <= 100 for i in its)


def _greedy_rounds(im, inn, M, N):
    """The greedy order restated as the GPU runs it: first every distance-0
    pair whose expert is the lowest index wanting that cell, then one round
    per remaining expert, each placing the smallest (distance, expert, cell)
    key over the unplaced experts' best free cells."""
    K = len(im)
    grid = [-1] * K
    free = [True] * (M * N)
    for k in range(K):
        c = int(im[k]) * N + int(inn[k])
        if all(int(im[j]) * N + int(inn[j]) != c for j in range(k)):
            grid[k] = c
            free[c] = False
    while any(g < 0 for g in grid):
        best = None
        for k in range(K):
            if grid[k] >= 0:
                continue
            for c in range(M * N):
                if free[c]:
                    key = ((c // N - im[k]) ** 2 + (c % N - inn[k]) ** 2, k, c)
                    best = key if best is None or key < best else best
        _, k, c = best
        grid[k] = c
        free[c] = False
    return np.array(grid, dtype=np.int32)


@pytest.mark.parametrize("K,M,N,spread,seed", [(64, 8, 8, 3, 0), (60, 6, 10, 2, 1), (8, 2, 4, 1, 2),
                                               (33, 4, 9, 4, 3), (5, 3, 3, 1, 4), (64, 8, 8, 1, 5)])
def test_greedy_round_form_matches_sorted_scan(K, M, N, spread, seed):
    """Ideal coordinates crowded into a corner (many conflicts): the round-by-
    round form with the distance-0 head gives the sorted-scan result."""
    rng = np.random.default_rng(seed)
    im = rng.integers(0, min(M, spread), K)
    inn = rng.integers(0, min(N, spread), K)
    assert np.array_equal(_greedy_rounds(im, inn, M, N), P.greedy_place(im, inn, M, N))


def _kmeans_gram_form(E, C, max_iter):
    """Lloyd K-Means evaluated as the GPU does: only the normalised Gram
    matrix G of the embeddings, every centre as weights a_j over the points,
    |e_i - c_j|^2 = G_ii - 2 (G a_j)_i + a_j^T G a_j."""
    G = E @ E.T
    n = np.sqrt(np.diag(G))
    inv = np.where(n > 0, 1.0 / np.where(n > 0, n, 1.0), 0.0)
    G = G * inv[:, None] * inv[None, :]
    P_ = len(E)
    alpha = np.zeros((C, P_))
    mind = None
    p = 0
    for j in range(C):
        if j > 0:
            p = int(np.argmax(mind))
        alpha[j, p] = 1.0
        d = np.diag(G) - 2 * G[:, p] + G[p, p]
        mind = d if j == 0 else np.minimum(mind, d)

    def assign():
        H = alpha @ G                                   # [C, P]
        q = np.einsum("jp,jp->j", alpha, H)
        return np.argmin(np.diag(G)[:, None] - 2 * H.T + q[None, :], axis=1)

    labels = assign()
    it = 0
    while it < max_iter:
        for j in range(C):
            m = labels == j
            if m.any():
                alpha[j] = m / m.sum()
        it += 1
        new = assign()
        if np.array_equal(new, labels):
            break
        labels = new
    return labels, it


@pytest.mark.parametrize("P_,D,C,seed", [(64, 3, 8, 0), (60, 2, 6, 1), (64, 40, 8, 2), (33, 7, 4, 3)])
def test_kmeans_gram_form_matches_direct(P_, D, C, seed):
    rng = np.random.default_rng(seed)
    E = rng.standard_normal((P_, D))
    E /= np.linalg.norm(E, axis=1, keepdims=True)
    lab, _, it = P.kmeans(E, C, 100)
    lab2, it2 = _kmeans_gram_form(E, C, 100)
    assert np.array_equal(lab, lab2) and it == it2
