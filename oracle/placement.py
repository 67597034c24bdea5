"""fp64 oracle of TileQ's expert placement (test infrastructure only).

TileQ technical summary, section 2.1 "2D-Tiling Structured Low-Rank
Quantization", steps 2-4: each expert's rank-r0 SVD factors (U_k, V_k),
flattened and scaled to unit norm, are its feature embeddings; K-Means on the
U side and on the V side picks a preferred cell (m, n) of the M x N grid for
every expert; a greedy pass settles experts that prefer the same cell, keeping
each as close to its preferred cell as it can.  The result is the
injective expert -> cell map (grid_assign) that W_big and the fused forward
use.

The pages name the steps but not their details.  The readings taken here:

  embedding   each column of a factor gets the sign that makes its entry of
              largest magnitude positive (the first such entry on ties; an
              SVD fixes a singular vector only up to sign), then the factor
              is flattened row-major and divided by its L2 norm (a zero
              factor stays zero).
  biclustering  rows share the left (output-space) basis, columns the right
              (input-space) one, so K-Means on the U-embeddings with
              min(M, K) clusters gives the row m, K-Means on the
              V-embeddings with min(N, K) clusters gives the column n.
  K-Means     Lloyd's algorithm on squared Euclidean distance.  The first
              centre is point 0; each further centre is the point farthest
              from the centres chosen so far (farthest-first traversal, no
              random draw; ties -> lowest point index).  Assignment: nearest
              centre, ties -> lowest centre index.  Update: each centre
              becomes the mean of its points; a centre with no points keeps
              its place.  Stop when an update leaves every assignment
              unchanged, or after max_iter updates.
  greedy      over all (expert, cell) pairs, repeatedly take the pair with
              the smallest squared grid distance (m - m*)^2 + (n - n*)^2
              between the cell and the expert's ideal (m*, n*), ties ->
              lower expert index, then lower cell index m*N + n, among
              experts not yet placed and cells still free.

PINS (tests/test_placement_oracle.py):
  embed ... hand case; invariance to the sign of any column; unit norm
  farthest_first ... hand case on points of a line
  kmeans ... scikit-learn's Lloyd KMeans from the same initial centres
      (labels equal); the fixed-point property (every point at its nearest
      centre, every centre the mean of its points); hand case
  greedy_place ... hand cases with conflicts; injective; experts whose ideal
      cell nobody else wants keep it; total distance equal to the optimal
      assignment (scipy's linear_sum_assignment) when there is no conflict
  place_experts ... recovers a planted grid (rows and columns up to a
      relabelling) from noisy, randomly sign-flipped factors
"""
from __future__ import annotations

import numpy as np

__all__ = ["canonical_signs", "embed", "farthest_first", "kmeans", "greedy_place",
           "place_experts"]


def canonical_signs(f) -> np.ndarray:
    """f [d, r] -> f with column j multiplied by the sign of its entry of
    largest magnitude (first such row on ties; +1 for a zero column)."""
    f = np.asarray(f, dtype=np.float64)
    out = f.copy()
    for j in range(f.shape[1]):
        i = int(np.argmax(np.abs(f[:, j])))     # argmax returns the first maximum
        if f[i, j] < 0:
            out[:, j] = -f[:, j]
    return out


def embed(f) -> np.ndarray:
    """The feature embedding of one factor [d, r]: sign-fixed, flattened
    row-major, unit L2 norm (a zero factor gives the zero vector)."""
    e = canonical_signs(f).reshape(-1)
    n = np.sqrt(np.sum(e * e))
    return e / n if n > 0 else e


def _sqdist(a, b) -> float:
    d = a - b
    return float(np.sum(d * d))


def farthest_first(E, C: int) -> list:
    """Indices of C initial centres among the rows of E (see the module text)."""
    E = np.asarray(E, dtype=np.float64)
    chosen = [0]
    mind = np.array([_sqdist(E[i], E[0]) for i in range(len(E))])
    while len(chosen) < C:
        best = 0
        for i in range(len(E)):
            if mind[i] > mind[best]:
                best = i
        chosen.append(best)
        for i in range(len(E)):
            mind[i] = min(mind[i], _sqdist(E[i], E[best]))
    return chosen


def kmeans(E, C: int, max_iter: int):
    """Lloyd's K-Means on the rows of E with C clusters (C <= len(E)).
    Returns (labels int32 [len(E)], centres float64 [C, D], updates run)."""
    E = np.asarray(E, dtype=np.float64)
    P = len(E)
    centres = E[farthest_first(E, C)].copy()

    def assign(cs):
        lab = np.zeros(P, dtype=np.int32)
        for i in range(P):
            d = [_sqdist(E[i], cs[j]) for j in range(C)]
            lab[i] = int(np.argmin(d))          # first minimum: lowest centre index
        return lab

    labels = assign(centres)
    it = 0
    while it < max_iter:
        for j in range(C):
            members = E[labels == j]
            if len(members):
                centres[j] = members.mean(axis=0)
        it += 1
        new = assign(centres)
        if np.array_equal(new, labels):
            break
        labels = new
    return labels, centres, it


def greedy_place(ideal_m, ideal_n, M: int, N: int) -> np.ndarray:
    """grid_assign int32 [K] (cell m*N + n) from the ideal coordinates."""
    K = len(ideal_m)
    pairs = []
    for k in range(K):
        for m in range(M):
            for n in range(N):
                d = (m - int(ideal_m[k])) ** 2 + (n - int(ideal_n[k])) ** 2
                pairs.append((d, k, m * N + n))
    pairs.sort()
    grid = np.full(K, -1, dtype=np.int32)
    free = np.ones(M * N, dtype=bool)
    for d, k, cell in pairs:
        if grid[k] < 0 and free[cell]:
            grid[k] = cell
            free[cell] = False
    return grid


def place_experts(u, v, M: int, N: int, max_iter: int = 100):
    """u [K, d_u, r0], v [K, d_v, r0] (the per-expert rank-r0 factors).
    Returns (ideal_m, ideal_n, grid_assign, (updates on U, updates on V))."""
    u = np.asarray(u, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    K = u.shape[0]
    EU = np.stack([embed(u[k]) for k in range(K)])
    EV = np.stack([embed(v[k]) for k in range(K)])
    lm, _, itu = kmeans(EU, min(M, K), max_iter)
    ln, _, itv = kmeans(EV, min(N, K), max_iter)
    return lm, ln, greedy_place(lm, ln, M, N), (itu, itv)
