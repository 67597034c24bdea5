"""fp64 oracle of the global low-rank step of TileQ (test infrastructure only).

TileQ technical summary, section 2.1 "2D-Tiling Structured Low-Rank
Quantization", step 5 (Quantization): W_big, the block matrix with expert k
in grid block (m, n) of the M x N grid, is decomposed once at low rank, by a
Gaussian sketch rather than a full SVD; that decomposition's factors U, Sigma,
V are the shared factors the fused forward reads.

The pages name the technique but not its steps.  The plainest reading, taken
here, is the randomised range finder with a Gaussian test matrix followed by
an exact SVD of the small projected matrix:

    Y = W_big Omega              (Omega: [N*d_in, l] Gaussian, l = r + p)
    Q = an orthonormal basis of range(Y)
    B = Q^T W_big                ([l, N*d_in])
    B = U_B diag(s) V_B^T        (SVD of the small matrix)
    U = Q U_B[:, :r],  Sigma = s[:r],  V = V_B[:, :r]

so that U diag(Sigma) V^T is the rank-r truncated SVD of Q Q^T W_big.  No power
iterations (the pages mention none).  Omega is an input: the random numbers are
drawn by the input generator, not here.  Library primitives (QR, SVD) serve as
steps, with no blocking or reordering.

PINS (tests/test_sketch_oracle.py):
  assemble_wbig ... every block equals its expert's weights, by construction
  sketch_lowrank ... exact recovery of a synthetic rank-r W_big (U0 diag(s0) V0^T
      with orthonormal U0, V0): Sigma == s0, the product == W_big, orthonormal
      U and V, also with l > r (rank-deficient sketch); a full-rank matrix with
      a known spectrum stays within the expectation bound of Halko, Martinsson
      and Tropp (2011) for the Gaussian range finder (plus sigma_{r+1} for the
      rank-r truncation), on the seeded draw
"""
from __future__ import annotations

import numpy as np

from .tileq import widen_bf16

__all__ = ["assemble_wbig", "sketch_lowrank", "range_finder_bound"]


def assemble_wbig(w_bits, grid_assign, M: int, N: int) -> np.ndarray:
    """W_big float64 [M*d_out, N*d_in]: expert k's bf16 weights [d_out, d_in] in block
    (m, n) with grid_assign[k] = m*N + n."""
    w = widen_bf16(w_bits)
    K, d_out, d_in = w.shape
    big = np.zeros((M * d_out, N * d_in), dtype=np.float64)
    for k in range(K):
        m, n = divmod(int(grid_assign[k]), N)
        big[m * d_out:(m + 1) * d_out, n * d_in:(n + 1) * d_in] = w[k]
    return big


def sketch_lowrank(w_big, omega, r: int):
    """Randomised range finder + SVD of the projected matrix (see the module text).

    w_big float64 [R, C]; omega float64 [C, l] with l >= r.
    Returns U [R, r], Sigma [r] (descending), V [C, r].
    """
    w_big = np.asarray(w_big, dtype=np.float64)
    omega = np.asarray(omega, dtype=np.float64)
    if omega.shape[1] < r:
        raise ValueError("sketch narrower than the rank")
    y = w_big @ omega
    q, _ = np.linalg.qr(y)
    b = q.T @ w_big
    ub, s, vbt = np.linalg.svd(b, full_matrices=False)
    return q @ ub[:, :r], s[:r], vbt[:r].T


def range_finder_bound(sigma_all, r: int, l: int) -> float:
    """Expectation bound of Halko, Martinsson and Tropp (2011) on the spectral
    error ||W - Q Q^T W|| of the range finder with l = r + p Gaussian samples:
        (1 + 4 sqrt(l) / (p - 1) * sqrt(min(R, C))) * sigma_{r+1}
    (p >= 2).  sigma_all: every singular value of W_big, descending."""
    p = l - r
    if p < 2:
        raise ValueError("oversampling p must be >= 2")
    n = len(sigma_all)
    return (1.0 + 4.0 * np.sqrt(l) / (p - 1) * np.sqrt(n)) * float(sigma_all[r])
