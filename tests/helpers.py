"""Test-side helpers: an independent packer for the stored residual format and
builders of hand-made layers.  Nothing here is shared with the oracle or the
CUDA library; the packer is the inverse of the format definition, written
separately so that a bit-order mistake on either side shows up."""
from __future__ import annotations

import numpy as np

import synth


def pack_codes(q: np.ndarray) -> np.ndarray:
    """codes uint8 [..., d_in] (values 0..3) -> uint32 [..., d_in/16], element j at bits 2*(j%16)."""
    q = np.asarray(q, dtype=np.uint64)
    d_in = q.shape[-1]
    assert d_in % 16 == 0
    q = q.reshape(q.shape[:-1] + (d_in // 16, 16))
    word = np.zeros(q.shape[:-1], dtype=np.uint64)
    for j in range(16):
        word |= q[..., j] << np.uint64(2 * j)
    return word.astype(np.uint32)


def pack_zeros(z: np.ndarray) -> np.ndarray:
    """zero points uint8 [..., G] -> uint8 [..., ceil(G/4)], group j at bits 2*(j%4) of byte j//4."""
    z = np.asarray(z, dtype=np.uint32)
    G = z.shape[-1]
    nb = (G + 3) // 4
    out = np.zeros(z.shape[:-1] + (nb,), dtype=np.uint32)
    for j in range(G):
        out[..., j // 4] |= z[..., j] << np.uint32(2 * (j % 4))
    return out.astype(np.uint8)


def make_proj(K, M, N, d_in, d_out, rank, group, q, z, s, U=None, V=None, sigma=None, grid=None):
    """Build a synth.Proj from unpacked residual values (q [K,d_out,d_in], z/s [K,d_out,G])."""
    if U is None:
        U = np.zeros((M * d_out, rank), dtype=np.float32)
    if V is None:
        V = np.zeros((N * d_in, rank), dtype=np.float32)
    if sigma is None:
        sigma = (1.0 / (1.0 + np.arange(rank))).astype(np.float32)
    if grid is None:
        grid = np.arange(K, dtype=np.int32)
    return synth.Proj(d_in, d_out, rank, group, np.asarray(grid, dtype=np.int32),
                      synth.to_bf16_bits(U), np.asarray(sigma, dtype=np.float32),
                      synth.to_bf16_bits(V), pack_codes(q), np.asarray(s, dtype=np.float16),
                      pack_zeros(z))


def diag_residual(K, d, group, diag_vals):
    """Residual with w = diag(diag_vals[k]) for each expert (s=1, z=0, q on the diagonal)."""
    q = np.zeros((K, d, d), dtype=np.uint8)
    for k in range(K):
        for i in range(d):
            q[k, i, i] = diag_vals[k]
    z = np.zeros((K, d, d // group), dtype=np.uint8)
    s = np.ones((K, d, d // group), dtype=np.float16)
    return q, z, s


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))
