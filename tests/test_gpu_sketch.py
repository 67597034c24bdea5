"""Gaussian-sketch global low-rank decomposition on the GPU against the fp64 oracle."""
import numpy as np
import pytest

import synth
from oracle import sketch as osk
from oracle import tileq as oracle

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


def _bf16_bits(a):
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((f + np.uint32(0x7FFF) + ((f >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def run_sketch(torch, w_bits, grid, M, N, omega_t_bits, r):
    """GPU sketch of the experts' bf16 weights w_bits [K][d_out][d_in]; omega_t_bits: the
    transposed Gaussian test matrix, bf16 bits [l][N*d_in]."""
    import ctypes
    from tiled_rank_b200 import _lib as L
    K, d_out, d_in = w_bits.shape
    l = omega_t_bits.shape[0]
    dev = torch.device("cuda:0")
    w = torch.from_numpy(w_bits.view(np.int16)).to(dev)
    om = torch.from_numpy(np.ascontiguousarray(omega_t_bits).view(np.int16)).to(dev)
    g = np.ascontiguousarray(grid, dtype=np.int32)
    wb = L.tileq_wbig()
    wb.K, wb.M, wb.N, wb.d_out, wb.d_in = K, M, N, d_out, d_in
    wb.w = w.data_ptr()
    wb.grid_assign = g.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    ws = torch.zeros(L.tileq_sketch_workspace_size(wb, l, r), dtype=torch.uint8, device=dev)
    U = torch.empty((M * d_out, r), dtype=torch.float32, device=dev)
    S = torch.empty((r,), dtype=torch.float32, device=dev)
    V = torch.empty((N * d_in, r), dtype=torch.float32, device=dev)
    L.tileq_sketch_lowrank(wb, om, l, r, U, S, V, ws)
    torch.cuda.synchronize()
    return U.cpu().numpy().astype(np.float64), S.cpu().numpy().astype(np.float64), V.cpu().numpy().astype(np.float64)


def gaussian_sketch(rng, C, l):
    """The transposed test matrix as bf16 bits [l][C] and its exact float64 value [C][l]."""
    bits = _bf16_bits(rng.standard_normal((l, C)))
    return bits, oracle.widen_bf16(bits).T


def check(gpu, ref, w_big, rtol_s, tol_prod):
    (u, s, v), (uo, so, vo) = gpu, ref
    np.testing.assert_allclose(s, so, rtol=rtol_s, atol=rtol_s * so[0])
    prod, prod_o = (u * s) @ v.T, (uo * so) @ vo.T
    assert np.abs(prod - prod_o).max() <= tol_prod * np.abs(prod_o).max()
    r = len(s)
    np.testing.assert_allclose(u.T @ u, np.eye(r), atol=1e-3)
    np.testing.assert_allclose(v.T @ v, np.eye(r), atol=1e-3)


@pytest.mark.parametrize("M,N,d_out,d_in,r,l", [(2, 2, 256, 128, 8, 8), (2, 3, 128, 128, 12, 20),
                                               (3, 2, 128, 256, 16, 24)])
def test_planted_rank(torch_cuda, M, N, d_out, d_in, r, l):
    """A rank-r W_big (rounded to bf16: a rank-r part plus a tiny full-rank rest)."""
    rng = np.random.default_rng(M * 100 + N * 10 + r)
    R, C = M * d_out, N * d_in
    u0, _ = np.linalg.qr(rng.standard_normal((R, r)))
    v0, _ = np.linalg.qr(rng.standard_normal((C, r)))
    big = (u0 * np.linspace(3.0, 1.0, r)) @ v0.T
    grid = rng.permutation(M * N)
    w = np.empty((M * N, d_out, d_in))
    for k in range(M * N):
        m, n = divmod(int(grid[k]), N)
        w[k] = big[m * d_out:(m + 1) * d_out, n * d_in:(n + 1) * d_in]
    w_bits = _bf16_bits(w)
    w_big = osk.assemble_wbig(w_bits, grid, M, N)
    om_bits, omega = gaussian_sketch(rng, C, l)
    ref = osk.sketch_lowrank(w_big, omega, r)
    gpu = run_sketch(torch_cuda, w_bits, grid, M, N, om_bits, r)
    check(gpu, ref, w_big, 1e-4, 1e-4)


def test_decaying_spectrum(torch_cuda):
    """A full-rank W_big with a geometric spectrum: the rank-r part of the sketch."""
    rng = np.random.default_rng(3)
    M, N, d_out, d_in, r, l = 2, 2, 128, 128, 16, 32
    R, C = M * d_out, N * d_in
    n = min(R, C)
    qa, _ = np.linalg.qr(rng.standard_normal((R, n)))
    qb, _ = np.linalg.qr(rng.standard_normal((C, n)))
    big = (qa * 0.85 ** np.arange(n)) @ qb.T
    grid = np.arange(M * N)
    w = np.stack([big[(k // N) * d_out:(k // N + 1) * d_out, (k % N) * d_in:(k % N + 1) * d_in]
                  for k in range(M * N)])
    w_bits = _bf16_bits(w)
    w_big = osk.assemble_wbig(w_bits, grid, M, N)
    om_bits, omega = gaussian_sketch(rng, C, l)
    ref = osk.sketch_lowrank(w_big, omega, r)
    gpu = run_sketch(torch_cuda, w_bits, grid, M, N, om_bits, r)
    check(gpu, ref, w_big, 1e-3, 1e-3)


@pytest.mark.slow
def test_mixtral_shaped_gate(torch_cuda):
    """The gate projection of the Mixtral-shaped layer (8 experts on 2x4, 14336 x 4096
    each): W_big 28672 x 16384, rank 128 with 8 columns of oversampling."""
    cfg = synth.CONFIGS[1]
    layer = synth.make_layer(cfg)
    p = layer.projs[0]
    w = np.stack([oracle.expert_weight(p, e, layer.N) for e in range(layer.K)])
    w_bits = _bf16_bits(w)
    del w
    r, l = 128, 136
    rng = np.random.default_rng(11)
    om_bits, omega = gaussian_sketch(rng, layer.N * p.d_in, l)
    w_big = osk.assemble_wbig(w_bits, p.grid_assign, layer.M, layer.N)
    ref = osk.sketch_lowrank(w_big, omega, r)
    gpu = run_sketch(torch_cuda, w_bits, p.grid_assign, layer.M, layer.N, om_bits, r)
    check(gpu, ref, w_big, 1e-3, 2e-3)
