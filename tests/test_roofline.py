"""Host-side algorithmic work accounting (the numerators of the bench's
roofline fractions), checked against the stored arrays and brute force."""
import numpy as np

import synth
from tiled_rank_b200 import roofline


def test_residual_bytes_match_stored_arrays():
    """One expert's residual bytes equal the bytes of its stored codes, scales
    and zero points (2-bit and 3-bit), for group sizes that fill and that do
    not fill the last zero-point byte."""
    for bits in (2, 3):
        for group in (64, 128, 256):
            cfg = synth.tiny_config(kind=synth.LINEAR, K=2, M=1, N=2, d_model=768 if group == 256 else 640,
                                    d_ff=32, rank=0, group=group, bits=bits)
            if cfg.d_model % group:
                continue
            p = synth.make_layer(cfg, seed=1).projs[0]
            stored = p.codes[0].nbytes + p.scales[0].nbytes + p.zeros[0].nbytes
            if bits == 3:
                stored += p.codes_hi[0].nbytes
            assert roofline.residual_bytes(p.d_out, p.d_in, p.group, bits) == stored, (bits, group)


def test_routing_sets_brute_force():
    rng = np.random.default_rng(3)
    K, M, N, T, k = 12, 3, 4, 40, 3
    grid = rng.permutation(M * N)[:K]
    idx = np.stack([rng.choice(K, size=k, replace=False) for _ in range(T)])
    s = roofline.routing_sets(idx, grid, N)
    assert set(s["experts"].tolist()) == set(idx.ravel().tolist())
    tr = {(t, int(grid[e]) // N) for t in range(T) for e in idx[t]}
    tc = {(t, int(grid[e]) % N) for t in range(T) for e in idx[t]}
    assert s["token_rows"] == len(tr) and s["token_cols"] == len(tc) and s["pairs"] == T * k


def test_work_of_a_linear_layer():
    """Linear layer: residual bytes of the active experts + U rows of active
    grid rows; FLOPs 2*d_in*d_out per pair + the U_m product per (token, row);
    the column projection per (token, column)."""
    cfg = synth.tiny_config(kind=synth.LINEAR, K=4, M=2, N=2, d_model=256, d_ff=64, rank=16, group=64, top_k=2)
    layer = synth.make_layer(cfg, seed=2)
    idx = np.array([[0, 1], [0, 1], [2, 0]])
    w = roofline.work(layer, idx)
    p = layer.projs[0]
    s = roofline.routing_sets(idx, p.grid_assign, layer.N)
    res = 3 * roofline.residual_bytes(p.d_out, p.d_in, p.group)
    assert w["stages"]["residual"]["bytes"] == res + len(s["rows"]) * p.d_out * p.rank * 2
    assert w["stages"]["residual"]["flops"] == 2 * 6 * p.d_in * p.d_out + 2 * s["token_rows"] * p.d_out * p.rank
    assert w["stages"]["zproj"]["flops"] == 2 * s["token_cols"] * p.d_in * p.rank
    io = 3 * p.d_in * 2 + 3 * layer.K * 4 + 3 * p.d_out * 2
    assert w["bytes"] == io + sum(v["bytes"] for v in w["stages"].values())
