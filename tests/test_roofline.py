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


def test_work_of_a_swiglu_layer_with_shared_expert():
    """SwiGLU layer, brute force: bytes from the stored arrays themselves (each
    active expert's codes, scales and zero points once per projection; the
    U_m / V_n slices of active grid rows / columns once; the shared expert's
    weights), FLOPs by a loop over the (token, slot) pairs and the distinct
    (token, row) / (token, column) sets."""
    cfg = synth.tiny_config(K=6, M=2, N=3, d_model=128, d_ff=192, rank=8, group=64, top_k=2,
                            shared_d_ff=64)
    layer = synth.make_layer(cfg, seed=5)
    idx = np.array([[0, 3], [3, 5], [1, 0], [5, 3]])
    T, k = idx.shape
    w = roofline.work(layer, idx)
    st = w["stages"]

    def stored(p, experts):
        return sum(p.codes[e].nbytes + p.scales[e].nbytes + p.zeros[e].nbytes for e in experts)

    def cells(p):
        return [[divmod(int(p.grid_assign[e]), layer.N) for e in row] for row in idx]

    def u_bytes(p):
        rows = {m for row in cells(p) for m, _ in row}
        return sum(p.U[m * p.d_out:(m + 1) * p.d_out].nbytes for m in rows)

    def v_bytes(p):
        cols = {n for row in cells(p) for _, n in row}
        return sum(p.V[n * p.d_in:(n + 1) * p.d_in].nbytes for n in cols)

    g, u, d = layer.projs
    experts = set(idx.ravel().tolist())
    assert st["gateup"]["bytes"] == stored(g, experts) + stored(u, experts) + u_bytes(g) + u_bytes(u)
    gu_flops = 0
    for t in range(T):
        for j in range(k):
            for p in (g, u):
                gu_flops += 2 * p.d_in * p.d_out + 2 * p.d_out * p.rank
    assert st["gateup"]["flops"] == gu_flops
    # every projection has its own grid placement, so its own (token, column) set
    def token_cols(p):
        return len({(t, n) for t, row in enumerate(cells(p)) for _, n in row})
    assert st["zproj"]["bytes"] == v_bytes(g) + v_bytes(u)
    assert st["zproj"]["flops"] == 2 * (token_cols(g) * g.d_in * g.rank + token_cols(u) * u.d_in * u.rank)
    assert st["zdown"]["bytes"] == v_bytes(d)
    assert st["zdown"]["flops"] == 2 * T * k * d.d_in * d.rank
    tr = {(t, m) for t, row in enumerate(cells(d)) for m, _ in row}
    assert st["residual"]["bytes"] == stored(d, experts) + u_bytes(d)
    assert st["residual"]["flops"] == 2 * T * k * d.d_in * d.d_out + 2 * len(tr) * d.d_out * d.rank
    sh = layer.shared
    assert st["shared"]["bytes"] == sh["gate"].nbytes + sh["up"].nbytes + sh["down"].nbytes
    assert st["shared"]["flops"] == T * 2 * (2 * cfg.d_model * cfg.shared_d_ff + cfg.shared_d_ff * cfg.d_model)
    io = T * cfg.d_model * 2 + T * layer.K * 4 + T * cfg.d_model * 2
    assert w["bytes"] == io + sum(v["bytes"] for v in st.values())
    assert w["flops"] == sum(v["flops"] for v in st.values())
