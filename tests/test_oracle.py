"""Pins of the fp64 oracle against what the TileQ paper and plain mathematics fix.

None of these compares the oracle with itself: each case has an independent
expectation (a hand-decoded fixture, a closed form, a brute-force definition,
a different association order, or a property of the global factorisation).
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth
from helpers import diag_residual, make_proj, pack_codes, pack_zeros, rel_err

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


# ---------------------------------------------------------------------------
# stored values
# ---------------------------------------------------------------------------
def test_widen_exact_values():
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x0000, 0x8000, 0x4049], dtype=np.uint16)
    got = oracle.widen_bf16(bits)
    assert got.tolist()[:5] == [1.0, -2.0, 0.25, 0.0, -0.0]
    assert got[5] == 3.140625
    assert oracle.widen_fp16(np.array([1.0, 0.5, -65504.0], dtype=np.float16)).tolist() == [1.0, 0.5, -65504.0]
    # bf16 rounding of the input generator: RNE at the half-way point
    assert synth.to_bf16_bits(np.array([1.0 + 2 ** -8], dtype=np.float32))[0] == 0x3F80
    assert synth.to_bf16_bits(np.array([1.0 + 3 * 2 ** -8], dtype=np.float32))[0] == 0x3F82


def test_dequant_golden_fixture():
    rows = list(_fixture_lines("dequant_16x2.txt"))
    assert len(rows) == 2
    words = np.array([[int(r[1], 16)] for r in rows], dtype=np.uint32)[None]   # [1, 2, 1]
    q_expected = np.array([[int(v) for v in r[2].split()] for r in rows])
    zbytes = np.array([[int(r[3], 16)] for r in rows], dtype=np.uint8)[None]  # [1, 2, 1]
    z_expected = np.array([[int(v) for v in r[4].split()] for r in rows])
    scales = np.array([[float(v) for v in r[5].split()] for r in rows], dtype=np.float16)[None]
    w_expected = np.array([[float(v) for v in r[6].split()] for r in rows])

    assert (oracle.unpack_codes(words[0], 16) == q_expected).all()
    assert (oracle.unpack_zeros(zbytes[0], 2) == z_expected).all()
    # the test-side packer agrees with the hand-decoded words
    assert (pack_codes(q_expected) == words[0]).all()
    assert (pack_zeros(z_expected) == zbytes[0]).all()

    p = synth.Proj(16, 2, 0, 8, np.zeros(1, np.int32), np.zeros((2, 0), np.uint16),
                   np.zeros(0, np.float32), np.zeros((16, 0), np.uint16), words, scales, zbytes)
    assert (oracle.dequant(p, 0) == w_expected).all()


def test_unpack_roundtrip_random():
    rng = np.random.default_rng(5)
    q = rng.integers(0, 4, size=(3, 5, 64), dtype=np.uint8)
    assert (oracle.unpack_codes(pack_codes(q), 64) == q).all()
    for G in (1, 2, 3, 4, 5, 11, 32, 112):
        z = rng.integers(0, 4, size=(2, 7, G), dtype=np.uint8)
        assert (oracle.unpack_zeros(pack_zeros(z), G) == z).all()


def test_generator_zero_tail_cleared():
    # G = 1408/128 = 11 groups: the last zero byte holds 3 fields, its top field is 0
    layer = synth.make_layer(synth.tiny_config(d_model=64, d_ff=176, group=16), seed=1)
    down = layer.projs[2]
    assert down.n_groups == 11
    assert ((down.zeros[..., -1] >> 6) == 0).all()


# ---------------------------------------------------------------------------
# routing and permutation
# ---------------------------------------------------------------------------
def test_route_golden_cases():
    n = 0
    for logits_s, k_s, idx_s, w_s in _fixture_lines("route_cases.txt"):
        logits = np.array([[float(v) for v in logits_s.split()]], dtype=np.float32)
        idx, w = oracle.route(logits, int(k_s))
        assert idx[0].tolist() == [int(v) for v in idx_s.split()]
        w_exp = [eval(e, {"math": math}) for e in w_s.split()]
        np.testing.assert_allclose(w[0], w_exp, rtol=1e-12, atol=0)
        n += 1
    assert n == 7


def _topk_property_holds(row, chosen, k):
    """Brute-force definition: chosen beats every unchosen expert (ties -> lower id)."""
    K = len(row)
    if len(set(chosen)) != k:
        return False
    rest = [e for e in range(K) if e not in chosen]
    for a in chosen:
        for b in rest:
            if not (row[a] > row[b] or (row[a] == row[b] and a < b)):
                return False
    # output order: descending logit, ties by id
    for a, b in zip(chosen, chosen[1:]):
        if not (row[a] > row[b] or (row[a] == row[b] and a < b)):
            return False
    return True


def test_route_bruteforce_tiny():
    rng = np.random.default_rng(11)
    for trial in range(200):
        K = int(rng.integers(1, 7))
        k = int(rng.integers(1, K + 1))
        # many ties: small integer logits
        row = rng.integers(-2, 3, size=K).astype(np.float32)
        idx, w = oracle.route(row[None], k)
        assert _topk_property_holds(row.tolist(), idx[0].tolist(), k)
        # brute force over all subsets: the chosen set is the unique one with the property
        winners = [s for s in itertools.permutations(range(K), k)
                   if _topk_property_holds(row.tolist(), list(s), k)]
        assert winners == [tuple(idx[0].tolist())]
        ex = np.exp(row[idx[0]].astype(np.float64) - row.max())
        np.testing.assert_allclose(w[0], ex / ex.sum(), rtol=1e-12)
        assert abs(w[0].sum() - 1.0) < 1e-12


def test_permute_bruteforce():
    rng = np.random.default_rng(3)
    for trial in range(50):
        K = int(rng.integers(1, 9))
        T = int(rng.integers(0, 20))
        k = int(rng.integers(1, K + 1))
        idx = np.stack([rng.permutation(K)[:k] for _ in range(T)]) if T else np.zeros((0, k), np.int32)
        off, sp = oracle.permute(idx, K)
        # definition: bucket e lists pairs p with expert e in increasing p
        flat = idx.reshape(-1).tolist()
        expected = []
        expected_off = [0]
        for e in range(K):
            expected += [p for p in range(len(flat)) if flat[p] == e]
            expected_off.append(len(expected))
        assert sp.tolist() == expected
        assert off.tolist() == expected_off


# ---------------------------------------------------------------------------
# 2D-tiled low-rank structure
# ---------------------------------------------------------------------------
def _random_proj(rng, K=6, M=2, N=3, d_in=32, d_out=48, rank=4, group=16):
    q = rng.integers(0, 4, size=(K, d_out, d_in), dtype=np.uint8)
    G = d_in // group
    z = rng.integers(0, 4, size=(K, d_out, G), dtype=np.uint8)
    s = rng.uniform(0.005, 0.02, size=(K, d_out, G))
    U = rng.standard_normal((M * d_out, rank)) / np.sqrt(d_out)
    V = rng.standard_normal((N * d_in, rank)) / np.sqrt(d_in)
    grid = rng.permutation(M * N)[:K]
    return make_proj(K, M, N, d_in, d_out, rank, group, q, z, s, U, V, grid=grid)


def test_factored_equals_reconstructed():
    rng = np.random.default_rng(7)
    p = _random_proj(rng)
    N = 3
    x = rng.standard_normal(p.d_in)
    for e in range(6):
        m, n = oracle.grid_cell(p, e, N)
        Um = oracle.widen_bf16(p.U)[m * p.d_out:(m + 1) * p.d_out]
        Vn = oracle.widen_bf16(p.V)[n * p.d_in:(n + 1) * p.d_in]
        sig = p.Sigma.astype(np.float64)
        factored = Um @ (sig * (Vn.T @ x)) + oracle.dequant(p, e) @ x
        dense = oracle.expert_weight(p, e, N) @ x
        assert rel_err(factored, dense) < 1e-9


def test_lowrank_is_block_of_global_product():
    rng = np.random.default_rng(8)
    M, N = 2, 3
    p = _random_proj(rng, M=M, N=N)
    Wbig = oracle.assemble_wbig_lowrank(p, M, N)
    assert Wbig.shape == (M * p.d_out, N * p.d_in)
    for e in range(6):
        cell = int(p.grid_assign[e])
        m, n = cell // N, cell % N
        block = Wbig[m * p.d_out:(m + 1) * p.d_out, n * p.d_in:(n + 1) * p.d_in]
        np.testing.assert_allclose(oracle.lowrank_block(p, e, N), block, rtol=1e-12, atol=1e-15)


def _hadamard(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_wbig_singular_values_equal_sigma():
    # Orthonormal U, V exactly representable in bf16 (scaled Hadamard columns):
    # the singular values of W_big's low-rank part are exactly Sigma.
    M, N, d_out, d_in, r = 2, 2, 8, 32, 5
    U = _hadamard(16)[:, 1:1 + r] / 4.0                 # [M*d_out=16, r], entries +-1/4
    V = _hadamard(64)[:, 2:2 + r] / 8.0                 # [N*d_in=64, r], entries +-1/8
    sig = np.array([3.0, 2.0, 1.0, 0.5, 0.25], dtype=np.float32)
    K = 4
    zq = np.zeros((K, d_out, d_in), np.uint8)
    zz = np.zeros((K, d_out, 2), np.uint8)
    p = make_proj(K, M, N, d_in, d_out, r, 16, zq, zz, np.ones((K, d_out, 2)), U, V, sig)
    Wbig = oracle.assemble_wbig_lowrank(p, M, N)
    sv = np.linalg.svd(Wbig, compute_uv=False)
    np.testing.assert_allclose(sv[:r], sig, rtol=1e-12)
    assert np.all(sv[r:] < 1e-12)
    # and the tiled blocks of the experts tile W_big exactly (every cell used)
    rebuilt = np.zeros_like(Wbig)
    for e in range(K):
        m, n = oracle.grid_cell(p, e, N)
        rebuilt[m * d_out:(m + 1) * d_out, n * d_in:(n + 1) * d_in] = oracle.expert_weight(p, e, N)
    np.testing.assert_allclose(rebuilt, Wbig, rtol=0, atol=1e-15)


def test_2d_sharing_locality():
    """Changing U block m changes exactly the experts of grid row m; V block n, column n."""
    rng = np.random.default_rng(9)
    M, N, K = 2, 3, 6
    p = _random_proj(rng, K=K, M=M, N=N)
    base = [oracle.expert_weight(p, e, N) for e in range(K)]
    rows = [int(c) // N for c in p.grid_assign]
    cols = [int(c) % N for c in p.grid_assign]
    for m in range(M):
        U2 = p.U.copy()
        U2[m * p.d_out:(m + 1) * p.d_out] ^= np.uint16(0x8000)     # flip signs of block m
        p2 = synth.Proj(**{**p.__dict__, "U": U2})
        for e in range(K):
            changed = not np.array_equal(oracle.expert_weight(p2, e, N), base[e])
            assert changed == (rows[e] == m)
    for n in range(N):
        V2 = p.V.copy()
        V2[n * p.d_in:(n + 1) * p.d_in] ^= np.uint16(0x8000)
        p2 = synth.Proj(**{**p.__dict__, "V": V2})
        for e in range(K):
            changed = not np.array_equal(oracle.expert_weight(p2, e, N), base[e])
            assert changed == (cols[e] == n)


# ---------------------------------------------------------------------------
# the layer: special cases with independent expectations
# ---------------------------------------------------------------------------
def _linear_layer(proj, K, M, N, top_k):
    return synth.Layer(synth.LINEAR, K, M, N, proj.d_in, proj.d_out, top_k, [proj])


def test_rank0_reduces_to_dequant_gemm():
    rng = np.random.default_rng(21)
    K, M, N, d_in, d_out, g = 4, 2, 2, 32, 16, 16
    q = rng.integers(0, 4, size=(K, d_out, d_in), dtype=np.uint8)
    z = rng.integers(0, 4, size=(K, d_out, d_in // g), dtype=np.uint8)
    s = np.array([0.5, 0.25, 1.0, 2.0])[rng.integers(0, 4, size=(K, d_out, d_in // g))]
    p = make_proj(K, M, N, d_in, d_out, 0, g, q, z, s)
    layer = _linear_layer(p, K, M, N, 2)
    x = synth.to_bf16_bits(rng.standard_normal((5, d_in)).astype(np.float32))
    logits = rng.standard_normal((5, K)).astype(np.float32)
    out = oracle.forward(layer, x, logits)
    idx, w = oracle.route(logits, 2)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(5):
        ref = np.zeros(d_out)
        for j in range(2):
            e = idx[t, j]
            Wd = (q[e].astype(np.float64) - np.repeat(z[e], g, axis=1)) * np.repeat(s[e], g, axis=1)
            ref += w[t, j] * (Wd @ xf[t])
        assert rel_err(out[t], ref) < 1e-12


def test_zero_residual_reduces_to_wbig_lowrank():
    rng = np.random.default_rng(22)
    K, M, N, d_in, d_out, g, r = 6, 2, 3, 32, 16, 16, 3
    z = rng.integers(0, 4, size=(K, d_out, d_in // g), dtype=np.uint8)
    q = np.repeat(z, g, axis=2)                       # q == z everywhere -> deq == 0 exactly
    s = rng.uniform(0.005, 0.02, size=(K, d_out, d_in // g))
    U = rng.standard_normal((M * d_out, r)) / 4
    V = rng.standard_normal((N * d_in, r)) / 6
    grid = rng.permutation(M * N)
    p = make_proj(K, M, N, d_in, d_out, r, g, q, z, s, U, V, grid=grid)
    layer = _linear_layer(p, K, M, N, 3)
    x = synth.to_bf16_bits(rng.standard_normal((4, d_in)).astype(np.float32))
    logits = rng.standard_normal((4, K)).astype(np.float32)
    out = oracle.forward(layer, x, logits)
    Wbig = oracle.assemble_wbig_lowrank(p, M, N)
    idx, w = oracle.route(logits, 3)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(4):
        ref = np.zeros(d_out)
        for j in range(3):
            cell = int(grid[idx[t, j]])
            m, n = cell // N, cell % N
            ref += w[t, j] * (Wbig[m * d_out:(m + 1) * d_out, n * d_in:(n + 1) * d_in] @ xf[t])
        assert rel_err(out[t], ref) < 1e-12


def _swiglu_diag_layer(K, d, diag_gate, diag_up, diag_down, top_k, shared=None):
    projs = []
    for diag in (diag_gate, diag_up, diag_down):
        q, z, s = diag_residual(K, d, 16, diag)
        projs.append(make_proj(K, 1, K, d, d, 0, 16, q, z, s))
    return synth.Layer(synth.SWIGLU, K, 1, K, d, d, top_k, projs, shared)


def test_swiglu_and_combine_closed_form():
    # Two experts whose gate/up/down are multiples of the identity (exact in the
    # stored format: s = 1, z = 0, q on the diagonal).  Expert e computes
    # y = c_d * silu(c_g x) * (c_u x) elementwise; the layer sums w_j y_j.
    d = 16
    layer = _swiglu_diag_layer(2, d, diag_gate=[1, 2], diag_up=[2, 1], diag_down=[1, 3], top_k=2)
    xs = np.array([1.0, -1.0, 0.5, 2.0, 0.0, -3.0, 0.25, 1.5] * 2, dtype=np.float32)
    x = synth.to_bf16_bits(xs[None])
    logits = np.array([[0.0, 1.0]], dtype=np.float32)
    out = oracle.forward(layer, x, logits)[0]
    w1 = 1 / (1 + math.exp(-1.0))        # expert 1 has the larger logit
    w0 = 1 - w1
    for i, a in enumerate(xs.astype(np.float64)):
        y0 = 1 * (a / (1 + math.exp(-a))) * (2 * a)
        y1 = 3 * ((2 * a) / (1 + math.exp(-2 * a))) * (1 * a)
        assert abs(out[i] - (w1 * y1 + w0 * y0)) < 1e-12


def test_shared_expert_added_with_unit_weight():
    # Routed experts contribute zero (q == z == 0).  The shared expert's
    # weights are the cyclic shift S (S x)_i = x_{i+1}, exact in bf16:
    # gate = S, up = 2S, down = S, so out_i = silu(x_{i+2}) * 2 x_{i+2}
    # (a transposed projection would shift the other way), whatever the
    # routing weights (top-2 with unequal logits: 0.27 / 0.73, none of which
    # may scale the shared expert).
    d = 16
    shift = np.roll(np.eye(d, dtype=np.float32), 1, axis=1)     # shift[i, (i+1) % d] = 1
    assert (shift @ np.arange(d) == (np.arange(d) + 1) % d).all()
    shared = {"gate": synth.to_bf16_bits(shift), "up": synth.to_bf16_bits(2 * shift),
              "down": synth.to_bf16_bits(shift)}
    layer = _swiglu_diag_layer(2, d, [0, 0], [0, 0], [0, 0], top_k=2, shared=shared)
    xs = np.linspace(-2, 2, d).astype(np.float32)
    x = synth.to_bf16_bits(xs[None])
    out = oracle.forward(layer, x, np.array([[0.0, 1.0]], np.float32))[0]
    xf = synth.bf16_bits_to_f32(x)[0].astype(np.float64)
    for i in range(d):
        a = xf[(i + 2) % d]
        assert abs(out[i] - (a / (1 + math.exp(-a))) * 2 * a) < 1e-12


def test_single_expert_top1_is_one_linear_layer():
    rng = np.random.default_rng(23)
    K, d_in, d_out, g = 1, 32, 16, 16
    q = rng.integers(0, 4, size=(K, d_out, d_in), dtype=np.uint8)
    z = rng.integers(0, 4, size=(K, d_out, d_in // g), dtype=np.uint8)
    s = np.full((K, d_out, d_in // g), 0.125)
    U = rng.standard_normal((d_out, 2))
    V = rng.standard_normal((d_in, 2))
    p = make_proj(K, 1, 1, d_in, d_out, 2, g, q, z, s, U, V, sigma=[1.0, 0.5])
    layer = _linear_layer(p, K, 1, 1, 1)
    x = synth.to_bf16_bits(rng.standard_normal((3, d_in)).astype(np.float32))
    out = oracle.forward(layer, x, np.zeros((3, 1), np.float32))
    Uf = synth.bf16_bits_to_f32(synth.to_bf16_bits(U)).astype(np.float64)
    Vf = synth.bf16_bits_to_f32(synth.to_bf16_bits(V)).astype(np.float64)
    W = Uf @ np.diag([1.0, 0.5]) @ Vf.T + 0.125 * (q[0].astype(np.float64) - np.repeat(z[0], g, axis=1))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(out, xf @ W.T, rtol=1e-12, atol=1e-13)


def test_batched_matches_per_token_loop():
    cfg = synth.tiny_config(K=6, M=2, N=3, d_model=32, d_ff=48, rank=4, group=16, top_k=2,
                            shared_d_ff=32)
    layer = synth.make_layer(cfg, seed=4)
    logits, x = synth.make_inputs(cfg, 9, seed=4)
    a = oracle.forward(layer, x, logits)
    b = oracle.forward_batched(layer, x, logits)
    assert rel_err(b, a) < 1e-12
    sub = oracle.forward(layer, x, logits, tokens=[7, 2])
    assert rel_err(sub, a[[7, 2]]) < 1e-12
    # the token subset of the batched form, in the given order, with a repeat
    subb = oracle.forward_batched(layer, x, logits, tokens=[8, 0, 3, 0])
    assert rel_err(subb, a[[8, 0, 3, 0]]) < 1e-12


def test_memory_closed_form():
    # shared tiled factors vs per-expert factors: ratio 2MN/(M+N) when d_in == d_out
    for M, N, expect in ((8, 8, 8.0), (2, 4, 16 / 6), (6, 10, 120 / 16)):
        tiled = oracle.lowrank_bytes_tiled(M, N, 1024, 1024, 64)
        per = oracle.lowrank_bytes_per_expert(M * N, 1024, 1024, 64)
        assert abs(per / tiled - expect) < 1e-12


def test_route_full_softmax_variant():
    """The chosen entries of the softmax over all K logits (not renormalised):
    the same order as the default; weights = renormalised weights times the
    chosen share of the full softmax mass; hand case below."""
    rng = np.random.default_rng(4)
    lg = (rng.standard_normal((20, 9)) * 2).astype(np.float32)
    i0, w0 = oracle.route(lg, 3)
    i1, w1 = oracle.route(lg, 3, full_softmax=True)
    assert np.array_equal(i0, i1)
    full = np.exp(lg.astype(np.float64) - lg.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)
    chosen = np.take_along_axis(full, i1.astype(np.int64), axis=1)
    np.testing.assert_allclose(w1, chosen, rtol=1e-13)
    np.testing.assert_allclose(w1, w0 * chosen.sum(axis=1, keepdims=True), rtol=1e-13)
    assert np.all(w1.sum(axis=1) < 1.0)
    # hand case: logits (0, ln 2, ln 3), top-2 -> 3/6 and 2/6
    i, w = oracle.route(np.log(np.array([[1.0, 2.0, 3.0]], dtype=np.float32)), 2, full_softmax=True)
    assert list(i[0]) == [2, 1]
    np.testing.assert_allclose(w[0], [0.5, 1.0 / 3.0], rtol=1e-6)


def test_layer_follows_the_route_mode():
    """The layer forward applies the layer's routing variant.  Three linear
    experts computing 1x, 2x, 3x (identity residuals); logits (0, ln 2, ln 3),
    top-2 picks experts 2 and 1: default weights 3/5, 2/5 give 13/5 x; the
    full-softmax variant's 3/6, 2/6 give 13/6 x (per token and batched)."""
    d = 16
    q, z, s = diag_residual(3, d, 16, [1, 2, 3])
    p = make_proj(3, 1, 3, d, d, 0, 16, q, z, s)
    xs = np.linspace(-2, 2, d).astype(np.float32)
    x = synth.to_bf16_bits(np.stack([xs, -xs]))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    logits = np.log(np.array([[1.0, 2.0, 3.0]] * 2, dtype=np.float32))
    for mode, factor in ((0, 13.0 / 5.0), (1, 13.0 / 6.0)):
        layer = synth.Layer(synth.LINEAR, 3, 1, 3, d, d, 2, [p], route_mode=mode)
        for out in (oracle.forward(layer, x, logits), oracle.forward_batched(layer, x, logits)):
            np.testing.assert_allclose(out, factor * xf, rtol=1e-6, atol=1e-12)


def test_dequant_3bit_hand_case():
    """3-bit residual, hand-packed: q_j = j % 8 for j < 32, group 16, zeros (5, 2),
    scales (0.5, 0.25).  Low 2 bits (0, 1, 2, 3, ...) at bits 2*(j%16): 0xE4 per
    byte; high bits (q >= 4 for j % 8 in 4..7) at bit j: 0xF0 per byte; zeros
    5 | 2 << 4 = 0x25."""
    import dataclasses
    p = synth.Proj(32, 1, 0, 16, np.zeros(1, np.int32), np.zeros((1, 0), np.uint16),
                   np.zeros(0, np.float32), np.zeros((1, 0), np.uint16),
                   np.array([[[0xE4E4E4E4, 0xE4E4E4E4]]], np.uint32),
                   np.array([[[0.5, 0.25]]], np.float16), np.array([[[0x25]]], np.uint8),
                   3, np.array([[[0xF0F0F0F0]]], np.uint32))
    j = np.arange(32)
    want = np.where(j < 16, 0.5 * (j % 8 - 5), 0.25 * (j % 8 - 2))
    assert np.array_equal(oracle.dequant(p, 0)[0], want)
    assert list(oracle.unpack_zeros(np.array([0x25, 0x07], np.uint8), 3, bits=3)) == [5, 2, 7]
    # a zero high plane with the same zero points is the 2-bit residual
    two = dataclasses.replace(p, bits=2, codes_hi=None, zeros=np.array([[[0x09]]], np.uint8))  # 1 | 2 << 2
    three = dataclasses.replace(p, codes_hi=np.zeros((1, 1, 1), np.uint32), zeros=np.array([[[0x21]]], np.uint8))
    assert np.array_equal(oracle.dequant(two, 0), oracle.dequant(three, 0))


def test_dequant_3bit_range():
    cfg = synth.tiny_config(K=3, M=2, N=2, d_model=128, d_ff=64, rank=0, group=64, bits=3)
    layer = synth.make_layer(cfg, seed=5)
    for p in layer.projs:
        assert p.bits == 3 and p.codes_hi.shape == (3, p.d_out, p.d_in // 32)
        G = p.d_in // p.group
        z = oracle.unpack_zeros(p.zeros, G, 3)
        assert z.max() <= 7 and z.shape[-1] == G
        s = oracle.widen_fp16(p.scales)
        for e in range(3):
            w = oracle.dequant(p, e)
            ratio = np.abs(w).reshape(p.d_out, G, p.group) / s[e][:, :, None]
            assert ratio.max() <= 7.0 and ratio.max() >= 6.0   # q and z span 0..7


def test_route_nonfinite_logits():
    """A NaN logit ranks as -inf (below every finite logit; among -inf and NaN the
    lower index first); a token whose chosen logits are all -inf gets equal weights."""
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    lg = np.array([[0.5, nan, -1.0, 2.0],
                   [nan, nan, 1.0, nan],
                   [-inf, nan, -inf, nan]], dtype=np.float32)
    idx, w = oracle.route(lg, 2)
    assert idx.tolist() == [[3, 0], [2, 0], [0, 1]]
    e = np.exp(0.5 - 2.0)
    np.testing.assert_allclose(w[0], [1 / (1 + e), e / (1 + e)], rtol=1e-15)
    np.testing.assert_allclose(w[1], [1.0, 0.0], atol=0)
    np.testing.assert_allclose(w[2], [0.5, 0.5], atol=0)
    idx_f, w_f = oracle.route(lg, 2, full_softmax=True)
    assert np.array_equal(idx_f, idx)
    np.testing.assert_allclose(w_f[1], [1.0, 0.0], atol=0)   # NaN entries add nothing to the mass
    np.testing.assert_allclose(w_f[2], [0.25, 0.25], atol=0)
