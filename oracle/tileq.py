"""fp64 oracle of the TileQ MoE-layer forward (test infrastructure only).

Everything here widens the stored bytes (bf16, fp16, packed 2-bit codes, fp32
logits) to float64 and follows the paper's definitions literally:

* Expert k at grid cell (m, n) applies
      W_k = U_m diag(Sigma) V_n^T + deq(Q_k)
  where U_m / V_n are the row-m / column-n blocks of the shared factors of the
  tiled block matrix W_big, and deq(Q_k) is its quantised residual
  (TileQ paper, section 2.1 "2D-Tiling Structured Low-Rank Quantization",
  steps 4-5 and the key technical insight: rows share the left/output basis,
  columns share the right/input basis).
* The residual is asymmetric 2-bit group quantisation along d_in,
  w = s * (q - z) (the residual quantisation of step 5; the stored format is
  the plainest reading, since the pages give no bit layout).
* An MoE layer routes each token to its top-k experts with softmax weights
  over the chosen logits and sums the weighted expert outputs; a SwiGLU expert
  computes h = silu(W_gate x) * (W_up x), y = W_down h (routing is implicit on
  the pages: "only a small subset of experts is active per token").

The W_k are reconstructed densely, the per-token path is a literal loop, and
top-k is an exact full sort: no blocking, fusion or reordering.

PINS (what each function is checked against, in tests/test_oracle.py):
  widen_bf16 / widen_fp16 ... exact bit patterns of known values
  unpack_codes / unpack_zeros / dequant ... hand-decoded golden fixture (2-bit);
      3-bit: hand-decoded case, a zero high plane reduces to the 2-bit result,
      and the residual range |q - z| <= 7
      tests/golden/dequant_16x2.txt, plus a test-side packer
  route ... hand cases (tests/golden/route_cases.txt), softmax closed form,
      brute-force top-k property on tiny inputs; the full-softmax variant
      against the closed form (chosen mass = renormalised weights x that mass)
  permute ... brute-force stable sort definition on tiny inputs
  lowrank_block / expert_weight ... factored == reconstructed (1e-9),
      block of the global product U diag(Sigma) V^T (W_big), singular values of
      W_big == Sigma with orthonormal factors, 2D-sharing perturbation locality
  forward ... rank-0 == dense integer GEMM, zero residual == W_big block
      product, SwiGLU / combine / shared-expert closed forms written in the tests
tests/test_oracle_mutations.py writes plausible mistakes into a copy of this
file (and of sketch.py and placement.py) and checks that these pins reject
every one.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "widen_bf16", "widen_fp16", "route", "permute", "unpack_codes", "unpack_zeros", "unpack_codes_hi",
    "dequant", "grid_cell", "lowrank_block", "expert_weight", "silu", "forward",
    "forward_batched", "assemble_wbig_lowrank", "lowrank_bytes_tiled",
    "lowrank_bytes_per_expert",
]


# ---------------------------------------------------------------------------
# widening of stored values
# ---------------------------------------------------------------------------
def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact): a bf16 is the top half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def widen_fp16(h) -> np.ndarray:
    """fp16 -> float64 (exact)."""
    return np.asarray(h, dtype=np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# routing (implicit on the pages; the plainest reading, see module docstring)
# ---------------------------------------------------------------------------
def route(logits, top_k: int, full_softmax: bool = False):
    """Exact top-k by a full sort and softmax weights.

    Order: descending logit; equal logits -> lower expert index first.
    Default: softmax over the chosen logits,
        w_j = exp(l_j - l_max) / sum_{chosen} exp(l - l_max);
    full_softmax: the chosen entries of the softmax over all K logits, not
    renormalised, w_j = exp(l_j - l_max) / sum_{all K} exp(l - l_max).
    Both in float64.  Returns (idx int32 [T, k], w float64 [T, k]).
    Non-finite logits (the pages only meet finite ones; this is the reading
    taken): a NaN ranks as -inf; when every chosen logit is -inf the weights are
    equal (1/k, or 1/K for the full softmax), the limit of equal logits.
    """
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    lg = np.where(np.isnan(lg), -np.inf, lg)
    T, K = lg.shape
    if not 1 <= top_k <= K:
        raise ValueError("top_k out of range")
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float64)
    for t in range(T):
        order = sorted(range(K), key=lambda e: (-float(lg[t, e]), e))
        chosen = order[:top_k]
        vals = np.array([float(lg[t, e]) for e in chosen], dtype=np.float64)
        idx[t] = chosen
        if vals.max() == -np.inf:
            w[t] = 1.0 / (K if full_softmax else top_k)
            continue
        ex = np.exp(vals - vals.max())
        if full_softmax:
            every = np.exp(lg[t] - vals.max())
            w[t] = ex / every.sum()
        else:
            w[t] = ex / ex.sum()
    return idx, w


def permute(idx, K: int):
    """Stable counting sort of the (token, slot) pairs by expert.

    Pair id p = t*k + j.  expert_offsets[e] .. expert_offsets[e+1] is the
    range of sorted_pairs holding expert e's pairs, in increasing pair id.
    Returns (expert_offsets int32 [K+1], sorted_pairs int32 [T*k]).
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.zeros(K, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(K + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    sorted_pairs = np.empty(flat.size, dtype=np.int32)
    fill = offsets[:-1].astype(np.int64).copy()
    for p, e in enumerate(flat):
        sorted_pairs[fill[e]] = p
        fill[e] += 1
    return offsets, sorted_pairs


# ---------------------------------------------------------------------------
# stored residual format
# ---------------------------------------------------------------------------
def unpack_codes(codes, d_in: int) -> np.ndarray:
    """uint32 [..., d_in/16] -> codes uint8 [..., d_in]; element j at bits 2*(j%16)."""
    c = np.asarray(codes, dtype=np.uint32)
    shifts = (2 * np.arange(16, dtype=np.uint32))
    q = (c[..., None] >> shifts) & np.uint32(3)
    return q.reshape(c.shape[:-1] + (c.shape[-1] * 16,))[..., :d_in].astype(np.uint8)


def unpack_zeros(zeros, n_groups: int, bits: int = 2) -> np.ndarray:
    """Zero points uint8 [..., G].  2-bit: uint8 [..., ceil(G/4)], group j at bits
    2*(j%4) of byte j//4.  3-bit: uint8 [..., ceil(G/2)], group j at bits 4*(j%2)
    of byte j//2 (values 0..7)."""
    zb = np.asarray(zeros, dtype=np.uint8)
    per, width, mask = (4, 2, 3) if bits != 3 else (2, 4, 7)
    shifts = (width * np.arange(per, dtype=np.uint8))
    z = (zb[..., None] >> shifts) & np.uint8(mask)
    return z.reshape(zb.shape[:-1] + (zb.shape[-1] * per,))[..., :n_groups]


def unpack_codes_hi(codes_hi, d_in: int) -> np.ndarray:
    """3-bit codes' high bits: uint32 [..., d_in/32] -> uint8 [..., d_in]; element j at bit j%32."""
    c = np.asarray(codes_hi, dtype=np.uint32)
    q = (c[..., None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)
    return q.reshape(c.shape[:-1] + (c.shape[-1] * 32,))[..., :d_in].astype(np.uint8)


def dequant(proj, e: int) -> np.ndarray:
    """deq(Q_e) float64 [d_out, d_in]: w[o, i] = s[o, i//g] * (q[o, i] - z[o, i//g]).
    2-bit: q from `codes`; 3-bit (proj.bits == 3; the TileQ summary's section 4,
    "Experimental Results", evaluates 2-bit and 3-bit): q = codes + 4 * codes_hi bit."""
    g = proj.group
    G = proj.d_in // g
    bits = getattr(proj, "bits", 2)
    q = unpack_codes(proj.codes[e], proj.d_in).astype(np.int64)
    if bits == 3:
        q = q + 4 * unpack_codes_hi(proj.codes_hi[e], proj.d_in)
    q = q.reshape(proj.d_out, G, g)
    z = unpack_zeros(proj.zeros[e], G, bits).astype(np.float64)
    s = widen_fp16(proj.scales[e])
    # group j of row o covers inputs j*g .. j*g+g-1
    w = (q - z[:, :, None]) * s[:, :, None]
    return w.reshape(proj.d_out, proj.d_in)


# ---------------------------------------------------------------------------
# 2D-tiled low-rank factors
# ---------------------------------------------------------------------------
def grid_cell(proj, e: int, N: int):
    """(m, n) of expert e: cell = m*N + n."""
    cell = int(proj.grid_assign[e])
    return cell // N, cell % N


def lowrank_block(proj, e: int, N: int) -> np.ndarray:
    """U_m diag(Sigma) V_n^T, float64 [d_out, d_in], for the grid cell of expert e."""
    m, n = grid_cell(proj, e, N)
    r = proj.rank
    if r == 0:
        return np.zeros((proj.d_out, proj.d_in), dtype=np.float64)
    Um = widen_bf16(proj.U[m * proj.d_out:(m + 1) * proj.d_out]).reshape(proj.d_out, r)
    Vn = widen_bf16(proj.V[n * proj.d_in:(n + 1) * proj.d_in]).reshape(proj.d_in, r)
    sig = np.asarray(proj.Sigma, dtype=np.float32).astype(np.float64)
    return (Um * sig[None, :]) @ Vn.T


def expert_weight(proj, e: int, N: int) -> np.ndarray:
    """Dense reconstruction W_e = U_m diag(Sigma) V_n^T + deq(Q_e), float64 [d_out, d_in]."""
    return lowrank_block(proj, e, N) + dequant(proj, e)


def assemble_wbig_lowrank(proj, M: int, N: int) -> np.ndarray:
    """The low-rank part of W_big as one product U diag(Sigma) V^T, [M*d_out, N*d_in]."""
    r = proj.rank
    U = widen_bf16(proj.U).reshape(M * proj.d_out, r)
    V = widen_bf16(proj.V).reshape(N * proj.d_in, r)
    sig = np.asarray(proj.Sigma, dtype=np.float32).astype(np.float64)
    return (U * sig[None, :]) @ V.T


def silu(a):
    """silu(a) = a / (1 + exp(-a))."""
    return a / (1.0 + np.exp(-a))


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------
class _WeightCache:
    def __init__(self, layer):
        self.layer = layer
        self.cache = {}

    def get(self, p: int, e: int) -> np.ndarray:
        key = (p, e)
        if key not in self.cache:
            self.cache[key] = expert_weight(self.layer.projs[p], e, self.layer.N)
        return self.cache[key]


def _shared_expert(layer, xt: np.ndarray) -> np.ndarray:
    sh = layer.shared
    Wg = widen_bf16(sh["gate"])
    Wu = widen_bf16(sh["up"])
    Wd = widen_bf16(sh["down"])
    return Wd @ (silu(Wg @ xt) * (Wu @ xt))


def forward(layer, x_bits, logits, tokens=None, return_h: bool = False):
    """Literal per-token forward of the TileQ MoE layer in float64.

    LINEAR:  out_t = sum_j w_j W_{e_j} x_t
    SWIGLU:  out_t = sum_j w_j W^down_{e_j} (silu(W^gate_{e_j} x_t) * (W^up_{e_j} x_t))
             (+ the shared expert's dense SwiGLU with weight 1, if present)
    ``tokens`` restricts the loop to a subset of token indices (routing is
    still computed for those tokens only, from their own logits).
    Returns out float64 [len(tokens), d_out] (and h [len(tokens), k, d_ff]).
    """
    x = widen_bf16(x_bits)
    lg = np.asarray(logits, dtype=np.float32)
    T = x.shape[0]
    toks = list(range(T)) if tokens is None else [int(t) for t in tokens]
    idx, w = route(lg[toks], layer.top_k, getattr(layer, "route_mode", 0) == 1)
    cache = _WeightCache(layer)
    d_y = layer.projs[-1].d_out
    out = np.zeros((len(toks), d_y), dtype=np.float64)
    hs = [] if return_h else None
    for i, t in enumerate(toks):
        xt = x[t]
        hrow = []
        for j in range(layer.top_k):
            e = int(idx[i, j])
            if layer.kind == 0:
                y = cache.get(0, e) @ xt
            else:
                h = silu(cache.get(0, e) @ xt) * (cache.get(1, e) @ xt)
                hrow.append(h)
                y = cache.get(2, e) @ h
            out[i] += w[i, j] * y
        if layer.shared is not None:
            out[i] += _shared_expert(layer, xt)
        if return_h:
            hs.append(hrow)
    if return_h:
        return out, np.array(hs)
    return out


def forward_batched(layer, x_bits, logits, tokens=None):
    """Whole-batch forward, one dense float64 matmul per (expert, projection).

    Same definition as ``forward``; the tokens routed to an expert are stacked
    so each reconstructed W_e is applied once, and only one W_e is held at a
    time.  ``tokens`` restricts the batch to a subset of token indices (their
    own logits route them), returned in the given order.  Used for full-size
    outputs.
    """
    x = widen_bf16(x_bits)
    lg = np.asarray(logits, dtype=np.float32)
    if tokens is not None:
        sel = np.asarray(tokens, dtype=np.int64)
        x = x[sel]
        lg = lg[sel]
    T = x.shape[0]
    idx, w = route(lg, layer.top_k, getattr(layer, "route_mode", 0) == 1)
    d_y = layer.projs[-1].d_out
    out = np.zeros((T, d_y), dtype=np.float64)
    for e in range(layer.K):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        Xe = x[rows]
        if layer.kind == 0:
            Y = Xe @ expert_weight(layer.projs[0], e, layer.N).T
        else:
            G = Xe @ expert_weight(layer.projs[0], e, layer.N).T
            Uu = Xe @ expert_weight(layer.projs[1], e, layer.N).T
            H = silu(G) * Uu
            del G, Uu
            Y = H @ expert_weight(layer.projs[2], e, layer.N).T
        np.add.at(out, rows, w[rows, slots][:, None] * Y)
    if layer.shared is not None:
        sh = layer.shared
        Wg, Wu, Wd = widen_bf16(sh["gate"]), widen_bf16(sh["up"]), widen_bf16(sh["down"])
        out += (silu(x @ Wg.T) * (x @ Wu.T)) @ Wd.T
    return out


# ---------------------------------------------------------------------------
# storage closed forms (memory claim of the paper's experiments section)
# ---------------------------------------------------------------------------
def lowrank_bytes_tiled(M, N, d_out, d_in, r, elem_bytes=2):
    """Bytes of the shared factors of one projection: U [M*d_out, r] + V [N*d_in, r]."""
    return elem_bytes * r * (M * d_out + N * d_in)


def lowrank_bytes_per_expert(K, d_out, d_in, r, elem_bytes=2):
    """Bytes of independent per-expert factors: K * r * (d_out + d_in)."""
    return elem_bytes * K * r * (d_out + d_in)
