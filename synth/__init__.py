"""Seeded synthetic TileQ MoE layers and inputs.

This module only draws random numbers and lays them out in the stored TileQ
format; it holds none of the method's arithmetic (no dequantisation, no
routing, no products).  Both the fp64 oracle and the CUDA path read what it
produces, so that they see the very same bytes.

Stored format of one projection (d_out x d_in) of a layer whose K experts sit
on an M x N grid (TileQ paper, "2D-Tiling Structured Low-Rank Quantization"):

* ``grid_assign`` int32 [K]: cell ``m*N + n`` of expert k, injective.
* ``U`` bf16 bits (uint16) [M*d_out, r]: block m = rows m*d_out .. (m+1)*d_out-1
  is the shared left (output-space) factor of grid row m.
* ``Sigma`` fp32 [r]: the shared diagonal.
* ``V`` bf16 bits (uint16) [N*d_in, r]: block n = the shared right (input-space)
  factor of grid column n.
* ``codes`` uint32 [K, d_out, d_in/16]: 2-bit residual codes, element j of a
  word at bits 2*(j%16).
* ``scales`` fp16 [K, d_out, d_in/g]: one scale per group of g inputs.
* ``zeros`` uint8 [K, d_out, ceil(d_in/g/4)]: 2-bit zero points, group j at
  bits 2*(j%4) of byte j//4; unused high fields are 0.

The residual dequantises as w = s * (q - z).

Draw recipe (seeded, numpy ``default_rng``):

* weights come from ``default_rng([seed, 1])`` in the order: for each
  projection U, V, codes, scales, zeros, grid permutation; then the Zipf
  permutation (if any); then the shared expert.  They do not depend on the
  batch size, so one packed layer serves every batch of a configuration.
* inputs come from ``default_rng([seed, 2, T])``: router logits, then x.
* U ~ N(0, 1/d_out) (std 1/sqrt(d_out)), V ~ N(0, 1/d_in): unit-norm-like
  columns as singular vectors have; Sigma_i = 1/(1+i).
* codes and zero points uniform in {0..3}: drawn as uniform random uint32
  words (resp. bytes), each 2-bit field of which is uniform.
* scales ~ U[0.005, 0.02] rounded to fp16; x ~ N(0,1) rounded to bf16 (RNE).
* logits ~ N(0, sigma^2) fp32, plus for the Zipf configuration a per-expert
  bias b_k = -s * ln(pi_k) with pi a seeded permutation of 1..K.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

LINEAR = 0
SWIGLU = 1


# --------------------------------------------------------------------------
# bf16 bit helpers (storage only; no method arithmetic)
# --------------------------------------------------------------------------
def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (round-to-nearest-even), returned as uint16 bits."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bits (uint16) to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# layer containers
# --------------------------------------------------------------------------
@dataclasses.dataclass
class Proj:
    d_in: int
    d_out: int
    rank: int
    group: int
    grid_assign: np.ndarray  # int32 [K]
    U: np.ndarray            # uint16 (bf16 bits) [M*d_out, r]
    Sigma: np.ndarray        # float32 [r]
    V: np.ndarray            # uint16 (bf16 bits) [N*d_in, r]
    codes: np.ndarray        # uint32 [K, d_out, d_in/16]
    scales: np.ndarray       # float16 [K, d_out, d_in/g]
    zeros: np.ndarray        # uint8 [K, d_out, ceil(G/4)] (2-bit) or [K, d_out, ceil(G/2)] (3-bit)
    bits: int = 2            # 2 or 3 (3: q = codes + 4 * bit of codes_hi)
    codes_hi: Optional[np.ndarray] = None  # 3-bit: uint32 [K, d_out, d_in/32], element j at bit j%32

    @property
    def n_groups(self) -> int:
        return self.d_in // self.group


@dataclasses.dataclass
class Layer:
    kind: int                # LINEAR or SWIGLU
    K: int
    M: int
    N: int
    d_model: int             # SWIGLU: model width; LINEAR: d_in of the single projection
    d_ff: int                # SWIGLU: expert hidden width; LINEAR: d_out
    top_k: int
    projs: list              # LINEAR: [proj]; SWIGLU: [gate, up, down]
    shared: Optional[dict] = None  # {"gate","up": uint16 [Fs, D], "down": uint16 [D, Fs]}
    route_mode: int = 0      # 0: softmax over the chosen logits; 1: chosen entries of the softmax over all K

    @property
    def d_x(self) -> int:
        return self.projs[0].d_in

    @property
    def d_y(self) -> int:
        return self.projs[-1].d_out

    @property
    def shared_d_ff(self) -> int:
        return 0 if self.shared is None else int(self.shared["gate"].shape[0])


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    kind: int
    K: int
    M: int
    N: int
    d_model: int
    d_ff: int
    rank: int
    group: int
    top_k: int
    batches: tuple
    logit_std: float = 1.0
    zipf_s: float = 0.0
    shared_d_ff: int = 0
    per_expert_layout: bool = False
    bits: int = 2


CONFIGS = {
    # single TileQ linear: 4 experts on 2x2, 256 -> 512, r=16, groups of 64, top-2
    0: Config("tiny-linear-4e-2x2", LINEAR, 4, 2, 2, 256, 512, 16, 64, 2, (64,)),
    # Mixtral-8x7B-shaped layer on a 2x4 grid, decode batches
    1: Config("mixtral8x7b-2x4-decode", SWIGLU, 8, 2, 4, 4096, 14336, 128, 128, 2, (1, 8, 32, 64)),
    # same layer, prefill with logits N(0, 1.5^2)
    2: Config("mixtral8x7b-2x4-prefill", SWIGLU, 8, 2, 4, 4096, 14336, 128, 128, 2, (4096,),
              logit_std=1.5),
    # Qwen1.5-MoE-A2.7B-shaped: 60 experts on 6x10, top-4, Zipf bias, shared expert
    3: Config("qwen15moe-6x10", SWIGLU, 60, 6, 10, 2048, 1408, 64, 128, 4, (1, 16, 256, 2048),
              zipf_s=1.1, shared_d_ff=5632),
    # fine-grained 64 experts on 8x8, top-8, 16k tokens, plus a per-expert layout
    4: Config("finegrained-64e-8x8", SWIGLU, 64, 8, 8, 4096, 1536, 128, 128, 8, (16384,),
              per_expert_layout=True),
}


def proj_shapes(kind: int, d_model: int, d_ff: int):
    """(d_in, d_out) of each projection."""
    if kind == LINEAR:
        return [(d_model, d_ff)]
    return [(d_model, d_ff), (d_model, d_ff), (d_ff, d_model)]


def _make_proj(rng, K, M, N, d_in, d_out, rank, group, bits=2) -> Proj:
    if d_in % 16 or d_in % group:
        raise ValueError("d_in must be a multiple of 16 and of the group size")
    G = d_in // group
    U = to_bf16_bits(rng.standard_normal((M * d_out, rank), dtype=np.float32) / np.sqrt(d_out))
    V = to_bf16_bits(rng.standard_normal((N * d_in, rank), dtype=np.float32) / np.sqrt(d_in))
    codes = rng.integers(0, 2**32, size=(K, d_out, d_in // 16), dtype=np.uint32)
    scales = rng.uniform(0.005, 0.02, size=(K, d_out, G)).astype(np.float16)
    zb = (G + 3) // 4
    zeros = rng.integers(0, 256, size=(K, d_out, zb), dtype=np.uint8)
    if G % 4:
        # clear the 2-bit fields past the last group in the final byte
        keep = (1 << (2 * (G % 4))) - 1
        zeros[..., -1] &= np.uint8(keep)
    grid = rng.permutation(M * N)[:K].astype(np.int32)
    sigma = (1.0 / (1.0 + np.arange(rank, dtype=np.float64))).astype(np.float32)
    if bits != 3:
        return Proj(d_in, d_out, rank, group, grid, U, sigma, V, codes, scales, zeros)
    # 3-bit: a high-bit plane and zero points 0..7, two per byte (drawn after the
    # 2-bit arrays, so the other draws of the layer are unchanged)
    codes_hi = rng.integers(0, 2**32, size=(K, d_out, d_in // 32), dtype=np.uint32)
    z3 = rng.integers(0, 8, size=(K, d_out, G), dtype=np.uint8)
    if G % 2:
        z3 = np.concatenate([z3, np.zeros((K, d_out, 1), np.uint8)], axis=-1)
    zeros3 = (z3[..., 0::2] | (z3[..., 1::2] << 4)).astype(np.uint8)
    return Proj(d_in, d_out, rank, group, grid, U, sigma, V, codes, scales, zeros3, 3, codes_hi)


def make_layer(cfg: Config | int, seed: int = 0, rank: Optional[int] = None) -> Layer:
    """Draw the layer weights of a configuration (independent of the batch size).

    ``rank`` overrides the configured rank (e.g. 0 for the residual-only layer);
    the residual draws are unchanged by it only when it equals the configured rank.
    """
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    r = cfg.rank if rank is None else rank
    rng = np.random.default_rng([seed, 1])
    projs = [_make_proj(rng, cfg.K, cfg.M, cfg.N, di, do, r, cfg.group, cfg.bits)
             for (di, do) in proj_shapes(cfg.kind, cfg.d_model, cfg.d_ff)]
    shared = None
    if cfg.shared_d_ff:
        D, Fs = cfg.d_model, cfg.shared_d_ff
        shared = {
            "gate": to_bf16_bits(rng.standard_normal((Fs, D), dtype=np.float32) / np.sqrt(D)),
            "up": to_bf16_bits(rng.standard_normal((Fs, D), dtype=np.float32) / np.sqrt(D)),
            "down": to_bf16_bits(rng.standard_normal((D, Fs), dtype=np.float32) / np.sqrt(Fs)),
        }
    return Layer(cfg.kind, cfg.K, cfg.M, cfg.N, cfg.d_model, cfg.d_ff, cfg.top_k, projs, shared)


def zipf_bias(cfg: Config, seed: int = 0) -> np.ndarray:
    """Per-expert router bias -s*ln(pi_k), pi a seeded permutation of 1..K (zeros if s=0)."""
    if not cfg.zipf_s:
        return np.zeros(cfg.K, dtype=np.float32)
    rng = np.random.default_rng([seed, 3])
    pi = rng.permutation(cfg.K) + 1
    return (-cfg.zipf_s * np.log(pi)).astype(np.float32)


def make_inputs(cfg: Config | int, T: int, seed: int = 0):
    """Router logits fp32 [T, K] and x bf16 bits [T, d_in] for a batch of T tokens."""
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    rng = np.random.default_rng([seed, 2, T])
    logits = (rng.standard_normal((T, cfg.K), dtype=np.float32) * np.float32(cfg.logit_std))
    logits = (logits + zipf_bias(cfg, seed)[None, :]).astype(np.float32)
    d_in = proj_shapes(cfg.kind, cfg.d_model, cfg.d_ff)[0][0]
    x = to_bf16_bits(rng.standard_normal((T, d_in), dtype=np.float32))
    return logits, x


def per_expert_lowrank(layer: Layer, p: Proj):
    """Copy the shared blocks into an independent per-expert layout.

    Returns U_pe uint16 [K, d_out, r] and V_pe uint16 [K, d_in, r] with
    U_pe[k] = U block of expert k's grid row and V_pe[k] = V block of its
    grid column (pure data movement: the effective weights are unchanged).
    """
    K, N = layer.K, layer.N
    U_pe = np.empty((K, p.d_out, p.rank), dtype=np.uint16)
    V_pe = np.empty((K, p.d_in, p.rank), dtype=np.uint16)
    for k in range(K):
        m, n = divmod(int(p.grid_assign[k]), N)
        U_pe[k] = p.U[m * p.d_out:(m + 1) * p.d_out]
        V_pe[k] = p.V[n * p.d_in:(n + 1) * p.d_in]
    return U_pe, V_pe


def tiny_config(kind=SWIGLU, K=4, M=2, N=2, d_model=64, d_ff=128, rank=8, group=32, top_k=2,
                shared_d_ff=0, zipf_s=0.0, logit_std=1.0, bits=2) -> Config:
    """A small configuration for tests (oracle runs it in milliseconds)."""
    return Config(f"tiny-{kind}-{K}e", kind, K, M, N, d_model, d_ff, rank, group, top_k, (16,),
                  logit_std=logit_std, zipf_s=zipf_s, shared_d_ff=shared_d_ff, bits=bits)


def planted_factors(K: int, M: int, N: int, d_u: int, d_v: int, r0: int, noise: float = 0.05,
                    seed: int = 0):
    """Per-expert rank-r0 factors with a planted grid structure.

    A seeded injective expert -> cell map (the planted grid_assign) puts expert
    k in cell (m_k, n_k); its left factor is an orthonormal basis of
    A_{m_k} + noise * G_k and its right factor one of B_{n_k} + noise * H_k
    (A_m [d_u, r0], B_n [d_v, r0], G_k, H_k standard normal), each column then
    multiplied by a random sign, as an SVD would return it.  Experts of one
    grid row thus have nearby left subspaces, experts of one column nearby
    right subspaces.  Returns (u fp32 [K, d_u, r0], v fp32 [K, d_v, r0],
    planted grid_assign int32 [K]).
    """
    rng = np.random.default_rng([seed, 5])
    cells = rng.permutation(M * N)[:K].astype(np.int32)
    A = rng.standard_normal((M, d_u, r0))
    B = rng.standard_normal((N, d_v, r0))
    u = np.empty((K, d_u, r0), dtype=np.float32)
    v = np.empty((K, d_v, r0), dtype=np.float32)
    for k in range(K):
        m, n = divmod(int(cells[k]), N)
        qu, _ = np.linalg.qr(A[m] + noise * rng.standard_normal((d_u, r0)))
        qv, _ = np.linalg.qr(B[n] + noise * rng.standard_normal((d_v, r0)))
        u[k] = qu * rng.choice([-1.0, 1.0], size=r0)[None, :]
        v[k] = qv * rng.choice([-1.0, 1.0], size=r0)[None, :]
    return u, v, cells
