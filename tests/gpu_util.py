"""Helpers of the GPU parity tests (CUDA path vs the fp64 oracle)."""
from __future__ import annotations

import numpy as np

import oracle
import synth

# parity bar: max|gpu - ref| <= 1e-2 * max|ref| and sum|gpu - ref| / sum|ref| <= 2e-3
MAX_REL = 1e-2
MEAN_REL = 2e-3


def parity_stats(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    diff = np.abs(g - r)
    return {
        "max_abs": float(diff.max()) if diff.size else 0.0,
        "max_ref": float(np.abs(r).max()) if r.size else 0.0,
        "mean_rel": float(diff.sum() / max(np.abs(r).sum(), 1e-300)),
    }


def assert_parity(gpu, ref, what=""):
    s = parity_stats(gpu, ref)
    assert np.all(np.isfinite(np.asarray(gpu, dtype=np.float64))), f"{what}: non-finite output"
    assert s["max_abs"] <= MAX_REL * s["max_ref"], f"{what}: {s}"
    assert s["mean_rel"] <= MEAN_REL, f"{what}: {s}"
    return s


def to_numpy(t):
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def device_inputs(logits, x, device):
    import torch
    lg = torch.from_numpy(np.ascontiguousarray(logits)).to(device)
    xt = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)
    return lg, xt


def zero_residual(layer: synth.Layer, lr_gain: float = 1.0) -> synth.Layer:
    """Same layer with every residual code equal to its group's zero point (deq == 0).

    ``lr_gain`` (a power of two, exact in bf16) scales every U block, so that at
    full model widths the low-rank-only activations keep realistic magnitudes
    (unit-norm factors alone give outputs near 1e-6, below fp16's normal range).
    """
    projs = []
    for p in layer.projs:
        G = p.d_in // p.group
        zb = p.zeros
        if p.bits == 3:   # zero points 0..7, two per byte; q = low 2 bits + 4 * high bit
            z = np.stack([(zb[..., j // 2] >> (4 * (j % 2))) & 7 for j in range(G)], axis=-1)
        else:
            z = np.stack([(zb[..., j // 4] >> (2 * (j % 4))) & 3 for j in range(G)], axis=-1)
        words_per_group = p.group // 16
        zw = np.repeat((z & 3).astype(np.uint32), words_per_group, axis=-1) * np.uint32(0x55555555)
        extra = {}
        if p.bits == 3:
            hw = np.repeat((z >> 2).astype(np.uint32), p.group // 32, axis=-1) * np.uint32(0xFFFFFFFF)
            extra["codes_hi"] = np.ascontiguousarray(hw)
        U = p.U
        if lr_gain != 1.0 and p.rank > 0:
            U = synth.to_bf16_bits(synth.bf16_bits_to_f32(p.U) * np.float32(lr_gain))
        projs.append(synth.Proj(**{**p.__dict__, "codes": np.ascontiguousarray(zw), "U": U, **extra}))
    return synth.Layer(layer.kind, layer.K, layer.M, layer.N, layer.d_model, layer.d_ff,
                       layer.top_k, projs, layer.shared, layer.route_mode)


N_DENSE = 256


def dense_tokens(logits, top_k, K, seed, n_min=N_DENSE, route_mode=0):
    """Tokens to compare at full size: every token when T <= n_min; otherwise the
    tokens holding each active expert's first and last slot and the first and
    last slot of every 128-slot run of each expert (so every 128- and 256-item
    tile of the GEMMs, its ragged tail and every K split of it are covered),
    topped up with seeded random tokens to at least n_min."""
    T = logits.shape[0]
    if T <= n_min:
        return np.arange(T)
    idx, _ = oracle.route(logits, top_k, route_mode == 1)
    off, sp = oracle.permute(idx, K)
    slots = []
    for e in range(K):
        a, b = int(off[e]), int(off[e + 1])
        if b <= a:
            continue
        for t0 in range(a, b, 128):
            slots += [t0, min(t0 + 127, b - 1)]
    toks = set(int(sp[s]) // top_k for s in slots)
    rng = np.random.default_rng(seed)
    rest = rng.permutation(T)
    i = 0
    while len(toks) < n_min:
        toks.add(int(rest[i]))
        i += 1
    return np.array(sorted(toks))
