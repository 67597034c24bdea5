"""Algorithmic work of the TileQ MoE forward: bytes the method must touch and
FLOPs it must do, from the realised routing (host logic, no GPU).

Bytes: the stored residual (2- or 3-bit codes, fp16 group scales, 2- or 3-bit
zero points, the latter stored in 4-bit fields)
of every active expert once per projection; the shared low-rank blocks U_m of
active grid rows and V_n of active grid columns once; x, router logits and the
output once; the shared expert's bf16 weights.
FLOPs: residual 2*d_in*d_out per (token, expert) pair and projection; the
low-rank terms per the fused schedule of the TileQ paper, section 2.2 (the
input-side projection once per distinct (token, column), the output-side
product once per pair for gate/up and once per distinct (token, row) for the
combined projection); the shared expert 6*D*Fs per token.
"""
from __future__ import annotations

import math

import numpy as np


def residual_bytes(d_out: int, d_in: int, group: int, bits: int = 2) -> int:
    """Stored bytes of one expert's residual in one projection."""
    G = d_in // group
    if bits == 3:
        return d_out * d_in * 3 // 8 + d_out * G * 2 + d_out * math.ceil(G / 2)
    return d_out * d_in // 4 + d_out * G * 2 + d_out * math.ceil(G / 4)


def routing_sets(topk_idx: np.ndarray, grid_assign: np.ndarray, N: int):
    """Active experts, distinct (t, col), distinct (t, row) counts for one projection."""
    idx = np.asarray(topk_idx)
    cells = np.asarray(grid_assign)[idx]
    rows, cols = cells // N, cells % N
    T = idx.shape[0]
    tr = {(t, int(r)) for t in range(T) for r in rows[t]}
    tc = {(t, int(c)) for t in range(T) for c in cols[t]}
    return {
        "experts": np.unique(idx),
        "rows": np.unique(rows),
        "cols": np.unique(cols),
        "token_rows": len(tr),
        "token_cols": len(tc),
        "pairs": idx.size,
    }


def work(layer, topk_idx: np.ndarray) -> dict:
    """Per-stage and total algorithmic bytes / FLOPs of one forward.

    ``layer`` has the stored-layer attributes (kind, K, M, N, projs, shared).
    Returns {"stages": {name: {"bytes": b, "flops": f}}, "bytes": B, "flops": F}.
    """
    T = topk_idx.shape[0]
    stages = {}
    P = topk_idx.size
    d_x = layer.projs[0].d_in
    d_y = layer.projs[-1].d_out
    io = T * d_x * 2 + T * layer.K * 4 + T * d_y * 2
    sets = [routing_sets(topk_idx, p.grid_assign, layer.N) for p in layer.projs]

    def lr_v_bytes(p, s):
        return len(s["cols"]) * p.d_in * p.rank * 2

    def lr_u_bytes(p, s):
        return len(s["rows"]) * p.d_out * p.rank * 2

    def res(p, s):
        return len(s["experts"]) * residual_bytes(p.d_out, p.d_in, p.group, getattr(p, "bits", 2))

    if layer.kind == 0:
        p, s = layer.projs[0], sets[0]
        stages["zproj"] = {"bytes": lr_v_bytes(p, s), "flops": 2 * s["token_cols"] * p.d_in * p.rank}
        stages["residual"] = {
            "bytes": res(p, s) + lr_u_bytes(p, s),
            "flops": 2 * P * p.d_in * p.d_out + 2 * s["token_rows"] * p.d_out * p.rank,
        }
    else:
        g, u, d = layer.projs
        sg, su, sd = sets
        stages["zproj"] = {
            "bytes": lr_v_bytes(g, sg) + lr_v_bytes(u, su),
            "flops": 2 * (sg["token_cols"] * g.d_in * g.rank + su["token_cols"] * u.d_in * u.rank),
        }
        stages["gateup"] = {
            "bytes": res(g, sg) + res(u, su) + lr_u_bytes(g, sg) + lr_u_bytes(u, su),
            "flops": 2 * P * (g.d_in * g.d_out + u.d_in * u.d_out) + 2 * P * (g.d_out * g.rank + u.d_out * u.rank),
        }
        stages["zdown"] = {"bytes": lr_v_bytes(d, sd), "flops": 2 * P * d.d_in * d.rank}
        stages["residual"] = {
            "bytes": res(d, sd) + lr_u_bytes(d, sd),
            "flops": 2 * P * d.d_in * d.d_out + 2 * sd["token_rows"] * d.d_out * d.rank,
        }
        if layer.shared is not None:
            Fs = layer.shared["gate"].shape[0]
            D = layer.d_model
            stages["shared"] = {"bytes": 3 * D * Fs * 2, "flops": 6 * T * D * Fs}
    total_b = io + sum(v["bytes"] for v in stages.values())
    total_f = sum(v["flops"] for v in stages.values())
    return {"stages": stages, "bytes": total_b, "flops": total_f, "io_bytes": io}
