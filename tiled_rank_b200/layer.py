"""Device-resident TileQ layer: uploads the stored-format arrays, packs them once,
and calls the C ABI.  PyTorch provides device memory and streams only.

``layer`` is any object with the attributes of a stored TileQ layer: kind, K,
M, N, d_model, d_ff, top_k, projs (each with d_in, d_out, rank, group,
grid_assign, U, Sigma, V, codes, scales, zeros as numpy arrays; U/V as bf16
bit patterns in uint16) and shared (None or dict of gate/up/down bf16 bits).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _lib as L


def _dev(a: np.ndarray, device, dtype=None):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:            # bf16 bit patterns
        t = torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    elif a.dtype == np.uint32:
        t = torch.from_numpy(a.view(np.int32)).to(device)
    else:
        t = torch.from_numpy(a).to(device)
    return t if dtype is None else t.view(dtype)


class DeviceLayer:
    def __init__(self, layer, device="cuda", stream=None, per_expert=None):
        import torch
        self.device = torch.device(device)
        self.kind = int(layer.kind)
        self.K, self.M, self.N = int(layer.K), int(layer.M), int(layer.N)
        self.top_k = int(layer.top_k)
        self.d_x = int(layer.projs[0].d_in)
        self.d_y = int(layer.projs[-1].d_out)
        self._keep = []
        c = L.tileq_layer()
        c.kind = self.kind
        c.K, c.M, c.N = self.K, self.M, self.N
        c.d_model = int(layer.d_model)
        c.d_ff = int(layer.d_ff)
        for i, p in enumerate(layer.projs):
            cp = c.proj[i]
            cp.d_in, cp.d_out, cp.rank, cp.group = int(p.d_in), int(p.d_out), int(p.rank), int(p.group)
            grid = np.ascontiguousarray(p.grid_assign, dtype=np.int32)
            self._keep.append(grid)
            cp.grid_assign = grid.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
            tens = {
                "codes": _dev(p.codes, self.device),
                "scales": _dev(p.scales, self.device),
                "zeros": _dev(p.zeros, self.device),
            }
            bits = int(getattr(p, "bits", 2))
            if bits == 3:
                tens["codes_hi"] = _dev(p.codes_hi, self.device)
            if p.rank > 0:
                tens["U"] = _dev(p.U, self.device)
                tens["V"] = _dev(p.V, self.device)
                tens["Sigma"] = _dev(np.asarray(p.Sigma, np.float32), self.device)
            self._keep.append(tens)
            cp.codes = L._ptr(tens["codes"])
            cp.scales = L._ptr(tens["scales"])
            cp.zeros = L._ptr(tens["zeros"])
            cp.bits = bits
            cp.codes_hi = L._ptr(tens.get("codes_hi"))
            cp.U = L._ptr(tens.get("U"))
            cp.V = L._ptr(tens.get("V"))
            cp.Sigma = L._ptr(tens.get("Sigma"))
        c.route_mode = int(getattr(layer, "route_mode", 0))
        c.shared_d_ff = 0
        if layer.shared is not None:
            c.shared_d_ff = int(layer.shared["gate"].shape[0])
            sh = [_dev(layer.shared[k], self.device) for k in ("gate", "up", "down")]
            self._keep.append(sh)
            for i in range(3):
                c.shared_w[i] = L._ptr(sh[i])
        self.c = c
        self.packed = torch.empty(L.tileq_packed_size(c), dtype=torch.uint8, device=self.device)
        L.tileq_pack(c, self.packed, stream)
        self.packed_pe = None
        if per_expert is not None:
            self.set_per_expert(per_expert, stream)
        self._ws = {}

    def set_per_expert(self, per_expert, stream=None):
        """per_expert: list over projections of (U_pe, V_pe) bf16-bit numpy arrays."""
        import torch
        pe = L.tileq_per_expert_lr()
        tens = []
        for i, (Upe, Vpe) in enumerate(per_expert):
            u, v = _dev(Upe, self.device), _dev(Vpe, self.device)
            tens += [u, v]
            pe.U_pe[i] = L._ptr(u)
            pe.V_pe[i] = L._ptr(v)
        self.packed_pe = torch.empty(L.tileq_packed_per_expert_size(self.c), dtype=torch.uint8,
                                     device=self.device)
        L.tileq_pack_per_expert(self.c, pe, self.packed_pe, stream)
        # the unpacked per-expert arrays are only needed until packing completes
        torch.cuda.current_stream(self.device).synchronize()
        del tens

    def workspace(self, T: int, top_k: int = None):
        import torch
        top_k = self.top_k if top_k is None else top_k
        key = (T, top_k)
        if key not in self._ws:
            n = L.tileq_workspace_size(self.c, T, top_k)
            self._ws[key] = torch.zeros(n, dtype=torch.uint8, device=self.device)
        return self._ws[key]

    def forward(self, x, logits, top_k: int = None, out=None, ws=None, route=None, stream=None,
                unfused: bool = False):
        import torch
        top_k = self.top_k if top_k is None else top_k
        T = int(x.shape[0])
        if out is None:
            out = torch.empty((T, self.d_y), dtype=torch.bfloat16, device=self.device)
        if ws is None:
            ws = self.workspace(T, top_k)
        if unfused:
            L.tileq_moe_forward_unfused(self.c, self.packed, self.packed_pe, x, T, logits, top_k,
                                        out, ws, route, stream)
        else:
            L.tileq_moe_forward(self.c, self.packed, x, T, logits, top_k, out, ws, route, stream)
        return out

    def route_buffers(self, T: int, top_k: int = None):
        import torch
        top_k = self.top_k if top_k is None else top_k
        dev = self.device
        return {
            "topk_idx": torch.empty((T, top_k), dtype=torch.int32, device=dev),
            "topk_w": torch.empty((T, top_k), dtype=torch.float32, device=dev),
            "expert_offsets": torch.empty((self.K + 1,), dtype=torch.int32, device=dev),
            "sorted_pairs": torch.empty((T * top_k,), dtype=torch.int32, device=dev),
        }
