"""The C ABI without a GPU: the library loads, exports every declared symbol,
the ctypes structs match the C layout, and host-side validation rejects bad
arguments before anything is launched."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tileq.h")


@pytest.fixture(scope="module")
def L():
    from tiled_rank_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from tiled_rank_b200 import build
        build.build()
    return _lib


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|tileq_status)\s*(tileq_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    fns = declared_functions()
    assert "tileq_moe_forward" in fns and "tileq_route" in fns and "tileq_pack" in fns
    assert len(fns) >= 11


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(L.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(L.EXPORTS) == set(declared_functions())
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tileq_\w+)", out))
    assert set(declared_functions()) <= exported


def test_struct_layout_matches_c(L, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "tileq.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n",'
                   'sizeof(tileq_proj), offsetof(tileq_proj, grid_assign), offsetof(tileq_proj, zeros),'
                   'offsetof(tileq_proj, bits), offsetof(tileq_proj, codes_hi),'
                   'sizeof(tileq_layer), offsetof(tileq_layer, proj), offsetof(tileq_layer, shared_d_ff),'
                   'offsetof(tileq_layer, shared_w), offsetof(tileq_layer, route_mode), sizeof(tileq_route_out), sizeof(tileq_per_expert_lr));'
                   'return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(L.tileq_proj), L.tileq_proj.grid_assign.offset, L.tileq_proj.zeros.offset,
            L.tileq_proj.bits.offset, L.tileq_proj.codes_hi.offset,
            ctypes.sizeof(L.tileq_layer), L.tileq_layer.proj.offset, L.tileq_layer.shared_d_ff.offset,
            L.tileq_layer.shared_w.offset, L.tileq_layer.route_mode.offset, ctypes.sizeof(L.tileq_route_out),
            ctypes.sizeof(L.tileq_per_expert_lr)]
    assert got == want


def _host_layer(L, cfg, rank=None, grids=None):
    """A tileq_layer with shapes and host grids only (device pointers left NULL)."""
    layer = synth.make_layer(cfg, seed=0, rank=rank) if not isinstance(cfg, synth.Layer) else cfg
    c = L.tileq_layer()
    c.kind, c.K, c.M, c.N = layer.kind, layer.K, layer.M, layer.N
    c.d_model, c.d_ff = layer.d_model, layer.d_ff
    keep = []
    for i, p in enumerate(layer.projs):
        g = np.ascontiguousarray(p.grid_assign if grids is None else grids[i], dtype=np.int32)
        keep.append(g)
        c.proj[i].d_in, c.proj[i].d_out, c.proj[i].rank, c.proj[i].group = p.d_in, p.d_out, p.rank, p.group
        c.proj[i].grid_assign = g.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    c.shared_d_ff = layer.shared_d_ff
    c._keep = keep
    return c, layer


def test_packed_size_closed_form(L):
    """Packed bytes: codes 2 bits/weight in two layouts (tcgen05 rows, warp-MMA
    fragments), one u32 (scale, zero) per row and group, U blocks and V_n^T
    blocks in fp16 with rows padded to multiples of 128 (V_n^T twice: fragment
    order and row-major), and Sigma repeated per grid column in fp32."""
    c, layer = _host_layer(L, 0)
    p = layer.projs[0]
    pad = lambda v: (v + 127) // 128 * 128  # noqa: E731
    K, M, N = layer.K, layer.M, layer.N
    expect = 0
    for nbytes in (K * pad(p.d_out) * p.d_in // 4, K * pad(p.d_out) * p.d_in // 4,
                   K * pad(p.d_out) * (p.d_in // p.group) * 4,
                   M * pad(p.d_out) * p.rank * 2, N * pad(p.rank) * pad(p.d_in) * 2,
                   N * pad(p.rank) * 4, N * pad(p.rank) * p.d_in * 2):
        expect += (nbytes + 255) // 256 * 256
    assert L.tileq_packed_size(c) == expect


def test_workspace_size_grows_with_T(L):
    c, _ = _host_layer(L, 0)
    a = L.tileq_workspace_size(c, 1, 2)
    b = L.tileq_workspace_size(c, 64, 2)
    assert 0 < a < b


def test_validation_rejects_bad_layers(L):
    c, layer = _host_layer(L, 0)
    bad_grid = np.array([0, 1, 1, 3], dtype=np.int32)            # not injective
    c2, _ = _host_layer(L, 0, grids=[bad_grid])
    with pytest.raises(L.TileQError) as e:
        L.tileq_packed_size(c2)
    assert e.value.status == L.TILEQ_ERR_INVALID_ARG
    c3, _ = _host_layer(L, 0, grids=[np.array([0, 1, 2, 4], dtype=np.int32)])  # cell out of grid
    with pytest.raises(L.TileQError):
        L.tileq_workspace_size(c3, 4, 2)
    c.proj[0].d_in = 96                                           # not a multiple of 128
    with pytest.raises(L.TileQError) as e:
        L.tileq_packed_size(c)
    assert e.value.status == L.TILEQ_ERR_UNSUPPORTED
    c.proj[0].d_in = 256
    with pytest.raises(L.TileQError) as e:
        L.tileq_workspace_size(c, 4, 5)                           # top_k > K
    assert e.value.status == L.TILEQ_ERR_INVALID_ARG
    c4, _ = _host_layer(L, 0)
    c4.route_mode = L.TILEQ_ROUTE_FULL_SOFTMAX
    assert L.tileq_packed_size(c4) == L.tileq_packed_size(_host_layer(L, 0)[0])
    c4.route_mode = 2                                             # no such routing
    with pytest.raises(L.TileQError) as e:
        L.tileq_packed_size(c4)
    assert e.value.status == L.TILEQ_ERR_INVALID_ARG


def test_forward_validation_before_launch(L):
    """Errors are returned before any CUDA call: no device is needed."""
    c, _ = _host_layer(L, 0)
    lib = L.lib()
    fake = ctypes.c_void_p(0x10000)
    # NULL packed/x/logits/out/ws -> INVALID_ARG (device pointers of the layer unset too)
    st = lib.tileq_moe_forward(ctypes.byref(c), None, None, 4, None, 2, None, None, 0, None, None)
    assert st == L.TILEQ_ERR_INVALID_ARG
    # T == 0 enqueues nothing and succeeds even with NULL pointers... once the layer is complete
    for i in range(1):
        c.proj[i].codes = c.proj[i].scales = c.proj[i].zeros = fake
        c.proj[i].U = c.proj[i].V = c.proj[i].Sigma = fake
    st = lib.tileq_moe_forward(ctypes.byref(c), None, None, 0, None, 2, None, None, 0, None, None)
    assert st == L.TILEQ_OK
    # too small a workspace
    st = lib.tileq_moe_forward(ctypes.byref(c), fake, fake, 4, fake, 2, fake, fake, 16, None, None)
    assert st == L.TILEQ_ERR_WORKSPACE
    # bad top_k
    st = lib.tileq_moe_forward(ctypes.byref(c), fake, fake, 4, fake, 0, fake, fake, 1 << 30, None, None)
    assert st == L.TILEQ_ERR_INVALID_ARG
    r = L.tileq_route_out()
    st = lib.tileq_route(fake, 4, 4, 2, ctypes.byref(r), fake, 1 << 20, None)
    assert st == L.TILEQ_ERR_INVALID_ARG                          # route outputs missing
    assert L.status_string(L.TILEQ_ERR_TIMEOUT) == "TILEQ_ERR_TIMEOUT"
    assert L.status_string(L.TILEQ_ERR_RANGE) == "TILEQ_ERR_RANGE"


def test_route_static_validation_before_launch(L):
    """Too many pairs is rejected on the host, before any device work."""
    fake = L.tileq_route_out(1, 1, 1, 1)  # never dereferenced: validation fails first
    for T, K, k, want in [(4097, 8, 2, L.TILEQ_ERR_UNSUPPORTED), (16, 8, 9, L.TILEQ_ERR_INVALID_ARG),
                          (16, 65, 2, L.TILEQ_ERR_INVALID_ARG)]:
        st = L.lib().tileq_route_static(1, T, K, k, ctypes.byref(fake), None)
        assert st == want, (T, K, k, st)


def test_route_static_scratch_covers_max_pairs(L):
    """The routing-only workspace at TILEQ_ROUTE_STATIC_MAX_PAIRS fits the 6 MiB static scratch."""
    max_pairs = 8192
    hdr = open(os.path.join(ROOT, "include", "tileq.h")).read()
    assert f"#define TILEQ_ROUTE_STATIC_MAX_PAIRS {max_pairs}" in hdr
    for K in (2, 8, 60, 64):
        grid = (ctypes.c_int32 * K)(*range(K))
        c = L.tileq_layer()
        c.kind, c.K, c.M, c.N = L.TILEQ_LINEAR, K, K, 1
        c.proj[0].d_in, c.proj[0].d_out, c.proj[0].group = 128, 16, 128
        c.proj[0].grid_assign = ctypes.cast(grid, ctypes.POINTER(ctypes.c_int32))
        for k in (1, 2, 4, 8):
            if k <= K:
                assert L.tileq_workspace_size(c, max_pairs // k, k) <= 6 << 20, (K, k)


def test_wbig_layout_matches_c(L, tmp_path):
    src = tmp_path / "wbig.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "tileq.h"\n'
                   'int main(void){printf("%zu %zu %zu %d\\n", sizeof(tileq_wbig), offsetof(tileq_wbig, w),'
                   'offsetof(tileq_wbig, grid_assign), TILEQ_SKETCH_MAX_L); return 0;}\n')
    exe = tmp_path / "wbig"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    assert got == [ctypes.sizeof(L.tileq_wbig), L.tileq_wbig.w.offset, L.tileq_wbig.grid_assign.offset,
                   L.TILEQ_SKETCH_MAX_L]


def _wbig(L, M, N, d_out, d_in, grid=None):
    K = M * N
    g = np.ascontiguousarray(np.arange(K) if grid is None else grid, dtype=np.int32)
    w = L.tileq_wbig()
    w.K, w.M, w.N, w.d_out, w.d_in = K, M, N, d_out, d_in
    w.w = 16  # never dereferenced by the host checks
    w.grid_assign = g.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    w._keep = g
    return w


def test_sketch_workspace_and_validation(L):
    w = _wbig(L, 2, 4, 256, 128)
    n = L.tileq_sketch_workspace_size(w, 24, 16)
    R, C, l, r = 2 * 256, 4 * 128, 24, 16
    assert n >= 8 * 256 * 128 * 2 + (2 * R * l + 2 * C * l) * 4 + 2 * l * R * 2 + 16 * l * l * 8
    with pytest.raises(L.TileQError):
        L.tileq_sketch_workspace_size(w, 23, 16)          # odd sketch width
    with pytest.raises(L.TileQError):
        L.tileq_sketch_workspace_size(w, L.TILEQ_SKETCH_MAX_L + 2, 16)
    with pytest.raises(L.TileQError):
        L.tileq_sketch_workspace_size(w, 24, 25)          # rank above the sketch width
    with pytest.raises(L.TileQError):
        L.tileq_sketch_workspace_size(_wbig(L, 2, 2, 128, 128, grid=[0, 1, 1, 3]), 8, 4)  # not a bijection
    with pytest.raises(L.TileQError):
        L.tileq_sketch_workspace_size(_wbig(L, 2, 2, 192, 128), 8, 4)  # d_out not a multiple of 128
    bad = _wbig(L, 2, 2, 128, 128)
    bad.K = 3
    with pytest.raises(L.TileQError):
        L.tileq_sketch_workspace_size(bad, 8, 4)          # K != M*N


def test_place_layout_matches_c(L, tmp_path):
    src = tmp_path / "place.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "tileq.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu %d\\n", sizeof(tileq_place_in),'
                   'offsetof(tileq_place_in, u), offsetof(tileq_place_in, max_iter), sizeof(tileq_place_out),'
                   'offsetof(tileq_place_out, ideal), offsetof(tileq_place_out, iterations),'
                   'TILEQ_PLACE_MAX_R0); return 0;}\n')
    exe = tmp_path / "place"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    assert got == [ctypes.sizeof(L.tileq_place_in), L.tileq_place_in.u.offset, L.tileq_place_in.max_iter.offset,
                   ctypes.sizeof(L.tileq_place_out), L.tileq_place_out.ideal.offset,
                   L.tileq_place_out.iterations.offset, L.TILEQ_PLACE_MAX_R0]


def _place(L, K, M, N, d_u=64, d_v=32, r0=8, max_iter=100):
    c = L.tileq_place_in()
    c.K, c.M, c.N, c.d_u, c.d_v, c.r0, c.max_iter = K, M, N, d_u, d_v, r0, max_iter
    c.u = c.v = 16   # never dereferenced by the host checks
    return c


def test_place_workspace_and_validation(L):
    """Errors are returned on the host, before any launch (no device needed)."""
    n = L.tileq_place_workspace_size(_place(L, 64, 8, 8, r0=16))
    assert n >= 2 * 148 * 64 * 64 * 8 + 2 * 64 * 64 * 8 + 2 * 64 * 16 * 12
    for bad, want in [((65, 8, 9), L.TILEQ_ERR_UNSUPPORTED), ((9, 2, 4), L.TILEQ_ERR_INVALID_ARG),
                      ((4, 2, 65), L.TILEQ_ERR_UNSUPPORTED), ((0, 2, 2), L.TILEQ_ERR_INVALID_ARG)]:
        with pytest.raises(L.TileQError) as e:
            L.tileq_place_workspace_size(_place(L, *bad))
        assert e.value.status == want, bad
    for kw, want in [(dict(r0=257), L.TILEQ_ERR_UNSUPPORTED), (dict(r0=0), L.TILEQ_ERR_INVALID_ARG),
                     (dict(max_iter=0), L.TILEQ_ERR_INVALID_ARG), (dict(d_v=0), L.TILEQ_ERR_INVALID_ARG),
                     (dict(max_iter=65537), L.TILEQ_ERR_UNSUPPORTED)]:
        with pytest.raises(L.TileQError) as e:
            L.tileq_place_workspace_size(_place(L, 4, 2, 2, **kw))
        assert e.value.status == want, kw
    out = L.tileq_place_out(None, None, None)      # grid_assign is required
    st = L.lib().tileq_place_experts(ctypes.byref(_place(L, 4, 2, 2)), ctypes.byref(out), 16, 1 << 30, None)
    assert st == L.TILEQ_ERR_INVALID_ARG
    out = L.tileq_place_out(16, None, None)
    st = L.lib().tileq_place_experts(ctypes.byref(_place(L, 4, 2, 2)), ctypes.byref(out), 16, 8, None)
    assert st == L.TILEQ_ERR_WORKSPACE


def test_3bit_validation_and_packed_size(L):
    """3-bit projections: bits in {0, 2, 3}; the packed copy adds the high-bit
    plane beside each of the two code layouts (1 bit/weight each)."""
    c2, layer = _host_layer(L, 0)
    n2 = L.tileq_packed_size(c2)
    cfg3 = synth.Config(**{**synth.CONFIGS[0].__dict__, "bits": 3})
    c3, _ = _host_layer(L, cfg3)
    for i in range(1):
        c3.proj[i].bits = 3
    n3 = L.tileq_packed_size(c3)
    p = layer.projs[0]
    assert n3 - n2 == 2 * (layer.K * p.d_out * p.d_in // 8)
    c3.proj[0].bits = 4
    with pytest.raises(L.TileQError) as e:
        L.tileq_packed_size(c3)
    assert e.value.status == L.TILEQ_ERR_UNSUPPORTED
    # gate and up share one residual kernel: their bits must agree
    cs, _ = _host_layer(L, synth.tiny_config(K=4, M=2, N=2, d_model=128, d_ff=128, rank=16, group=64))
    cs.proj[0].bits = 3
    with pytest.raises(L.TileQError) as e:
        L.tileq_packed_size(cs)
    assert e.value.status == L.TILEQ_ERR_UNSUPPORTED
    cs.proj[1].bits = 3
    assert L.tileq_packed_size(cs) > 0
