"""tileq_route_static: routing through the library's static scratch, checked
against tileq_route (caller workspace) on the same logits, two calls in a row.

Kept in a file of its own that sorts last, so that it runs both after the
other GPU tests and alone in a fresh process."""
import numpy as np
import pytest

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


def _route_bufs(torch, T, K, k, dev, fill):
    return {
        "topk_idx": torch.full((T, k), fill, dtype=torch.int32, device=dev),
        "topk_w": torch.full((T, k), float(fill), dtype=torch.float32, device=dev),
        "expert_offsets": torch.full((K + 1,), fill, dtype=torch.int32, device=dev),
        "sorted_pairs": torch.full((T * k,), fill, dtype=torch.int32, device=dev),
    }


@pytest.mark.parametrize("T,K,k", [(64, 8, 2), (4096, 8, 2), (1000, 60, 4), (1024, 64, 8)])
def test_route_static_matches_route(torch_cuda, T, K, k):
    torch = torch_cuda
    from tiled_rank_b200 import tileq_route, tileq_route_static
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(7 * T + K)
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device=dev)
    for call in range(2):
        # quantised logits: many exact ties between experts
        logits = (np.round(rng.standard_normal((T, K)) * 4) / 4).astype(np.float32)
        lg = torch.from_numpy(logits).to(dev)
        ref = _route_bufs(torch, T, K, k, dev, -1)
        got = _route_bufs(torch, T, K, k, dev, -7)
        tileq_route(lg, T, K, k, ref, ws)
        tileq_route_static(lg, T, K, k, got)
        torch.cuda.synchronize()
        for name in ("topk_idx", "expert_offsets", "sorted_pairs"):
            assert torch.equal(got[name], ref[name]), f"call {call}: {name} differs"
        # same kernel, same inputs: the weights agree to the bit, well within 1e-6
        assert torch.allclose(got["topk_w"], ref["topk_w"], rtol=1e-6, atol=0), f"call {call}"


def test_route_static_rejects_too_many_pairs(torch_cuda):
    torch = torch_cuda
    from tiled_rank_b200 import TileQError, tileq_route_static, _lib
    dev = torch.device("cuda:0")
    T, K, k = 4097, 8, 2  # 8194 pairs > TILEQ_ROUTE_STATIC_MAX_PAIRS
    lg = torch.zeros((T, K), dtype=torch.float32, device=dev)
    with pytest.raises(TileQError) as e:
        tileq_route_static(lg, T, K, k, _route_bufs(torch, T, K, k, dev, 0))
    assert e.value.status == _lib.TILEQ_ERR_UNSUPPORTED
