"""Host checks of the token subsets the full-size GPU parity tests compare."""
import oracle
import synth
from gpu_util import N_DENSE, dense_tokens


def test_dense_tokens_cover_tiles():
    """The subset holds every 128-slot run's first and last slot of every expert."""
    cfg = synth.CONFIGS[4]
    logits, _ = synth.make_inputs(cfg, 4096)
    toks = set(dense_tokens(logits, cfg.top_k, cfg.K, seed=1).tolist())
    idx, _ = oracle.route(logits, cfg.top_k)
    off, sp = oracle.permute(idx, cfg.K)
    for e in range(cfg.K):
        for t0 in range(int(off[e]), int(off[e + 1]), 128):
            assert int(sp[t0]) // cfg.top_k in toks
            assert int(sp[min(t0 + 127, int(off[e + 1]) - 1)]) // cfg.top_k in toks
    assert len(toks) >= N_DENSE


def test_dense_tokens_small_batch_is_every_token():
    cfg = synth.CONFIGS[1]
    logits, _ = synth.make_inputs(cfg, 64)
    assert dense_tokens(logits, cfg.top_k, cfg.K, seed=0).tolist() == list(range(64))
