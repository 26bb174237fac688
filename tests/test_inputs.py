"""The seeded generator against the oracle's routing (CPU only): planted sink
labels equal the oracle's route mask, every group score stays at least 0.05
from tau (so fp32 and fp64 routing cannot disagree), and the draws are
reproducible."""
import pytest
import torch

from kv_cache_routing_sr_b200 import inputs

SMALL = {  # reduced contexts / batches that keep every structural feature
    "tiny_4k": dict(),
    "llama8b_128k": dict(max_ctx=2048),
    "llama8b_512k": dict(max_ctx=1024),
    "llama70b_ragged": dict(max_ctx=1024),
    "llava7b_mha": dict(max_ctx=1024),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_planted_labels_match_oracle(oracle_lib, name):
    x = inputs.make(name, seed=3, **SMALL[name])
    mask, active, score = oracle_lib.route(x.q, x.k0, x.tau)
    planted = x.planted_sink.flatten().to(torch.uint8)
    assert torch.equal(mask, planted)
    margin = (score - x.tau).abs().min().item()
    assert margin >= 0.05, f"score within {margin} of tau"


@pytest.mark.parametrize("frac,k", [(0.0, 0), (0.25, 2), (0.5, 4), (0.75, 6), (1.0, 8)])
def test_512k_sweep_fractions(oracle_lib, frac, k):
    x = inputs.make("llama8b_512k", seed=0, max_ctx=256, sink_fraction=frac)
    mask, active, _ = oracle_lib.route(x.q, x.k0, x.tau)
    assert mask.tolist() == [1] * k + [0] * (8 - k)
    assert int(active[0]) == 8 - k


def test_reproducible_and_seed_sensitive():
    a = inputs.make("llama70b_ragged", seed=5, max_ctx=256)
    b = inputs.make("llama70b_ragged", seed=5, max_ctx=256)
    c = inputs.make("llama70b_ragged", seed=6, max_ctx=256)
    for n in ("q", "k_cache", "v_cache", "seq_lens"):
        assert torch.equal(getattr(a, n), getattr(b, n))
    assert not torch.equal(a.k_cache, c.k_cache)


def test_shapes_and_structure():
    x = inputs.make("llava7b_mha", seed=1, max_ctx=1024, batch=2)
    assert x.q.shape == (2, 32, 128) and x.k_cache.shape == (2, 32, 1024, 128)
    # image-token positions are drawn wider than the text positions
    img = x.v_cache[:, :, 1:577].float().std().item()
    txt = x.v_cache[:, :, 577:].float().std().item()
    assert 1.4 < img < 1.6 and 0.9 < txt < 1.1
    r = inputs.make("llama70b_ragged", seed=2, max_ctx=1000)
    assert bool(((r.seq_lens >= 500) & (r.seq_lens <= 1000)).all())
    assert r.q.shape == (4, 64, 128)


def test_poison_padding_marks_only_padding():
    x = inputs.make("llama70b_ragged", seed=4, max_ctx=512, poison_padding=True)
    for b in range(4):
        L = int(x.seq_lens[b])
        assert not torch.isnan(x.k_cache[b, :, :L].float()).any()
        if L < 512:
            assert torch.isnan(x.v_cache[b, :, L:].float()).all()


def test_sink_keys_are_large_and_cached():
    x = inputs.make("tiny_4k", seed=0, max_ctx=64)
    n = x.k0.float().norm(dim=-1)
    assert torch.allclose(n[0, :4], torch.full((4,), 40.0), rtol=1e-2)
    assert torch.equal(x.k0, x.k_cache[:, :, 0]) and torch.equal(x.v0, x.v_cache[:, :, 0])
