"""The routing-proxy quality analysis (CPU): its counting, and the graded
generator's behaviour measured with the oracle (a stronger planted sink gives a
larger cosine score and a larger full-attention weight on position 0)."""
import math

import torch

import oracle
from kv_cache_routing_sr_b200 import inputs, proxy_quality


def test_pr_curve_counts():
    event = torch.tensor([1, 1, 0, 0, 1, 0], dtype=torch.bool)
    preds = {0.5: torch.tensor([1, 0, 1, 0, 1, 0], dtype=torch.bool),
             0.9: torch.tensor([0, 0, 0, 0, 1, 0], dtype=torch.bool),
             2.0: torch.zeros(6, dtype=torch.bool)}
    rows = {r["tau"]: r for r in proxy_quality.pr_curve(preds, event)}
    assert rows[0.5]["precision"] == round(2 / 3, 4) and rows[0.5]["recall"] == round(2 / 3, 4)
    assert rows[0.9]["precision"] == 1.0 and rows[0.9]["recall"] == round(1 / 3, 4)
    assert rows[2.0]["recall"] == 0.0 and rows[2.0]["f1"] == 0.0 and rows[2.0]["predicted_sinks"] == 0


def test_graded_inputs_span_sink_strength():
    x = inputs.make_graded(seed=3, batch=6, ctx=512)
    t = x.extra["strength"].flatten()
    mask, _, score = oracle.route(x.q, x.k0, -math.inf)
    out, p0 = oracle.decode(x.q, x.k_cache, x.v_cache, x.v0, x.seq_lens, torch.zeros_like(mask), n_threads=4)
    p0_unit = p0.view(6, 8, 4).mean(-1).flatten()
    # strength orders both the proxy score and the sink weight (rank correlation)
    def rank(v):
        return torch.argsort(torch.argsort(v)).double()
    def spearman(a, b):
        ra, rb = rank(a), rank(b)
        ra, rb = ra - ra.mean(), rb - rb.mean()
        return float((ra * rb).sum() / (ra.norm() * rb.norm()))
    assert spearman(t, score) > 0.9
    # p0 saturates at 1 for strong units: compare the two ends of the strength range
    order = torch.argsort(t)
    third = len(t) // 3
    assert float(p0_unit[order[:third // 2]].mean()) < 0.1
    assert float(p0_unit[order[-third:]].min()) > 0.99
    # with the oracle standing in for the GPU, strong units are the predicted sinks
    event = p0_unit >= 0.5
    rows = proxy_quality.pr_curve({tau: (score >= tau) for tau in (0.3, 0.6, 0.9)}, event)
    assert rows[-1]["precision"] == 1.0  # only clear sinks pass tau = 0.9
