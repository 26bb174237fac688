"""How well the cosine routing proxy predicts full-attention sink behaviour, on
synthetic decode steps with graded sink strength.

The pith.science review of arXiv 2604.16883 (Figure 10 caption) evaluates
cos(q, K_BOS) at the KV-group level as a predictor of an "oracle sink event"
defined from full-attention BOS scores, with precision, recall and F1 as
functions of the threshold (operating point 0.55). Here, on synthetic inputs:

* the oracle sink event of a unit is: the mean over its query heads of the
  full-attention weight of position 0, p0, is at least `cutoff` (the pages do
  not define the event exactly; this is the reading taken);
* p0 comes from the decode kernel run with routing disabled, through its
  log-sum-exp output and sr_position0_weight: p0 = exp(<q_h, K_0> / sqrt(d) - lse_h);
* the proxy decision at threshold tau is sr_route's mask (min over the group's
  heads of the cosine with k0, >= tau).

The counting itself (`pr_curve`) is plain host code.
"""
from __future__ import annotations

import math

import torch

from . import inputs as _inputs
from . import native


def pr_curve(scores_by_tau: dict, event: torch.Tensor) -> list:
    """Precision / recall / F1 of predicted sinks against the event, per tau.
    scores_by_tau: tau -> bool tensor of predicted sinks (same shape as event)."""
    rows = []
    ev = event.bool().flatten()
    for tau, pred in sorted(scores_by_tau.items()):
        pr = pred.bool().flatten()
        tp = int((pr & ev).sum())
        fp = int((pr & ~ev).sum())
        fn = int((~pr & ev).sum())
        prec = tp / (tp + fp) if tp + fp else 1.0
        rec = tp / (tp + fn) if tp + fn else 1.0
        f1 = 2 * prec * rec / (prec + rec) if prec + rec else 0.0
        rows.append({"tau": tau, "precision": round(prec, 4), "recall": round(rec, 4), "f1": round(f1, 4),
                     "predicted_sinks": tp + fp, "events": tp + fn})
    return rows


def full_attention_p0(x: _inputs.DecodeInputs) -> torch.Tensor:
    """p0 [B, Hq] of dense attention (routing disabled) via the kernel's lse."""
    B, Hq, Hkv = x.batch, x.n_q_heads, x.n_kv_heads
    dec = native.Decoder(B, Hq, Hkv, x.max_seq_len, device=x.q.device)
    native.route(x.q, x.k0, math.inf, dec.route_mask, dec.active_list)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=x.q.device)
    native.decode_attention(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, dec.active_list, dec.out,
                            workspace=dec.workspace, lse=lse)
    return native.position0_weight(x.q, x.k_cache, lse)


def evaluate(x: _inputs.DecodeInputs, taus, cutoff: float = 0.5) -> dict:
    """Run the proxy at every tau and compare with the full-attention event."""
    B, Hq, Hkv = x.batch, x.n_q_heads, x.n_kv_heads
    M = Hq // Hkv
    p0 = full_attention_p0(x)
    event = p0.view(B, Hkv, M).mean(-1) >= cutoff
    preds = {}
    for tau in taus:
        mask, _ = native.route(x.q, x.k0, float(tau))
        preds[float(tau)] = mask.view(B, Hkv).bool()
    torch.cuda.synchronize()
    rows = pr_curve({t: m.cpu() for t, m in preds.items()}, event.cpu())
    best = max(rows, key=lambda r: r["f1"])
    return {"units": B * Hkv, "cutoff": cutoff, "event_rate": round(float(event.float().mean()), 4),
            "curve": rows, "best_f1": best}
