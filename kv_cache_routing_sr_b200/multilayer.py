"""A whole decode token's attention: every layer's routed decode step, with the
layer-range gating of the method, captured in one CUDA graph.

SinkRouter applies routing only to layers in a configured range; layers outside
it take the standard attention path (SinkRouter README, routing controls: the
layer start / end settings and the cosine threshold). Here a gated-out layer is
the same decode kernel with tau = +inf, which routes nothing. Each layer has
its own KV cache, position-0 key/value and query, and its own Decoder
(workspace, route buffers), so the layers are independent and the graph runs
them back to back the way a decode forward reaches them.

The per-token attention latency this measures is the attention part of the
pages' per-token decode latency (pith.science review of arXiv 2604.16883,
Figures 6 and 7); projections and MLPs are not part of the path.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

from . import inputs as _inputs
from . import native


@dataclass
class LayerGate:
    """Routing applies to layers start .. end (inclusive)."""
    start: int = 0
    end: int = 31
    tau: float = 0.6

    def tau_for(self, layer: int) -> float:
        return self.tau if self.start <= layer <= self.end else math.inf


class LayerStack:
    """n_layers decode steps of one workload, each with its own seeded inputs
    and its own Decoder. A gate decides which layers route."""

    def __init__(self, workload: str, n_layers: int, seed: int = 0, device="cuda", **make_kwargs):
        self.layers = []
        for layer in range(n_layers):
            x = _inputs.make(workload, seed=seed * 1000 + layer, device=device, **make_kwargs)
            dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, device=device)
            self.layers.append((x, dec))

    @property
    def n_layers(self) -> int:
        return len(self.layers)

    def step_eager(self, gate: LayerGate):
        """Every layer once, launched from the host; returns the outputs."""
        return [dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, gate.tau_for(i))
                for i, (x, dec) in enumerate(self.layers)]

    def capture(self, gate: LayerGate) -> torch.cuda.CUDAGraph:
        """All layers' routed steps under `gate`, captured in one CUDA graph.
        Graphs captured from one stack share its buffers: replay them one at a
        time."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step_eager(gate)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step_eager(gate)
        return g

    def outputs(self):
        return [dec.out for _, dec in self.layers]

    def needed_bytes(self) -> int:
        """Bytes the token must move under the last routing: every layer's active
        K/V, k0/v0, q and out."""
        total = 0
        for x, dec in self.layers:
            n = int(dec.active_list[0])
            act = dec.active_list[1:1 + n].tolist()
            total += _inputs.needed_bytes(x.seq_lens.tolist(), act, x.n_kv_heads, x.n_q_heads, x.batch)
        return total

    def active_fraction(self) -> float:
        units = sum(x.batch * x.n_kv_heads for x, _ in self.layers)
        act = sum(int(dec.active_list[0]) for _, dec in self.layers)
        return act / units
