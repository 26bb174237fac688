"""Seeded synthetic decode-step inputs shaped like the SinkRouter workloads.

This module only draws tensors. It holds none of the method's arithmetic (no
cosine routing, no softmax, no attention); the oracle and the CUDA path both
consume what it returns, and the tests check the planted labels against the
oracle's routing.

Workloads (SinkRouter README, decode benchmark commands and model list; sota2
summary, Abstract, for the backbones): single-token decode of one attention
layer of Llama-3.1-8B (32 query / 8 KV heads), Llama-3.1-70B (64 / 8) and
LLaVA-1.5-7B (32 / 32, MHA), head_dim 128, bf16 KV cache laid out
[batch, kv_head, position, head_dim]. No weights or datasets are involved: the
queries and caches are random with planted sink structure.

Planted sink group: a random unit direction u, position-0 key k0 = 40 u, every
query head of the group q_h = k0 + N(0, 0.2^2 I) (cosine with k0 about 0.998).
Active group: k0 is the random cache row at position 0; every query head is
built with a cosine to k0 inside (-0.2, 0.2) by mixing a component orthogonal
to k0 with a small random share along it. Values are N(0, 1) everywhere; for
the LLaVA-shaped workload positions 1..576 (the image tokens) are N(0, 1.5^2).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

HEAD_DIM = 128
SINK_KEY_NORM = 40.0
SINK_QUERY_NOISE = 0.2
ACTIVE_MAX_COS = 0.2
IMAGE_TOKENS = 576
IMAGE_SCALE = 1.5

# Seed offsets per tensor role, so each role has its own stream.
_ROLE = {"k": 1, "v": 2, "k0dir": 3, "qnoise": 4, "qactive": 5, "lens": 6, "sinks": 7, "strength": 8,
         "qin": 9, "knew": 10, "vnew": 11}


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    max_ctx: int
    n_kv_heads: int
    group: int  # query heads per KV head (M)
    ragged: bool = False  # seq_lens ~ U{max_ctx/2 .. max_ctx}
    sink_groups: tuple = ()  # fixed sink groups (same for every sequence)
    sink_prob: float | None = None  # independent Bernoulli per (sequence, group)
    image_tokens: int = 0
    tau: float = 0.6
    description: str = ""

    @property
    def n_q_heads(self) -> int:
        return self.n_kv_heads * self.group


WORKLOADS = {
    "tiny_4k": Workload(
        "tiny_4k", 1, 4096, 8, 4, sink_groups=(0, 1, 2, 3),
        description="batch 1, context 4096, 32 q / 8 kv heads, groups 0-3 planted sinks"),
    "llama8b_128k": Workload(
        "llama8b_128k", 1, 131072, 8, 4, sink_groups=(0, 1, 2, 3),
        description="Llama-3.1-8B-shaped layer, batch 1, context 131072, 32 q / 8 kv heads, "
                    "4 of 8 groups planted sinks"),
    "llama8b_512k": Workload(
        "llama8b_512k", 1, 524288, 8, 4, sink_groups=(0, 1, 2, 3),
        description="Llama-3.1-8B-shaped layer, batch 1, context 524288, 32 q / 8 kv heads; "
                    "sink fraction swept over 0/25/50/75/100% (first k groups)"),
    "llama70b_ragged": Workload(
        "llama70b_ragged", 4, 131072, 8, 8, ragged=True, sink_prob=0.4,
        description="Llama-3.1-70B-shaped layer, batch 4, ragged contexts U{65536..131072}, "
                    "64 q / 8 kv heads, sink probability 0.4 per (sequence, group)"),
    "llava7b_mha": Workload(
        "llava7b_mha", 8, 32768, 32, 1, sink_prob=0.6, image_tokens=IMAGE_TOKENS,
        description="LLaVA-1.5-7B-shaped layer, MHA 32 heads, batch 8, context 32768, "
                    "positions 1-576 image tokens N(0,1.5^2), sink probability 0.6 per head"),
}


@dataclass
class DecodeInputs:
    workload: Workload
    seed: int
    q: torch.Tensor  # [B, Hq, 128] bf16
    k_cache: torch.Tensor  # [B, Hkv, Lmax, 128] bf16
    v_cache: torch.Tensor  # [B, Hkv, Lmax, 128] bf16
    k0: torch.Tensor  # [B, Hkv, 128] bf16
    v0: torch.Tensor  # [B, Hkv, 128] bf16
    seq_lens: torch.Tensor  # [B] int32
    planted_sink: torch.Tensor  # [B, Hkv] bool
    tau: float
    extra: dict = field(default_factory=dict)

    @property
    def batch(self):
        return self.q.shape[0]

    @property
    def n_q_heads(self):
        return self.q.shape[1]

    @property
    def n_kv_heads(self):
        return self.k_cache.shape[1]

    @property
    def max_seq_len(self):
        return self.k_cache.shape[2]

    def to(self, device) -> "DecodeInputs":
        moved = {n: getattr(self, n).to(device) for n in
                 ("q", "k_cache", "v_cache", "k0", "v0", "seq_lens", "planted_sink")}
        return DecodeInputs(self.workload, self.seed, tau=self.tau, extra=dict(self.extra), **moved)


def _gen(seed: int, role: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + _ROLE[role])
    return g


def _fill_normal_bf16(out: torch.Tensor, gen: torch.Generator, image_tokens: int = 0):
    """Fill a [B, H, L, d] bf16 tensor with N(0,1) drawn in fp32 then rounded,
    one (b, h) slab at a time to bound the fp32 scratch."""
    B, H, L, d = out.shape
    for b in range(B):
        for h in range(H):
            x = torch.randn((L, d), generator=gen, device=out.device, dtype=torch.float32)
            if image_tokens:
                x[1:1 + image_tokens] *= IMAGE_SCALE
            out[b, h].copy_(x)


def make(name: str, seed: int = 0, device="cpu", *, max_ctx: int | None = None,
         batch: int | None = None, sink_fraction: float | None = None,
         sink_groups=None, poison_padding: bool = False, tau: float | None = None) -> DecodeInputs:
    """Draw one decode step of the named workload.

    Overrides: ``max_ctx`` (shrink the context for quick cases; ragged contexts
    scale with it), ``batch``, ``sink_fraction`` (first round(f*Hkv) groups are
    sinks, the 512K sweep), ``sink_groups`` (explicit tuple), ``poison_padding``
    (cache rows at positions >= seq_len are NaN, to catch over-reads), ``tau``.
    """
    w = WORKLOADS[name]
    B = batch if batch is not None else w.batch
    Lmax = max_ctx if max_ctx is not None else w.max_ctx
    Hkv, M = w.n_kv_heads, w.group
    Hq = Hkv * M
    d = HEAD_DIM
    device = torch.device(device)

    # Context lengths.
    if w.ragged:
        lo = max(1, Lmax // 2)
        gl = _gen(seed, "lens", "cpu")
        seq_lens = torch.randint(lo, Lmax + 1, (B,), generator=gl, dtype=torch.int32)
    else:
        seq_lens = torch.full((B,), Lmax, dtype=torch.int32)

    # Which groups are planted sinks.
    if sink_groups is not None:
        planted = torch.zeros(B, Hkv, dtype=torch.bool)
        planted[:, list(sink_groups)] = True
    elif sink_fraction is not None:
        k = int(round(sink_fraction * Hkv))
        planted = torch.zeros(B, Hkv, dtype=torch.bool)
        planted[:, :k] = True
    elif w.sink_prob is not None:
        gs = _gen(seed, "sinks", "cpu")
        planted = torch.rand((B, Hkv), generator=gs) < w.sink_prob
    else:
        planted = torch.zeros(B, Hkv, dtype=torch.bool)
        planted[:, list(w.sink_groups)] = True

    k_cache = torch.empty((B, Hkv, Lmax, d), dtype=torch.bfloat16, device=device)
    v_cache = torch.empty((B, Hkv, Lmax, d), dtype=torch.bfloat16, device=device)
    _fill_normal_bf16(k_cache, _gen(seed, "k", device), w.image_tokens)
    _fill_normal_bf16(v_cache, _gen(seed, "v", device), w.image_tokens)

    # Planted sink keys at position 0.
    gdir = _gen(seed, "k0dir", device)
    n_sink = int(planted.sum())
    if n_sink:
        u = torch.randn((n_sink, d), generator=gdir, device=device, dtype=torch.float32)
        u = u / u.norm(dim=1, keepdim=True)
        idx = planted.nonzero(as_tuple=False).to(device)
        k_cache[idx[:, 0], idx[:, 1], 0] = (SINK_KEY_NORM * u).to(torch.bfloat16)

    k0 = k_cache[:, :, 0].clone()
    v0 = v_cache[:, :, 0].clone()

    # Queries: per head, built against the (bf16) position-0 key of its group.
    k0f = k0.float()  # [B, Hkv, d]
    khat = k0f / k0f.norm(dim=-1, keepdim=True)
    khat_h = khat.repeat_interleave(M, dim=1)  # [B, Hq, d]
    k0_h = k0f.repeat_interleave(M, dim=1)
    noise = torch.randn((B, Hq, d), generator=_gen(seed, "qnoise", device), device=device)
    q_sink = k0_h + SINK_QUERY_NOISE * noise
    ga = _gen(seed, "qactive", device)
    r = torch.randn((B, Hq, d), generator=ga, device=device)
    beta = (torch.rand((B, Hq, 1), generator=ga, device=device) * 2.0 - 1.0) * ACTIVE_MAX_COS
    r_perp = r - (r * khat_h).sum(-1, keepdim=True) * khat_h
    q_active = r_perp + beta * r_perp.norm(dim=-1, keepdim=True) * khat_h
    sink_h = planted.to(device).repeat_interleave(M, dim=1).unsqueeze(-1)
    q = torch.where(sink_h, q_sink, q_active).to(torch.bfloat16)

    if poison_padding:
        for b in range(B):
            L = int(seq_lens[b])
            if L < Lmax:
                k_cache[b, :, L:] = float("nan")
                v_cache[b, :, L:] = float("nan")

    t = w.tau if tau is None else tau
    return DecodeInputs(w, seed, q, k_cache, v_cache, k0, v0, seq_lens.to(device), planted, t)


def make_graded(seed: int = 0, device="cpu", *, batch: int = 16, n_kv_heads: int = 8, group: int = 4,
                ctx: int = 4096, tau: float = 0.6) -> DecodeInputs:
    """Decode steps with a continuum of sink strength, for studying the routing
    proxy against full attention. Every unit (b, g) draws a strength t ~ U(0, 1):
    its position-0 key is k0 = (4 + 36 t) u for a random unit direction u, and
    each query head is q_h = 40 t u + r_h with r_h ~ N(0, I). Weak units look like
    ordinary heads (small cosine to k0, small weight on position 0); strong ones
    like planted sinks. ``extra["strength"]`` holds t [B, Hkv]."""
    device = torch.device(device)
    B, Hkv, M, d = batch, n_kv_heads, group, HEAD_DIM
    Hq = Hkv * M
    k_cache = torch.empty((B, Hkv, ctx, d), dtype=torch.bfloat16, device=device)
    v_cache = torch.empty((B, Hkv, ctx, d), dtype=torch.bfloat16, device=device)
    _fill_normal_bf16(k_cache, _gen(seed, "k", device))
    _fill_normal_bf16(v_cache, _gen(seed, "v", device))
    t = torch.rand((B, Hkv), generator=_gen(seed, "strength", device), device=device)
    u = torch.randn((B, Hkv, d), generator=_gen(seed, "k0dir", device), device=device)
    u = u / u.norm(dim=-1, keepdim=True)
    k_cache[:, :, 0] = ((4.0 + 36.0 * t).unsqueeze(-1) * u).to(torch.bfloat16)
    r = torch.randn((B, Hq, d), generator=_gen(seed, "qnoise", device), device=device)
    q = ((40.0 * t).repeat_interleave(M, dim=1).unsqueeze(-1) * u.repeat_interleave(M, dim=1) + r)
    seq_lens = torch.full((B,), ctx, dtype=torch.int32, device=device)
    w = Workload("graded", B, ctx, Hkv, M, tau=tau, description="graded sink strength t ~ U(0,1) per unit")
    return DecodeInputs(w, seed, q.to(torch.bfloat16), k_cache, v_cache, k_cache[:, :, 0].clone(),
                        v_cache[:, :, 0].clone(), seq_lens, t > 0.5, tau, extra={"strength": t})


def rope_tables(max_pos: int, head_dim: int = HEAD_DIM, base: float = 500000.0, device="cpu"):
    """cos / sin tables, fp32 [max_pos, head_dim / 2], for the rotate-half
    rotary embedding: row p, column i holds cos / sin of p * base^(-2i/d).
    base 500000 is Llama 3's; no context-extension rescaling of the frequencies
    (synthetic inputs). The angles are formed in fp64 and the results rounded
    to fp32. These are inputs: both the oracle and the CUDA path read them."""
    inv = base ** (-torch.arange(0, head_dim, 2, dtype=torch.float64) / head_dim)
    ang = torch.arange(max_pos, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cos(ang).float().to(device), torch.sin(ang).float().to(device)


def make_projections(batch: int, n_q_heads: int, n_kv_heads: int, seed: int = 0, device="cpu"):
    """The new token's projections before RoPE: q_in [B, Hq, d], k_new and
    v_new [B, Hkv, d], N(0, 1) rounded to bf16."""
    device = torch.device(device)
    d = HEAD_DIM

    def draw(shape, role):
        return torch.randn(shape, generator=_gen(seed, role, device), device=device).to(torch.bfloat16)

    return (draw((batch, n_q_heads, d), "qin"), draw((batch, n_kv_heads, d), "knew"),
            draw((batch, n_kv_heads, d), "vnew"))


def needed_bytes(seq_lens, active_units, n_kv_heads: int, n_q_heads: int, batch: int,
                 head_dim: int = HEAD_DIM) -> int:
    """Bytes a routed decode step must move: the active groups' K and V rows,
    k0/v0 of every group, the query read and the output write (bf16)."""
    sl = [int(x) for x in seq_lens]
    kv = sum(sl[u // n_kv_heads] for u in active_units) * head_dim * 2 * 2
    return kv + batch * n_kv_heads * head_dim * 2 * 2 + 2 * batch * n_q_heads * head_dim * 2


def expected_active_fraction(name: str) -> float:
    w = WORKLOADS[name]
    if w.sink_prob is not None:
        return 1.0 - w.sink_prob
    return 1.0 - len(w.sink_groups) / w.n_kv_heads


def describe(name: str) -> str:
    return WORKLOADS[name].description


__all__ = ["WORKLOADS", "Workload", "DecodeInputs", "make", "make_graded", "needed_bytes", "describe",
           "expected_active_fraction", "HEAD_DIM"]
