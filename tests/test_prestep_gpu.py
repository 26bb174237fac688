"""Parity of sr_rope_append_route -- RoPE of the query and the new key, the
append at slot seq_lens[b], the position-0 capture, routing and the length
update in one launch -- with the oracle.

Bars: the rotated query, both caches, k0 / v0 and the lengths are bit-exact
(the kernel's rotation is the correctly rounded bf16 of the fp64 value, which
is the oracle's definition); the mask and active list equal sr_route on the
kernel's own (q_out, k0) bit for bit, and equal the oracle's fp64 routing away
from ties. A decode step after the append is checked against the oracle on the
appended state.
"""
from __future__ import annotations

import types

import pytest
import torch

import oracle
from kv_cache_routing_sr_b200 import inputs, native
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"
TAU = 0.6


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16)


def _case(B, Hkv, M, Lmax, seed, positions, sink_units=(), max_pos=None):
    """CPU tensors of one append step. Units in sink_units get query heads
    that, once rotated to their slot, point along the group's (post-step)
    position-0 key: they are built by rotating the target back with the
    oracle (a table with the sines negated rotates by minus the angle)."""
    Hq = Hkv * M
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn(B, Hkv, Lmax, 128, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, 128, generator=g).to(torch.bfloat16)
    k0, v0 = kc[:, :, 0].clone(), vc[:, :, 0].clone()
    q_in, kn, vn = inputs.make_projections(B, Hq, Hkv, seed=seed)
    cs, sn = inputs.rope_tables(max_pos or Lmax)
    seq = torch.tensor(positions, dtype=torch.int32)
    o = oracle.load()
    if sink_units:
        k0_after = o.rope_append(q_in, kn, vn, cs, sn, seq, kc, vc, k0, v0)[4]
        target = q_in.clone()
        for u in sink_units:
            b, gg = divmod(u, Hkv)
            for m in range(M):
                noise = 0.03 * torch.randn(128, generator=g) * k0_after[b, gg].float().norm() / 11.3
                target[b, gg * M + m] = (k0_after[b, gg].float() + noise).to(torch.bfloat16)
        back = o.rope_append(target, kn, vn, cs, -sn, seq, kc, vc, k0, v0)[1]
        for u in sink_units:
            b, gg = divmod(u, Hkv)
            q_in[b, gg * M:(gg + 1) * M] = back[b, gg * M:(gg + 1) * M]
    return dict(q_in=q_in, k_new=kn, v_new=vn, rope_cos=cs, rope_sin=sn, seq_lens=seq, k_cache=kc, v_cache=vc,
                k0=k0, v0=v0)


def _run_gpu(c, tau=TAU, in_place=False):
    d = {k: v.to(DEV).clone() for k, v in c.items()}
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    q_out = d["q_in"] if in_place else None
    q_out, mask, active = native.rope_append_route(
        d["q_in"], d["k_new"], d["v_new"], d["rope_cos"], d["rope_sin"], d["seq_lens"], d["k_cache"],
        d["v_cache"], d["k0"], d["v0"], tau, q_out=q_out, device_error=err)
    torch.cuda.synchronize()
    d["q_out"], d["mask"], d["active"], d["error"] = q_out, mask, active, int(err.item())
    return d


def _run_oracle(c):
    st, q_out, kc, vc, k0, v0, sl = oracle.load().rope_append(
        c["q_in"], c["k_new"], c["v_new"], c["rope_cos"], c["rope_sin"], c["seq_lens"], c["k_cache"],
        c["v_cache"], c["k0"], c["v0"])
    return dict(status=st, q_out=q_out, k_cache=kc, v_cache=vc, k0=k0, v0=v0, seq_lens=sl)


def _assert_state_equal(gpu, ref):
    for name in ("q_out", "k_cache", "v_cache", "k0", "v0"):
        a, b = _bits(gpu[name]), _bits(ref[name])
        if not torch.equal(a, b):
            bad = (a != b).nonzero()
            raise AssertionError(f"{name} differs from the oracle at {bad.shape[0]} elements, first {bad[0].tolist()}")
    assert torch.equal(gpu["seq_lens"].cpu(), ref["seq_lens"]), "seq_lens differ"


def _assert_routing(gpu, ref, tau=TAU):
    # bit for bit the routing kernel's decision on the same rows
    m2, a2 = native.route(gpu["q_out"], gpu["k0"], tau)
    torch.cuda.synchronize()
    H.assert_route_equal(gpu["mask"].cpu(), gpu["active"].cpu(), m2.cpu(), a2.cpu())
    # the oracle's fp64 routing of the (identical) rotated rows, away from ties
    mr, ar, score = oracle.route(ref["q_out"], ref["k0"], H.tau32(tau))
    assert (score - H.tau32(tau)).abs().min().item() > 1e-4, "test input too close to the threshold"
    H.assert_route_equal(gpu["mask"].cpu(), gpu["active"].cpu(), mr, ar)
    return mr


SHAPES = [
    # B, Hkv, M, Lmax, positions, sink units
    (2, 8, 4, 64, [0, 37], (0, 1, 9, 12)),
    (3, 4, 1, 64, [63, 5, 0], (2, 5, 11)),
    (2, 4, 2, 40, [17, 39], (0, 7)),
    (2, 8, 8, 16, [0, 15], (3, 8, 15)),
    (1, 32, 1, 100, [99], tuple(range(0, 32, 3))),
]


@pytest.mark.parametrize("B,Hkv,M,Lmax,pos,sinks", SHAPES, ids=[f"B{s[0]}_Hkv{s[1]}_M{s[2]}" for s in SHAPES])
def test_rope_append_route_matches_oracle(B, Hkv, M, Lmax, pos, sinks):
    c = _case(B, Hkv, M, Lmax, seed=B * 100 + M, positions=pos, sink_units=sinks)
    gpu, ref = _run_gpu(c), _run_oracle(c)
    assert ref["status"] == 0 and gpu["error"] == 0
    _assert_state_equal(gpu, ref)
    mask = _assert_routing(gpu, ref)
    assert all(int(mask[u]) == 1 for u in sinks), "planted sinks not routed as sinks"
    assert int(mask.sum()) < B * Hkv, "no active unit left"


@pytest.mark.parametrize("B,Hkv,M", [(40, 8, 8), (700, 1, 1), (96, 8, 4)])
def test_rope_append_route_many_chunks(B, Hkv, M):
    """More units than one shared-memory chunk holds (71 units at M = 8, 320 at
    M = 1, 128 at M = 4): every chunk is rotated, appended and routed."""
    Lmax = 8
    g = torch.Generator().manual_seed(B)
    pos = torch.randint(0, Lmax, (B,), generator=g).tolist()
    U = B * Hkv
    sinks = tuple(range(0, U, 5))
    c = _case(B, Hkv, M, Lmax, seed=B + 7, positions=pos, sink_units=sinks)
    gpu, ref = _run_gpu(c), _run_oracle(c)
    assert ref["status"] == 0 and gpu["error"] == 0
    _assert_state_equal(gpu, ref)
    mask = _assert_routing(gpu, ref)
    assert all(int(mask[u]) == 1 for u in sinks)


def test_rope_append_route_in_place_query():
    c = _case(2, 8, 4, 32, seed=5, positions=[3, 31], sink_units=(1, 10))
    gpu, ref = _run_gpu(c, in_place=True), _run_oracle(c)
    _assert_state_equal(gpu, ref)
    _assert_routing(gpu, ref)


def test_rope_append_route_refuses_bad_slots():
    """Slots -1, Lmax (a full cache) and >= max_pos are refused: the error bit
    is set, that sequence's state is untouched and its query rows are zero; the
    valid sequence proceeds; the mask is still sr_route(q_out, k0)."""
    Lmax, max_pos = 24, 20
    c = _case(4, 4, 4, Lmax, seed=9, positions=[-1, 24, 21, 6], sink_units=(13,), max_pos=max_pos)
    gpu, ref = _run_gpu(c), _run_oracle(c)
    assert ref["status"] == 1
    assert gpu["error"] == 8  # SR_DEVERR_APPEND_SLOT
    _assert_state_equal(gpu, ref)
    assert gpu["seq_lens"].cpu().tolist() == [-1, 24, 21, 7]
    assert (gpu["q_out"][:3].float() == 0).all()
    for tau in (TAU, -0.5):  # zero rows route to 0 <= tau: active at 0.6, sink at -0.5
        g2 = _run_gpu(c, tau=tau)
        m2, a2 = native.route(g2["q_out"], g2["k0"], tau)
        torch.cuda.synchronize()
        H.assert_route_equal(g2["mask"].cpu(), g2["active"].cpu(), m2.cpu(), a2.cpu())
    assert int(g2["mask"][:12].sum()) == 12


def test_rope_append_route_repeated_steps():
    """Three steps in a row on the same buffers (lengths advance 5 -> 8), each
    equal to the oracle applied to the previous step's state."""
    c = _case(2, 8, 4, 16, seed=21, positions=[5, 0], sink_units=(2,))
    d = {k: v.to(DEV).clone() for k, v in c.items()}
    state = dict(c)
    for step in range(3):
        q_in, kn, vn = inputs.make_projections(2, 32, 8, seed=100 + step)
        state.update(q_in=q_in, k_new=kn, v_new=vn)
        d.update(q_in=q_in.to(DEV), k_new=kn.to(DEV), v_new=vn.to(DEV))
        q_out, mask, active = native.rope_append_route(
            d["q_in"], d["k_new"], d["v_new"], d["rope_cos"], d["rope_sin"], d["seq_lens"], d["k_cache"],
            d["v_cache"], d["k0"], d["v0"], TAU)
        torch.cuda.synchronize()
        ref = _run_oracle(state)
        _assert_state_equal(dict(d, q_out=q_out), ref)
        state.update(k_cache=ref["k_cache"], v_cache=ref["v_cache"], k0=ref["k0"], v0=ref["v0"],
                     seq_lens=ref["seq_lens"])
    assert d["seq_lens"].cpu().tolist() == [8, 3]


def _unrotate(q, positions, cs, sn):
    """q [B, Hq, d] rotated back from slot positions[b] by the oracle (a one-row
    table holding row p with the sines negated, applied at slot 0)."""
    out = torch.empty_like(q, device="cpu")
    o = oracle.load()
    z = torch.zeros(1, 1, 128, dtype=torch.bfloat16)
    for b, p in enumerate(positions):
        r = o.rope_append(q[b:b + 1].cpu(), z, z, cs[p:p + 1].cpu(), -sn[p:p + 1].cpu(),
                          torch.zeros(1, dtype=torch.int32), torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16),
                          torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16), z, z)
        assert r[0] == 0
        out[b] = r[1][0]
    return out


def _after_append(x, gpu_q, n_q_heads):
    return types.SimpleNamespace(batch=x.batch, n_q_heads=n_q_heads, n_kv_heads=x.n_kv_heads, q=gpu_q,
                                 k_cache=x.k_cache, v_cache=x.v_cache, k0=x.k0, v0=x.v0, seq_lens=x.seq_lens)


@pytest.mark.parametrize("name,kw", [("llama8b_128k", dict(max_ctx=3000)),
                                     ("llama70b_ragged", dict(max_ctx=2500)),
                                     ("llava7b_mha", dict(max_ctx=1200, batch=3))])
def test_append_step_then_decode_matches_oracle(name, kw):
    """Decoder.append_step (append + route, then the scan) equals the oracle's
    rope_append followed by its routed attention on the appended state."""
    x = inputs.make(name, seed=31, device=DEV, **kw)
    x.seq_lens -= 1  # the last slot of every sequence is free for the new token
    B, Hq, Hkv = x.batch, x.n_q_heads, x.n_kv_heads
    _, kn, vn = inputs.make_projections(B, Hq, Hkv, seed=32, device=DEV)
    cs, sn = inputs.rope_tables(x.max_seq_len, device=DEV)
    # the planted (post-RoPE) query, rotated back to each sequence's slot
    q_in = _unrotate(x.q, x.seq_lens.tolist(), cs, sn).to(DEV)
    ref = oracle.load().rope_append(q_in, kn, vn, cs, sn, x.seq_lens, x.k_cache, x.v_cache, x.k0, x.v0)
    dec = native.Decoder(B, Hq, Hkv, x.max_seq_len)
    out = dec.append_step(q_in, kn, vn, cs, sn, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
    torch.cuda.synchronize()
    _assert_state_equal(dict(q_out=dec.q, k_cache=x.k_cache, v_cache=x.v_cache, k0=x.k0, v0=x.v0,
                             seq_lens=x.seq_lens), dict(zip(("status", "q_out", "k_cache", "v_cache", "k0", "v0",
                                                             "seq_lens"), ref)))
    full = oracle.routed_attention(ref[1], ref[2], ref[3], ref[4], ref[5], ref[6], H.tau32(x.tau), n_threads=8)
    H.assert_route_equal(dec.route_mask.cpu(), dec.active_list.cpu(), full.mask, full.active_list)
    assert torch.equal(full.mask, x.planted_sink.flatten().to(torch.uint8).cpu())
    H.check_against_oracle(_after_append(x, dec.q, Hq), dec.out.cpu(), dec.route_mask.cpu(), what=name)


def test_append_step_full_size_llama8b_128k():
    """At the full 131072-token cache: the appended slot is the last one, the
    step's routing equals the oracle's, and sampled units match it."""
    x = inputs.make("llama8b_128k", seed=41, device=DEV)
    x.seq_lens -= 1
    B, Hq, Hkv = x.batch, x.n_q_heads, x.n_kv_heads
    _, kn, vn = inputs.make_projections(B, Hq, Hkv, seed=42, device=DEV)
    cs, sn = inputs.rope_tables(x.max_seq_len, device=DEV)
    q_in = _unrotate(x.q, x.seq_lens.tolist(), cs, sn).to(DEV)
    dec = native.Decoder(B, Hq, Hkv, x.max_seq_len)
    dec.append_step(q_in, kn, vn, cs, sn, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
    torch.cuda.synchronize()
    assert x.seq_lens.cpu().tolist() == [x.max_seq_len] * B
    mr, ar, _ = oracle.route(dec.q.cpu(), x.k0.cpu(), H.tau32(x.tau))
    H.assert_route_equal(dec.route_mask.cpu(), dec.active_list.cpu(), mr, ar)
    assert torch.equal(mr, x.planted_sink.flatten().to(torch.uint8).cpu())
    act = [u for u in range(B * Hkv) if int(dec.route_mask[u]) == 0]
    H.check_against_oracle(_after_append(x, dec.q, Hq), dec.out.cpu(), dec.route_mask.cpu(),
                           units=act[:2] + [u for u in range(B * Hkv) if int(dec.route_mask[u])][:1],
                           what="128k append step")
