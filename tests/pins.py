"""Pins for the fp64 oracle: checks against facts fixed outside the oracle.

Each pin takes a loaded ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with the pages or the mathematics. They are collected as
tests in ``test_oracle_pins.py`` and re-run against deliberately broken builds
of the oracle in ``test_oracle_mutants.py`` (every planted mistake must trip at
least one pin).

Sources of truth, none of them the oracle itself:
* torch's fp64 ``scaled_dot_product_attention`` (a library routine) for dense
  softmax attention (SinkRouter README, active path is standard attention);
* hand-derived closed forms (``tests/golden/hand_worked.json`` and below);
* invariants: permutation of cached positions, routing isolation, the planted
  sink bound derived from eq. (1) of the pith.science review (Figure 1 caption);
* exact special cases: tau=-inf routes everything (sink output is v0 bit for
  bit), tau=+inf routes nothing.
"""
from __future__ import annotations

import json
import math
import os

import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_worked.json")
INF = float("inf")


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float64).to(torch.bfloat16)


def _rand_case(seed, B, Hkv, M, L, d=128, Lmax=None, v_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    Lmax = Lmax or L
    Hq = Hkv * M
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    v = (v_scale * torch.randn(B, Hkv, Lmax, d, generator=g)).to(torch.bfloat16)
    k0 = k[:, :, 0].clone()
    v0 = v[:, :, 0].clone()
    seq = torch.full((B,), L, dtype=torch.int32)
    return q, k, v, k0, v0, seq


def _sdpa_reference(q, k, v, seq_lens):
    """Dense attention by torch's fp64 CPU SDPA, KV heads repeated per group."""
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    M = Hq // Hkv
    out = torch.empty(B, Hq, d, dtype=torch.float64)
    for b in range(B):
        L = int(seq_lens[b])
        kk = k[b, :, :L].double().repeat_interleave(M, dim=0)  # [Hq, L, d]
        vv = v[b, :, :L].double().repeat_interleave(M, dim=0)
        qq = q[b].double().unsqueeze(1)  # [Hq, 1, d]
        out[b] = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv).squeeze(1)
    return out


def _run(o, q, k, v, k0, v0, seq, tau, units=None, n_threads=1):
    mask, active, score = o.route(q, k0, tau)
    out, p0 = o.decode(q, k, v, v0, seq, mask, units, n_threads)
    return mask, active, score, out, p0


# --- attention pins -----------------------------------------------------------------

def pin_dense_matches_sdpa(o):
    """tau=+inf routes nothing: the oracle is dense attention (torch SDPA, fp64)."""
    for seed, (B, Hkv, M, L) in enumerate([(1, 2, 4, 37), (2, 2, 1, 64), (1, 1, 8, 5),
                                            (2, 3, 2, 17)]):
        q, k, v, k0, v0, seq = _rand_case(100 + seed, B, Hkv, M, L, Lmax=L + 3)
        if B == 2:
            seq[1] = max(1, L - 9)
        mask, _, _, out, _ = _run(o, q, k, v, k0, v0, seq, INF)
        assert int(mask.sum()) == 0
        ref = _sdpa_reference(q, k, v, seq)
        err = (out - ref).abs().max().item()
        assert err <= 1e-12, f"dense attention differs from SDPA by {err}"


def pin_all_sinks_return_v0(o):
    """tau=-inf routes every group (s >= -inf always): output is v0 bit for bit."""
    q, k, v, k0, v0, seq = _rand_case(7, 2, 4, 4, 33)
    v0 = (torch.randn(v0.shape, generator=torch.Generator().manual_seed(8)) * 3).to(torch.bfloat16)
    mask, active, _, out, p0 = _run(o, q, k, v, k0, v0, seq, -INF)
    assert bool((mask == 1).all()) and int(active[0]) == 0
    expect = v0.double().repeat_interleave(4, dim=1)
    assert torch.equal(out, expect), "sink output is not v0 exactly"
    assert bool(torch.isnan(p0).all())


def pin_routing_isolation(o):
    """Routing never changes an active group's output."""
    q, k, v, k0, v0, seq = _rand_case(11, 2, 4, 4, 50)
    # Make groups (0,1) and (1,3) sink-like: q heads along k0.
    for b, g in [(0, 1), (1, 3)]:
        q[b, 4 * g:4 * g + 4] = (k0[b, g].double() * 2.0).to(torch.bfloat16)
    mask, _, _, out_r, _ = _run(o, q, k, v, k0, v0, seq, 0.6)
    _, _, _, out_d, _ = _run(o, q, k, v, k0, v0, seq, INF)
    m = mask.view(2, 4)
    assert bool(m[0, 1]) and bool(m[1, 3]) and int(m.sum()) == 2
    for b in range(2):
        for g in range(4):
            sl = slice(4 * g, 4 * g + 4)
            if m[b, g]:
                assert torch.equal(out_r[b, sl], v0[b, g].double().expand(4, -1))
            else:
                assert torch.equal(out_r[b, sl], out_d[b, sl]), "routing changed an active group"


def pin_planted_sink_bound(o):
    """|dense_out - v0| <= 2 (1 - p0) max_j |v_j| elementwise, with v0 = V[., 0]:
    dense_out - v0 = sum_{j>=1} p_j (v_j - v_0) (eq. (1), pith.science review,
    Figure 1 caption). Checked on strongly and weakly sink-dominated heads."""
    q, k, v, k0, v0, seq = _rand_case(21, 1, 3, 4, 200)
    # group 0: planted sink (large k0, queries along it); group 1: mild; group 2: random
    g = torch.Generator().manual_seed(22)
    u = torch.randn(128, generator=g, dtype=torch.float64)
    u = u / u.norm()
    k[0, 0, 0] = (40 * u).to(torch.bfloat16)
    k[0, 1, 0] = (6 * u).to(torch.bfloat16)
    for h in range(4):
        q[0, h] = (40 * u + 0.2 * torch.randn(128, generator=g, dtype=torch.float64)).to(torch.bfloat16)
        q[0, 4 + h] = (6 * u + 0.5 * torch.randn(128, generator=g, dtype=torch.float64)).to(torch.bfloat16)
    v0 = v[:, :, 0].clone()
    _, _, _, out, p0 = _run(o, q, k, v, k0, v0, seq, INF)
    seen_strong = False
    for grp in range(3):
        vmax = v[0, grp, :200].double().abs().amax(dim=0)  # per coordinate
        for h in range(4 * grp, 4 * grp + 4):
            lhs = (out[0, h] - v[0, grp, 0].double()).abs()
            rhs = 2.0 * (1.0 - p0[0, h]) * vmax
            assert bool((lhs <= rhs + 1e-15).all()), "planted-sink bound violated"
            assert 0.0 < p0[0, h] <= 1.0
            if p0[0, h] > 1 - 1e-12:
                seen_strong = True
    assert seen_strong, "planted sink is not sink-dominated"


def pin_permutation_invariance(o):
    """Permuting cached positions 1..L-1 (K and V jointly) leaves outputs (to
    1e-12) and the route decision unchanged."""
    q, k, v, k0, v0, seq = _rand_case(31, 2, 2, 4, 77)
    q[0, 0:4] = (k0[0, 0].double() * 4).to(torch.bfloat16)  # one sink group
    perm = torch.cat([torch.tensor([0]), 1 + torch.randperm(76, generator=torch.Generator().manual_seed(32))])
    kp, vp = k[:, :, perm].clone(), v[:, :, perm].clone()
    m1, _, _, o1, _ = _run(o, q, k, v, k0, v0, seq, 0.6)
    m2, _, _, o2, _ = _run(o, q, kp, vp, k0, v0, seq, 0.6)
    assert torch.equal(m1, m2)
    assert (o1 - o2).abs().max().item() <= 1e-12


def pin_closed_forms(o):
    """All keys equal => mean of values; L=1 => V[0]; one logit 60 above the rest
    => that value (the rest weigh at most e^-60 each)."""
    d = 128
    g = torch.Generator().manual_seed(41)
    # equal keys
    L = 23
    q = torch.randn(1, 2, d, generator=g).to(torch.bfloat16)
    krow = torch.randn(d, generator=g).to(torch.bfloat16)
    k = krow.expand(1, 1, L, d).clone()
    v = torch.randn(1, 1, L, d, generator=g).to(torch.bfloat16)
    seq = torch.tensor([L], dtype=torch.int32)
    mask = torch.zeros(1, dtype=torch.uint8)
    out, p0 = o.decode(q, k, v, v[:, :, 0], seq, mask)
    mean = v[0, 0].double().mean(dim=0)
    assert (out[0] - mean).abs().max().item() <= 1e-13
    assert abs(p0[0, 0].item() - 1.0 / L) <= 1e-15
    # single position
    seq1 = torch.tensor([1], dtype=torch.int32)
    out1, p01 = o.decode(q, k, v, v[:, :, 0], seq1, mask)
    assert torch.equal(out1[0], v[0, 0, 0].double().expand(2, -1))
    assert bool((p01 == 1.0).all())
    # dominant position: q = 2 e_0, k_j = 0 except k_5 = (60*sqrt(128)/2) e_0
    q = torch.zeros(1, 1, d, dtype=torch.bfloat16)
    q[0, 0, 0] = 2.0
    k = torch.zeros(1, 1, 64, d, dtype=torch.bfloat16)
    k[0, 0, 5, 0] = 30.0 * math.sqrt(128.0)  # logit = 2 * 30*sqrt(128) / sqrt(128) = 60
    kval = float(k[0, 0, 5, 0].double())  # bf16-rounded; logit stays >= 59
    assert 2.0 * kval / math.sqrt(128.0) >= 59.0
    v = torch.randn(1, 1, 64, d, generator=g).to(torch.bfloat16)
    out2, _ = o.decode(q, k, v, v[:, :, 0], torch.tensor([64], dtype=torch.int32), mask)
    assert (out2[0, 0] - v[0, 0, 5].double()).abs().max().item() <= 1e-20


def pin_hand_worked(o):
    """The hand-derived cases of tests/golden/hand_worked.json."""
    with open(GOLDEN) as f:
        fx = json.load(f)
    env = {"e": math.e, "exp": math.exp, "sqrt": math.sqrt}
    ev = lambda s: float(eval(str(s), {"__builtins__": {}}, env))  # noqa: E731
    for case in fx["cases"]:
        d, Hq, Hkv, L = case["d"], case["Hq"], case["Hkv"], case["seq_len"]
        q = _bf16(case["q"]).view(1, Hq, d)
        if "k_heads" in case:
            k = _bf16(case["k_heads"]).view(1, Hkv, L, d)
            v = _bf16(case["v_heads"]).view(1, Hkv, L, d)
        else:
            k = _bf16(case["k"]).view(1, Hkv, L, d)
            v = _bf16(case["v"]).view(1, Hkv, L, d)
        k0 = _bf16(case["k0"]).view(1, Hkv, d) if "k0" in case else k[:, :, 0].clone()
        v0 = _bf16(case["v0"]).view(1, Hkv, d) if "v0" in case else v[:, :, 0].clone()
        seq = torch.tensor([L], dtype=torch.int32)
        for run in case["runs"]:
            tau = INF if run["tau"] == "inf" else float(run["tau"])
            mask, active, score, out, p0 = _run(o, q, k, v, k0, v0, seq, tau)
            if "score" in run:
                assert abs(score[0].item() - ev(run["score"])) <= 1e-15, case["name"]
            if "sink" in run:
                assert bool(mask[0]) == run["sink"], case["name"]
            exp_out = torch.tensor([[ev(x) for x in row] for row in run["out"]], dtype=torch.float64)
            assert (out[0] - exp_out).abs().max().item() <= 1e-15, case["name"]
            if "p0" in run:
                exp_p0 = torch.tensor([ev(x) for x in run["p0"]], dtype=torch.float64)
                assert (p0[0] - exp_p0).abs().max().item() <= 1e-15, case["name"]


# --- routing pins ---------------------------------------------------------------------

def pin_route_geometry(o):
    """Cosines with known values: parallel (+1), anti-parallel (-1), disjoint
    support (0), the 3-4-5 triangle (exactly 0.6, which is a sink at tau=0.6
    since ties route), zero-norm query (0 by the reading), and the group score
    is the minimum over the group's heads."""
    d = 128
    k0 = torch.zeros(1, 4, d, dtype=torch.float64)
    k0[0, :, 0] = 1.0
    k0[0, 2, 0] = 0.5
    q = torch.zeros(1, 8, d, dtype=torch.float64)  # M = 2
    q[0, 0, 0], q[0, 1, 0] = 4.0, 0.25  # group 0: cos 1, 1
    q[0, 2, 0], q[0, 3, 1] = -2.0, 3.0  # group 1: cos -1, 0
    q[0, 4, 0], q[0, 4, 1] = 3.0, 4.0  # group 2: cos 0.6, and
    q[0, 5, 0] = 1.0  # cos 1
    q[0, 7, 0] = 1.0  # group 3: head 6 zero-norm (cos 0), head 7 cos 1
    mask, active, score = o.route(q.to(torch.bfloat16), k0.to(torch.bfloat16), 0.6)
    assert score.tolist() == [1.0, -1.0, 0.6, 0.0], score.tolist()
    assert mask.tolist() == [1, 0, 1, 0]
    assert active[:3].tolist() == [2, 1, 3]
    # ties route; strictly above does not
    m2, _, _ = o.route(q.to(torch.bfloat16), k0.to(torch.bfloat16), math.nextafter(0.6, 1.0))
    assert m2.tolist() == [1, 0, 0, 0]


def pin_route_scale_invariance(o):
    """cos(a q, b k0) = cos(q, k0) for a, b > 0 (powers of two keep bf16 exact);
    with one head per group, negating the query negates the group score."""
    q, k, v, k0, v0, seq = _rand_case(51, 3, 4, 2, 4)
    _, _, s1 = o.route(q, k0, 0.0)
    _, _, s2 = o.route((q.double() * 8).to(torch.bfloat16), (k0.double() / 4).to(torch.bfloat16), 0.0)
    assert (s1 - s2).abs().max().item() <= 1e-15
    q1, _, _, k01, _, _ = _rand_case(52, 2, 6, 1, 4)
    _, _, a = o.route(q1, k01, 0.0)
    _, _, b = o.route((-q1.double()).to(torch.bfloat16), k01, 0.0)
    assert torch.equal(a, -b)


def pin_active_list_order(o):
    """The active list holds the count, then the non-sink group indices in
    ascending order, and agrees with the mask."""
    q, k, v, k0, v0, seq = _rand_case(61, 5, 8, 2, 4)
    g = torch.Generator().manual_seed(62)
    pick = torch.rand(5, 8, generator=g) < 0.5
    for b in range(5):
        for gg in range(8):
            if pick[b, gg]:
                q[b, 2 * gg:2 * gg + 2] = (k0[b, gg].double() * 2).to(torch.bfloat16)
    mask, active, _ = o.route(q, k0, 0.6)
    n = int(active[0])
    idx = active[1:1 + n].tolist()
    assert idx == sorted(idx) and len(set(idx)) == n
    assert idx == [u for u in range(40) if mask[u] == 0]
    assert mask.view(5, 8).bool().equal(pick)


# --- the step before the scan: RoPE, append, position-0 capture ----------------------

def _rope_case(seed, B, Hkv, M, Lmax, max_pos=64, d=128):
    g = torch.Generator().manual_seed(seed)
    Hq = Hkv * M
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, Lmax, d, generator=g).to(torch.bfloat16)
    k0 = kc[:, :, 0].clone()
    v0 = vc[:, :, 0].clone()
    inv = 500000.0 ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
    ang = torch.arange(max_pos, dtype=torch.float64)[:, None] * inv[None, :]
    return q, kn, vn, kc, vc, k0, v0, torch.cos(ang).float(), torch.sin(ang).float()


def pin_rope_identity_at_position_zero(o):
    """At position 0 (cos 1, sin 0) the rotation is the identity: the query is
    unchanged, the new key / value land in slot 0 and become k0 / v0."""
    q, kn, vn, kc, vc, k0, v0, cs, sn = _rope_case(81, 2, 3, 4, 16)
    seq = torch.zeros(2, dtype=torch.int32)
    st, qo, kc2, vc2, k02, v02, sl = o.rope_append(q, kn, vn, cs, sn, seq, kc, vc, k0, v0)
    assert st == 0 and sl.tolist() == [1, 1]
    assert torch.equal(qo.view(torch.int16), q.view(torch.int16))
    assert torch.equal(kc2[:, :, 0].view(torch.int16), kn.view(torch.int16))
    assert torch.equal(vc2[:, :, 0].view(torch.int16), vn.view(torch.int16))
    assert torch.equal(k02.view(torch.int16), kn.view(torch.int16))
    assert torch.equal(v02.view(torch.int16), vn.view(torch.int16))
    assert torch.equal(kc2[:, :, 1:], kc[:, :, 1:])


def pin_rope_closed_form_and_ties(o):
    """Exact values: x_i = 2, x_(i+64) = 1 with c = 0.5, s = 0.75 gives
    (2*0.5 - 1*0.75, 1*0.5 + 2*0.75) = (0.25, 2). Ties round to even:
    1 + 2^-8 (between 1 and 1 + 2^-7) -> 1, and 1 + 3*2^-8 -> 1 + 2^-6."""
    d = 128
    q = torch.zeros(1, 3, d, dtype=torch.bfloat16)
    q[0, 0, 5], q[0, 0, 69] = 2.0, 1.0
    q[0, 1, 7] = 1.0
    q[0, 2, 9] = 1.0
    cs = torch.zeros(4, 64)
    sn = torch.zeros(4, 64)
    cs[3, 5], sn[3, 5] = 0.5, 0.75
    cs[3, 7] = 1.0 + 2.0 ** -8
    cs[3, 9] = 1.0 + 3 * 2.0 ** -8
    kc = torch.zeros(1, 1, 8, d, dtype=torch.bfloat16)
    st, qo, *_ = o.rope_append(q.view(1, 3, d), torch.zeros(1, 1, d, dtype=torch.bfloat16),
                               torch.zeros(1, 1, d, dtype=torch.bfloat16), cs, sn,
                               torch.tensor([3], dtype=torch.int32), kc, kc.clone(),
                               torch.zeros(1, 1, d, dtype=torch.bfloat16), torch.zeros(1, 1, d, dtype=torch.bfloat16))
    assert st == 0
    assert qo[0, 0, 5].item() == 0.25 and qo[0, 0, 69].item() == 2.0
    assert qo[0, 1, 7].item() == 1.0
    assert qo[0, 2, 9].item() == 1.0 + 2.0 ** -6


def pin_rope_rotation_preserves_norm_and_inverts(o):
    """A true rotation keeps every pair's norm (up to bf16 rounding), and
    rotating by an angle then by its negative returns the input."""
    q, kn, vn, kc, vc, k0, v0, cs, sn = _rope_case(82, 2, 2, 2, 48, max_pos=64)
    seq = torch.tensor([17, 40], dtype=torch.int32)
    st, qo, *_ = o.rope_append(q, kn, vn, cs, sn, seq, kc, vc, k0, v0)
    assert st == 0
    a, b = q.double()[..., :64], q.double()[..., 64:]
    c, d_ = qo.double()[..., :64], qo.double()[..., 64:]
    n_in, n_out = (a * a + b * b).sqrt(), (c * c + d_ * d_).sqrt()
    assert ((n_out - n_in).abs() <= 2.0 ** -7 * n_in + 1e-30).all()
    # inverse: a table whose row p holds the negative angle
    sn_neg = -sn
    st2, back, *_ = o.rope_append(qo, kn, vn, cs, sn_neg, seq, kc, vc, k0, v0)
    assert st2 == 0
    # two bf16 roundings of a rotated pair, each at most 2^-9 of the pair's norm
    err = (back.double() - q.double()).abs()
    assert (err[..., :64] <= 2.0 ** -7 * n_in).all() and (err[..., 64:] <= 2.0 ** -7 * n_in).all()


def pin_rope_append_bookkeeping(o):
    """Only slot p is written, k0 / v0 change only when p == 0, lengths advance,
    and a slot past the cache or the table is refused for that sequence."""
    q, kn, vn, kc, vc, k0, v0, cs, sn = _rope_case(83, 3, 2, 2, 10, max_pos=64)
    seq = torch.tensor([4, 0, 10], dtype=torch.int32)  # the last one is full
    st, qo, kc2, vc2, k02, v02, sl = o.rope_append(q, kn, vn, cs, sn, seq, kc, vc, k0, v0)
    assert st == 1 and sl.tolist() == [5, 1, 10]
    for b, p in ((0, 4), (1, 0)):
        keep = [j for j in range(10) if j != p]
        assert torch.equal(kc2[b][:, keep], kc[b][:, keep]) and torch.equal(vc2[b][:, keep], vc[b][:, keep])
        assert torch.equal(vc2[b, :, p].view(torch.int16), vn[b].view(torch.int16))
    assert torch.equal(k02[0], k0[0]) and torch.equal(v02[0], v0[0])  # p = 4: k0 kept
    assert torch.equal(k02[1], kc2[1, :, 0]) and torch.equal(v02[1], vn[1])  # p = 0: captured
    assert torch.equal(kc2[2], kc[2]) and torch.equal(k02[2], k0[2])  # refused: untouched
    assert (qo[2].float() == 0).all() and (qo[:2].float() != 0).any()  # ... and a zero query


PINS = [pin_dense_matches_sdpa, pin_all_sinks_return_v0, pin_routing_isolation,
        pin_planted_sink_bound, pin_permutation_invariance, pin_closed_forms,
        pin_hand_worked, pin_route_geometry, pin_route_scale_invariance, pin_active_list_order,
        pin_rope_identity_at_position_zero, pin_rope_closed_form_and_ties,
        pin_rope_rotation_preserves_norm_and_inverts, pin_rope_append_bookkeeping]
