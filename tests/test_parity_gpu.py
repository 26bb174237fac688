"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded bf16 inputs. Masks and active lists bit-exact; sink outputs equal
v0 bit for bit; active outputs within the tolerances of tests/gpu_helpers.py."""
import pytest
import torch

import math
import os

import oracle
from kv_cache_routing_sr_b200 import inputs, native, proxy_quality
from tests import gpu_helpers as H
from tests.conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

DEV = "cuda"
FULL = ["tiny_4k", "llama8b_128k", "llama8b_512k", "llama70b_ragged", "llava7b_mha"]


# ---- routing ----------------------------------------------------------------------------

@pytest.mark.parametrize("name", FULL)
def test_route_bit_exact_full_size(name):
    x = inputs.make(name, seed=0, device=DEV)
    mask_g, act_g = native.route(x.q, x.k0, x.tau)
    torch.cuda.synchronize()
    mask_r, act_r, score = oracle.route(x.q.cpu(), x.k0.cpu(), H.tau32(x.tau))
    H.assert_route_equal(mask_g.cpu(), act_g.cpu(), mask_r, act_r)
    assert (score - x.tau).abs().min().item() >= 0.05
    assert torch.equal(mask_r, x.planted_sink.flatten().to(torch.uint8))


def test_route_mixed_heads_use_the_minimum():
    """A group with one non-sink head is active; ties at tau route."""
    x = inputs.make("tiny_4k", seed=1, device=DEV, max_ctx=64)
    q = x.q.clone()
    q[0, 1] = x.q[0, 16]  # group 0 (sink) gets one head from an active group
    m, a = native.route(q, x.k0, x.tau)
    mr, ar, _ = oracle.route(q.cpu(), x.k0.cpu(), H.tau32(x.tau))
    H.assert_route_equal(m.cpu(), a.cpu(), mr, ar)
    assert int(m[0]) == 0 and int(m[1]) == 1


def test_route_extreme_thresholds():
    x = inputs.make("llava7b_mha", seed=2, device=DEV, max_ctx=64)
    m, a = native.route(x.q, x.k0, float("inf"))
    assert int(m.sum()) == 0 and int(a[0]) == 256
    assert torch.equal(a[1:].cpu(), torch.arange(256, dtype=torch.int32))
    m, a = native.route(x.q, x.k0, float("-inf"))
    assert int(m.sum()) == 256 and int(a[0]) == 0


# ---- attention, whole problem compared at reduced contexts --------------------------------

SMALL = [
    ("tiny_4k", {}),
    ("llama8b_128k", dict(max_ctx=3000)),
    ("llama8b_512k", dict(max_ctx=2048, sink_fraction=0.25)),
    ("llama70b_ragged", dict(max_ctx=2500, poison_padding=True)),
    ("llava7b_mha", dict(max_ctx=1500, batch=3)),
]


@pytest.mark.parametrize("name,kw", SMALL, ids=[s[0] for s in SMALL])
def test_decode_matches_oracle_small(name, kw):
    x = inputs.make(name, seed=11, device=DEV, **kw)
    mask_g, act_g, out_g, _ = H.gpu_step(x)
    ref = H.oracle_full(x, x.tau)
    H.assert_route_equal(mask_g, act_g, ref.mask, ref.active_list)
    M = x.n_q_heads // x.n_kv_heads
    for u in range(x.batch * x.n_kv_heads):
        b, g = divmod(u, x.n_kv_heads)
        if mask_g[u]:
            H.assert_sink_exact(out_g[b, g * M:(g + 1) * M], x.v0[b, g])
    act = mask_g.view(x.batch, x.n_kv_heads).repeat_interleave(M, dim=1) == 0
    H.assert_active_close(out_g[act], ref.out[act], name)


@pytest.mark.parametrize("n_splits", [1, 2, 7, 64, 0])
def test_split_count_sweep(n_splits):
    x = inputs.make("llama70b_ragged", seed=12, device=DEV, max_ctx=4096, poison_padding=True)
    mask_g, _, out_g, _ = H.gpu_step(x, n_splits=n_splits)
    H.check_against_oracle(x, out_g, mask_g, what=f"n_splits={n_splits}")


@pytest.mark.parametrize("L", [1, 2, 15, 63, 64, 65, 129, 257, 4097])
def test_ragged_lengths(L):
    """Lengths around tile and split edges, poisoned padding behind them."""
    x = inputs.make("tiny_4k", seed=13, device=DEV, max_ctx=4160, sink_groups=(1, 6))
    x.seq_lens.fill_(L)
    x.k_cache[:, :, L:] = float("nan")
    x.v_cache[:, :, L:] = float("nan")
    for ns in (0, 3):
        mask_g, _, out_g, _ = H.gpu_step(x, n_splits=ns)
        H.check_against_oracle(x, out_g, mask_g, what=f"L={L} n_splits={ns}")


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_group_sizes(M):
    from tests.pins import _rand_case
    q, k, v, k0, v0, seq = _rand_case(14 + M, 2, 3, M, 777, Lmax=800)
    seq[1] = 555
    x = inputs.DecodeInputs(inputs.WORKLOADS["tiny_4k"], 0, q, k, v, k0, v0, seq,
                            torch.zeros(2, 3, dtype=torch.bool), 0.6).to(DEV)
    for tau in (float("inf"), 0.0):
        mask_g, _, out_g, _ = H.gpu_step(x, tau=tau)
        mr, _, _ = oracle.route(q, k0, H.tau32(tau))
        assert torch.equal(mask_g, mr)
        H.check_against_oracle(x, out_g, mask_g, what=f"M={M} tau={tau}")


# ---- full-size configs: sampled units -------------------------------------------------------

def _sample(mask, k_active=2):
    act = [u for u in range(len(mask)) if mask[u] == 0]
    pick = act[:1] + act[-1:] if len(act) > 1 else act
    return sorted(set(pick[:k_active] + [u for u in range(len(mask)) if mask[u]]))


@pytest.mark.parametrize("name", FULL)
def test_decode_full_size_sampled(name):
    x = inputs.make(name, seed=0, device=DEV)
    mask_g, act_g, out_g, _ = H.gpu_step(x)
    mask_r, act_r, _ = oracle.route(x.q.cpu(), x.k0.cpu(), H.tau32(x.tau))
    H.assert_route_equal(mask_g, act_g, mask_r, act_r)
    H.check_against_oracle(x, out_g, mask_g, units=_sample(mask_g), what=name)


def _every_unit(x, what):
    """Every unit of a full-size workload against the oracle (run once on the
    whole problem, one thread per host core): sink heads bit-exact v0, active
    heads within the tolerances, per (sequence, head)."""
    mask_g, act_g, out_g, _ = H.gpu_step(x)
    ref = H.oracle_full(x, x.tau, n_threads=os.cpu_count() or 8)
    H.assert_route_equal(mask_g, act_g, ref.mask, ref.active_list)
    Hkv, M = x.n_kv_heads, x.n_q_heads // x.n_kv_heads
    v0 = x.v0.cpu()
    act = []
    for u in range(x.batch * Hkv):
        b, g = divmod(u, Hkv)
        if mask_g[u]:
            H.assert_sink_exact(out_g[b, g * M:(g + 1) * M], v0[b, g])
        else:
            act.append((b, g))
    if act:
        got = torch.stack([out_g[b, g * M:(g + 1) * M] for b, g in act])
        want = torch.stack([ref.out[b, g * M:(g + 1) * M] for b, g in act])
        H.assert_active_close(got, want, f"{what}, all {len(act)} active units")
    return len(act)


@pytest.mark.parametrize("name", ["llama8b_128k", "llama70b_ragged", "llava7b_mha"])
def test_decode_full_size_every_unit(name):
    _every_unit(inputs.make(name, seed=21, device=DEV), name)


@pytest.mark.parametrize("frac", [0.0, 0.5])
def test_512k_every_unit(frac):
    """The full-size 512K workload (8 groups of 524288 positions; the automatic
    plan gives each active group about 37 splits at half sinks and 18.5 with
    none, each split thousands of positions long): every group against the
    oracle."""
    x = inputs.make("llama8b_512k", seed=23, device=DEV, sink_fraction=frac)
    n_act = _every_unit(x, f"512k frac={frac}")
    assert n_act == 8 - round(8 * frac)


@pytest.mark.parametrize("frac", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_512k_sink_sweep_sampled(frac):
    x = inputs.make("llama8b_512k", seed=3, device=DEV, sink_fraction=frac)
    mask_g, act_g, out_g, _ = H.gpu_step(x)
    assert int(mask_g.sum()) == round(8 * frac)
    act = [u for u in range(8) if mask_g[u] == 0]
    H.check_against_oracle(x, out_g, mask_g, units=sorted(set(act[:1] + [u for u in range(8) if mask_g[u]])),
                           what=f"512k frac={frac}")


# ---- invariants, edge cases, error reporting ----------------------------------------------

def test_all_sink_and_all_active():
    x = inputs.make("llama70b_ragged", seed=15, device=DEV, max_ctx=1024)
    mask_g, act_g, out_g, _ = H.gpu_step(x, tau=float("-inf"))
    assert int(act_g[0]) == 0
    M = 8
    for u in range(32):
        b, g = divmod(u, 8)
        H.assert_sink_exact(out_g[b, g * M:(g + 1) * M], x.v0[b, g])
    mask_g, act_g, out_g, _ = H.gpu_step(x, tau=float("inf"))
    assert int(act_g[0]) == 32
    H.check_against_oracle(x, out_g, mask_g)


def test_single_unit():
    x = inputs.make("llama8b_128k", seed=16, device=DEV, max_ctx=5000, batch=1)
    x = inputs.DecodeInputs(x.workload, 0, x.q[:, :4].contiguous(), x.k_cache[:, :1].contiguous(),
                            x.v_cache[:, :1].contiguous(), x.k0[:, :1].contiguous(), x.v0[:, :1].contiguous(),
                            x.seq_lens, x.planted_sink[:, :1], 0.6)
    for tau in (float("inf"), float("-inf")):
        mask_g, _, out_g, _ = H.gpu_step(x, tau=tau)
        H.check_against_oracle(x, out_g, mask_g)


def test_routing_isolation_on_gpu():
    x = inputs.make("llama8b_128k", seed=17, device=DEV, max_ctx=8192)
    mask_r, _, out_r, _ = H.gpu_step(x)
    _, _, out_d, _ = H.gpu_step(x, tau=float("inf"))
    act = mask_r.view(1, 8).repeat_interleave(4, dim=1) == 0
    mx, _, _ = H.active_error(out_r[act], out_d[act].double())
    assert mx <= 2 ** -8 * out_d[act].double().abs().max().item() + 1e-6


def test_repeat_calls_identical_and_counters_reset():
    x = inputs.make("llama70b_ragged", seed=18, device=DEV, max_ctx=3000)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    outs = []
    for _ in range(3):
        _, _, o, _ = H.gpu_step(x, decoder=dec)
        outs.append(o.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    U = x.batch * x.n_kv_heads
    cnt = dec.workspace.view[256:256 + 4 * U].view(torch.int32)
    assert int(cnt.abs().sum()) == 0
    assert dec.workspace.device_error() == 0


def test_seq_len_out_of_range_is_clamped_and_reported():
    x = inputs.make("tiny_4k", seed=19, device=DEV, max_ctx=512)
    ref_hi = inputs.DecodeInputs(x.workload, 0, x.q, x.k_cache, x.v_cache, x.k0, x.v0,
                                 torch.full((1,), 512, dtype=torch.int32, device=DEV), x.planted_sink, x.tau)
    x.seq_lens.fill_(10_000)
    dec = native.Decoder(1, 32, 8, 512)
    mask_g, _, out_g, _ = H.gpu_step(x, decoder=dec)
    assert dec.workspace.device_error() & native.SR_DEVERR_SEQ_LEN
    H.check_against_oracle(ref_hi, out_g, mask_g)
    dec.workspace.clear_device_error()
    assert dec.workspace.device_error() == 0


def test_bad_active_list_is_reported_not_fatal():
    x = inputs.make("tiny_4k", seed=20, device=DEV, max_ctx=256)
    dec = native.Decoder(1, 32, 8, 256)
    bad = torch.tensor([3, 5, 4, 6, 0, 0, 0, 0, 0], dtype=torch.int32, device=DEV)  # 4 after 5: out of order
    native.decode_attention(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, bad, dec.out,
                            workspace=dec.workspace)
    torch.cuda.synchronize()
    assert dec.workspace.device_error() & native.SR_DEVERR_ACTIVE_LIST
    assert torch.isfinite(dec.out.float()).all()


def test_step_graph_replay_matches_eager_and_tracks_inputs():
    """A captured step (route + decode in one CUDA graph) gives the eager result,
    and replays read the bound tensors' current contents."""
    x = inputs.make("llama70b_ragged", seed=23, device=DEV, max_ctx=2000)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    eager = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau).clone()
    mask_e = dec.route_mask.clone()
    g = native.StepGraph(dec, x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
    for _ in range(2):
        out = g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager) and torch.equal(dec.route_mask, mask_e)
    # change the inputs in place: make every group of sequence 0 a sink
    x.q[0] = x.k0[0].repeat_interleave(8, dim=0)
    out = g.replay().cpu()
    torch.cuda.synchronize()
    mask = dec.route_mask.cpu()
    assert bool(mask[:8].all())
    H.check_against_oracle(x, out, mask)


# ---- fused routing + decode (one launch) -------------------------------------------------

FUSED_CASES = [
    ("tiny_4k", {}),
    ("llama8b_128k", dict(max_ctx=5000)),
    ("llama70b_ragged", dict(max_ctx=3000, poison_padding=True)),
    ("llava7b_mha", dict(max_ctx=1500)),
    ("llama8b_512k", dict(max_ctx=2048, sink_fraction=1.0)),
    ("llama8b_512k", dict(max_ctx=2048, sink_fraction=0.0)),
]


@pytest.mark.parametrize("name,kw", FUSED_CASES, ids=[f"{c[0]}-{i}" for i, c in enumerate(FUSED_CASES)])
def test_fused_step_equals_two_calls(name, kw):
    x = inputs.make(name, seed=31, device=DEV, **kw)
    two = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    one = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    for ns in (0, 3):
        ref = two.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau, n_splits=0 if ns == 0 else ns)
        got = one.step_fused(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau,
                             n_splits=0 if ns == 0 else ns)
        torch.cuda.synchronize()
        assert torch.equal(one.route_mask, two.route_mask)
        n = int(two.active_list[0])
        assert torch.equal(one.active_list[:1 + n], two.active_list[:1 + n])
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), "fused output differs from two calls"
    assert one.workspace.device_error() == 0
    H.check_against_oracle(x, got.cpu(), one.route_mask.cpu())


def test_fused_full_size_and_optional_outputs():
    x = inputs.make("llama8b_128k", seed=0, device=DEV)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    out = native.route_decode_attention(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau,
                                        workspace=dec.workspace)  # no route outputs requested
    torch.cuda.synchronize()
    mask_r, _, _ = oracle.route(x.q.cpu(), x.k0.cpu(), H.tau32(x.tau))
    H.check_against_oracle(x, out.cpu(), mask_r, units=[0, 3, 4, 7])
    g = native.StepGraph(dec, x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
    assert torch.equal(g.replay(), out)


def test_layer_stack_graph_and_gating():
    """A 4-layer stack in one CUDA graph: replay equals the eager steps, layers
    outside the gate route nothing, and each layer matches the oracle."""
    from kv_cache_routing_sr_b200 import multilayer
    stack = multilayer.LayerStack("llama8b_128k", 4, seed=5, max_ctx=1500)
    gate = multilayer.LayerGate(1, 2)
    eager = [o.clone() for o in stack.step_eager(gate)]
    masks = [dec.route_mask.clone() for _, dec in stack.layers]
    g = stack.capture(gate)
    g.replay()
    torch.cuda.synchronize()
    for i, ((x, dec), ref) in enumerate(zip(stack.layers, eager)):
        assert torch.equal(dec.out, ref)
        assert torch.equal(dec.route_mask, masks[i])
        if i in (0, 3):
            assert int(dec.route_mask.sum()) == 0  # gated out: standard attention
        else:
            assert int(dec.route_mask.sum()) == 4
        H.check_against_oracle(x, dec.out.cpu(), dec.route_mask.cpu())


# ---- shape edges: chunked routing, large batches, the unit limit ------------------------

def _random_problem(seed, B, Hkv, M, Lmax, ragged=True, sink_share=0.5):
    """Random bf16 problem with a chosen share of sink-like groups (queries along k0)."""
    g = torch.Generator().manual_seed(seed)
    Hq = Hkv * M
    q = torch.randn(B, Hq, 128, generator=g)
    k = torch.randn(B, Hkv, Lmax, 128, generator=g)
    v = torch.randn(B, Hkv, Lmax, 128, generator=g)
    k0 = k[:, :, 0].clone()
    sink = torch.rand(B, Hkv, generator=g) < sink_share
    q = torch.where(sink.repeat_interleave(M, dim=1).unsqueeze(-1), k0.repeat_interleave(M, dim=1) * 3.0, q)
    seq = (torch.randint(1, Lmax + 1, (B,), generator=g, dtype=torch.int32) if ragged
           else torch.full((B,), Lmax, dtype=torch.int32))
    bf = lambda t: t.to(torch.bfloat16)  # noqa: E731
    kb = bf(k)
    return inputs.DecodeInputs(inputs.WORKLOADS["tiny_4k"], seed, bf(q), kb, bf(v), kb[:, :, 0].clone(),
                               bf(v)[:, :, 0].clone(), seq, sink, 0.6).to(DEV)


@pytest.mark.parametrize("B,Hkv,M,Lmax", [
    (16, 8, 8, 300),     # 128 units of M = 8: the routing kernel stages rows in two chunks
    (4200, 1, 2, 40),    # B beyond the shared seq_lens table; 20 routing chunks
    (16384, 1, 1, 17),   # the unit limit: prologue tables fill the whole stage area
])
def test_shape_edges(B, Hkv, M, Lmax):
    x = _random_problem(40 + B, B, Hkv, M, Lmax)
    for fused in (False, True):
        dec = native.Decoder(B, Hkv * M, Hkv, Lmax)
        if fused:
            out = dec.step_fused(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
        else:
            out = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
        torch.cuda.synchronize()
        assert dec.workspace.device_error() == 0
        mr, ar, _ = oracle.route(x.q.cpu(), x.k0.cpu(), H.tau32(x.tau))
        H.assert_route_equal(dec.route_mask.cpu(), dec.active_list.cpu(), mr, ar)
        units = list(range(B * Hkv))
        if len(units) > 600:  # sample: every sink plus a spread of active units
            act = [u for u in units if mr[u] == 0]
            units = sorted(set([u for u in units if mr[u] == 1][:300] + act[::max(1, len(act) // 300)]))
        H.check_against_oracle(x, out.cpu(), dec.route_mask.cpu(), units=units, what=f"{B}x{Hkv}x{M}")


def test_forced_splits_beyond_length():
    """More forced splits than positions: most splits are empty and must weigh 0."""
    x = _random_problem(51, 3, 4, 4, 20, ragged=True)
    x.seq_lens[:] = torch.tensor([1, 7, 20], dtype=torch.int32, device=DEV)
    for ns in (16, 64):
        mask_g, _, out_g, _ = H.gpu_step(x, n_splits=ns)
        H.check_against_oracle(x, out_g, mask_g, what=f"n_splits={ns}")


def test_exact_cosine_tie_routes():
    """An exact tie is a sink on both sides, each in its own precision: with
    q = (3, 4, 0, ...) and k0 = (1, 0, ...) the kernel's fp32 cosine is fl(3/5),
    which equals tau = 0.6f, and the oracle's fp64 cosine is exactly 0.6, which
    equals tau = 0.6 in fp64. (Comparing the fp64 cosine with the fp32 tau would
    not be a tie; parity workloads keep every score 0.05 away from tau.)"""
    x = inputs.make("tiny_4k", seed=52, device=DEV, max_ctx=128)
    k0 = torch.zeros_like(x.k0)
    k0[0, :, 0] = 1.0
    q = torch.zeros_like(x.q)
    q[0, :, 0], q[0, :, 1] = 3.0, 4.0
    q[0, 16:32] = x.q[0, 16:32]  # groups 4-7 keep random queries
    k0[0, 4:] = x.k0[0, 4:]
    mask, act = native.route(q, k0, 0.6)
    mr, ar, score = oracle.route(q.cpu(), k0.cpu(), 0.6)
    assert score[:4].tolist() == [0.6] * 4
    H.assert_route_equal(mask.cpu(), act.cpu(), mr, ar)
    assert mask[:4].tolist() == [1, 1, 1, 1]


# ---- log-sum-exp output and the routing-proxy analysis ------------------------------------

def test_lse_output_matches_logsumexp_and_oracle_p0():
    x = inputs.make_graded(seed=61, batch=4, ctx=3000, device=DEV)
    x.seq_lens[1] = 1234
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    native.route(x.q, x.k0, 0.6, dec.route_mask, dec.active_list)
    lse = torch.full((x.batch, x.n_q_heads), -7.0, dtype=torch.float32, device=DEV)
    native.decode_attention(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, dec.active_list, dec.out,
                            workspace=dec.workspace, lse=lse)
    torch.cuda.synchronize()
    mask = dec.route_mask.cpu().view(x.batch, x.n_kv_heads).repeat_interleave(4, dim=1).bool()
    lse = lse.cpu().double()
    assert torch.isnan(lse[mask]).all()
    q, k = x.q.cpu().double(), x.k_cache.cpu().double()
    for b in range(x.batch):
        L = int(x.seq_lens[b])
        logits = torch.einsum("hd,hld->hl", q[b], k[b].repeat_interleave(4, dim=0)[:, :L]) / math.sqrt(128)
        ref = torch.logsumexp(logits, dim=-1)
        act = ~mask[b]
        assert (lse[b][act] - ref[act]).abs().max().item() < 2e-3
    p0 = proxy_quality.full_attention_p0(x).cpu().double()
    ref = H.oracle_full(x, float("inf")).p0
    assert (p0 - ref).abs().max().item() < 1e-2


def test_proxy_quality_analysis_runs_and_matches_oracle_event():
    x = inputs.make_graded(seed=62, batch=16, ctx=2048, device=DEV)
    res = proxy_quality.evaluate(x, taus=[0.2, 0.4, 0.55, 0.6, 0.8], cutoff=0.5)
    assert 0.0 < res["event_rate"] < 1.0 and len(res["curve"]) == 5
    ref = H.oracle_full(x, float("inf"))
    ev_ref = ref.p0.view(16, 8, 4).mean(-1) >= 0.5
    p0 = proxy_quality.full_attention_p0(x).cpu().view(16, 8, 4).mean(-1)
    near = (p0 - 0.5).abs() < 0.02  # decisions this close to the cutoff may differ by rounding
    assert torch.equal((p0 >= 0.5)[~near], ev_ref[~near])


@pytest.mark.parametrize("M,ns,L", [(4, 70, 9000), (8, 40, 6000), (1, 140, 20000), (2, 7, 3000), (2, 66, 9000)])
def test_unit_result_independent_of_the_rest_of_the_launch(M, ns, L):
    """With forced splits a unit's partials depend only on n_splits and its
    length, and the last-CTA merge takes them in a fixed order, so unit 0's
    bits (lse included) must not depend on the rest of the launch: unit 0
    alone (every CTA holds at most one split, so the merging CTA has no
    further work) against unit 0 among many active units (more splits than
    CTAs: CTA j's split j is never its last), and the first sequence as a
    launch of its own, whose 8 units take the prologue's register path.
    ns = 70 at M = 4, 40 at M = 8, 140 at M = 1 and 66 at M = 2 take several
    batches of the merge (at M < 4 in several partial groups)."""
    G = native.grid_size()
    Hkv = 8
    B = max(1, -(-(G + ns) // (ns * Hkv)) + 1)  # B*Hkv*ns > G + ns
    x = inputs.make("tiny_4k", seed=7, device=DEV, max_ctx=L)
    g = torch.Generator(device=DEV).manual_seed(M * 1000 + ns)
    q = torch.randn((B, Hkv * M, 128), generator=g, device=DEV).to(torch.bfloat16)
    kc = torch.randn((B, Hkv, L, 128), generator=g, device=DEV).to(torch.bfloat16)
    vc = torch.randn((B, Hkv, L, 128), generator=g, device=DEV).to(torch.bfloat16)
    k0, v0 = kc[:, :, 0].contiguous(), vc[:, :, 0].contiguous()
    sl = torch.full((B,), L, dtype=torch.int32, device=DEV)
    U = B * Hkv
    assert U * ns > G + ns and ns <= G
    del x
    runs = {}
    # "one_sequence": the first sequence alone (8 units: the prologue's register
    # path); the other two runs have more than 32 units (its block-wide path).
    for name, nb, units in (("alone", B, [0]), ("among_many", B, list(range(U))), ("one_sequence", 1, [0])):
        act = torch.tensor([len(units)] + units, dtype=torch.int32, device=DEV)
        ws = native.Workspace(nb, Hkv * M, Hkv, L, max_splits=ns, device=DEV)
        lse = torch.empty((nb, Hkv * M), dtype=torch.float32, device=DEV)
        out = native.decode_attention(q[:nb].contiguous(), kc[:nb].contiguous(), vc[:nb].contiguous(),
                                      k0[:nb].contiguous(), v0[:nb].contiguous(), sl[:nb].contiguous(), act,
                                      n_splits=ns, workspace=ws, lse=lse)
        torch.cuda.synchronize()
        assert ws.device_error() == 0
        runs[name] = (out[0, :M].cpu(), lse[0, :M].cpu())
    a = runs["alone"]
    # and unit 0 itself against the oracle (one-unit sub-problem, routed active)
    ref, _ = oracle.decode(q[:1, :M].cpu(), kc[:1, :1].cpu(), vc[:1, :1].cpu(), v0[:1, :1].cpu(), sl[:1].cpu(),
                           torch.zeros(1, dtype=torch.uint8))
    H.assert_active_close(a[0].unsqueeze(0), ref, f"unit 0, M={M}, {ns} forced splits")
    for other in ("among_many", "one_sequence"):
        b = runs[other]
        assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)), f"unit 0 differs ({other})"
        assert torch.equal(a[1].view(torch.int32), b[1].view(torch.int32)), f"lse of unit 0 differs ({other})"
    # and both agree with the oracle
    ref, _ = oracle.decode(q[:1, :M].cpu(), kc[:1, :1].cpu(), vc[:1, :1].cpu(), v0[:1, :1].cpu(),
                           sl[:1].cpu(), torch.zeros(1, dtype=torch.uint8))
    H.assert_active_close(a[0].unsqueeze(0), ref[0].unsqueeze(0), f"M={M} ns={ns}")


def test_concurrent_host_threads_on_separate_streams():
    """Two host threads, each with its own Decoder (workspace, route buffers)
    and CUDA stream, run decode steps concurrently; every output equals the
    serial result bit for bit (the library's lazily built per-device state is
    safe to share)."""
    import threading

    xs = [inputs.make("llama70b_ragged", seed=70 + i, device=DEV, max_ctx=3000) for i in range(2)]
    refs = []
    for x in xs:
        _, _, out, _ = H.gpu_step(x)
        refs.append(out.clone())
    results, errors = [[], []], []

    def worker(i):
        try:
            x = xs[i]
            st = torch.cuda.Stream()
            dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
            with torch.cuda.stream(st):
                for _ in range(30):
                    out = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau, stream=st)
                    results[i].append(out.clone())
            st.synchronize()
        except Exception as e:  # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for i in range(2):
        assert len(results[i]) == 30
        for out in results[i]:
            assert torch.equal(out.cpu().view(torch.int16), refs[i].cpu().view(torch.int16))


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8), (64, 8)])
def test_position0_weight_matches_its_definition(Hq, Hkv):
    """sr_position0_weight against exp(<q, K[., g, 0]> / sqrt(d) - lse) in fp64,
    for given lse values (NaN ones propagate), at M = 1, 4 and 8."""
    g = torch.Generator(device=DEV).manual_seed(Hq * 7 + Hkv)
    B, L = 3, 40
    q = torch.randn((B, Hq, 128), generator=g, device=DEV).to(torch.bfloat16)
    kc = torch.randn((B, Hkv, L, 128), generator=g, device=DEV).to(torch.bfloat16)
    lse = (torch.rand((B, Hq), generator=g, device=DEV) * 4.0 + 1.0).float()
    lse[0, 1] = float("nan")
    p0 = native.position0_weight(q, kc, lse).cpu().double()
    M = Hq // Hkv
    k0 = kc[:, :, 0].cpu().double().repeat_interleave(M, dim=1)
    ref = torch.exp((q.cpu().double() * k0).sum(-1) / math.sqrt(128) - lse.cpu().double())
    assert torch.isnan(p0[0, 1]) and torch.isnan(ref[0, 1])
    ok = ~torch.isnan(ref)
    assert ((p0[ok] - ref[ok]).abs() / ref[ok]).max().item() < 1e-5


def test_two_million_positions_every_unit():
    """Contexts four times the longest workload (2^21 positions, one sequence
    77 short of it): 64-bit offsets, long shares and the tail tile, on every
    unit at M = 8 with routing off, against the oracle element by element."""
    import types
    g = torch.Generator(device=DEV).manual_seed(2021)
    B, Hkv, M, L = 2, 1, 8, 1 << 21
    q = (2.0 * torch.randn((B, Hkv * M, 128), generator=g, device=DEV)).to(torch.bfloat16)
    kc = torch.randn((B, Hkv, L, 128), generator=g, device=DEV).to(torch.bfloat16)
    vc = torch.randn((B, Hkv, L, 128), generator=g, device=DEV).to(torch.bfloat16)
    sl = torch.tensor([L, L - 77], dtype=torch.int32, device=DEV)
    x = types.SimpleNamespace(q=q, k_cache=kc, v_cache=vc, k0=kc[:, :, 0].contiguous(), v0=vc[:, :, 0].contiguous(),
                              seq_lens=sl, batch=B, n_q_heads=Hkv * M, n_kv_heads=Hkv, max_seq_len=L)
    dec = native.Decoder(B, Hkv * M, Hkv, L)
    out = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, float("inf"))
    torch.cuda.synchronize()
    assert dec.workspace.device_error() == 0
    mask = dec.route_mask.cpu()
    assert int(mask.sum()) == 0
    H.check_against_oracle(x, out.cpu(), mask, what="2M positions")
