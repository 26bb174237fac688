"""Context parallelism on one GPU: the partial scan, the combine kernel, and
the whole sharded step emulated rank by rank, against the oracle.

Bars: bf16 of the fp32 partial output equals sr_decode_attention's output bit
for bit and its lse equals sr_decode_attention_lse's bit for bit (same kernel,
same arithmetic, no rounding step left out); the combine kernel matches the
log-sum-exp combination computed in fp64 to within one bf16 rounding; the
sharded step matches the oracle's full attention within the tolerances of the
single-GPU step, with sink heads bit-exact copies of v0.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
from kv_cache_routing_sr_b200 import context_parallel as cp
from kv_cache_routing_sr_b200 import inputs, native
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,kw,ns", [("llama8b_128k", dict(max_ctx=3000), 0),
                                        ("llama70b_ragged", dict(max_ctx=2500), 0),
                                        ("llava7b_mha", dict(max_ctx=1200, batch=3), 0),
                                        ("llama8b_128k", dict(max_ctx=3000), 9)])
def test_partial_output_is_the_unrounded_output(name, kw, ns):
    x = inputs.make(name, seed=3, device=DEV, **kw)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, max_splits=ns)
    native.route(x.q, x.k0, x.tau, dec.route_mask, dec.active_list)
    lse = torch.empty((x.batch, x.n_q_heads), dtype=torch.float32, device=DEV)
    out = native.decode_attention(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, dec.active_list, n_splits=ns,
                                  workspace=dec.workspace, lse=lse)
    o_p, lse_p = native.decode_attention_partial(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens,
                                                 dec.active_list, n_splits=ns, workspace=dec.workspace)
    torch.cuda.synchronize()
    assert dec.workspace.device_error() == 0
    assert torch.equal(o_p.to(torch.bfloat16).view(torch.int16), out.view(torch.int16))
    assert torch.equal(lse_p.view(torch.int32), lse.view(torch.int32))  # NaN bits for sinks included
    M = x.n_q_heads // x.n_kv_heads
    mask = dec.route_mask.cpu()
    for u in range(x.batch * x.n_kv_heads):
        if mask[u]:
            b, g = divmod(u, x.n_kv_heads)
            assert torch.equal(o_p[b, g * M:(g + 1) * M].cpu(), x.v0[b, g].float().cpu().expand(M, -1))


def _combine_ref(o, lse):
    """fp64 log-sum-exp combination of parts o [R, N, 128], lse [R, N]."""
    o, lse = o.double(), lse.double()
    sink = torch.isnan(lse[0])
    m = lse.max(dim=0).values
    w = torch.exp(lse - m)
    ref = (w.unsqueeze(-1) * o).sum(0) / w.sum(0).unsqueeze(-1)
    ref[sink] = o[0][sink]
    return ref


@pytest.mark.parametrize("R", [1, 3, 8])
def test_combine_kernel_matches_fp64(R):
    B, Hq = 3, 32
    N = B * Hq
    g = torch.Generator(device=DEV).manual_seed(R)
    stride = cp.row_floats(B, Hq)
    buf = torch.zeros(R * stride, dtype=torch.float32, device=DEV)
    rows = buf.view(R, stride)
    o = torch.randn((R, N, 128), generator=g, device=DEV)
    lse = 40 * torch.randn((R, N), generator=g, device=DEV)  # spreads of many e-folds
    if R > 1:
        lse[1, :5] = -math.inf  # empty parts weigh nothing
    lse[:, 7] = float("nan")  # a sink head: copied from part 0
    rows[:, :N * 128] = o.reshape(R, -1)
    rows[:, N * 128:N * 128 + N] = lse
    out = native.combine_partials(buf, buf[N * 128:], stride, R, B, Hq)
    torch.cuda.synchronize()
    ref = _combine_ref(o.cpu(), lse.cpu())
    got = out.double().cpu().reshape(N, 128)
    # the fp32 combination then one bf16 rounding: within 2^-8 relative of the fp64 value
    assert ((got - ref).abs() <= 2.0 ** -8 * ref.abs() + 1e-5).all()
    assert torch.equal(out.reshape(N, 128)[7].cpu(), o[0, 7].to(torch.bfloat16).cpu())


def test_combine_rejects_bad_layouts():
    buf = torch.zeros(4 * 4200, dtype=torch.float32, device=DEV)
    with pytest.raises(native.SinkRouterError):
        native.combine_partials(buf, buf[4096:], 4098, 2, 1, 32)  # stride not a multiple of 4
    with pytest.raises(native.SinkRouterError):
        native.combine_partials(buf, buf[4096:], 4000, 2, 1, 32)  # parts would overlap
    with pytest.raises(native.SinkRouterError):
        native.combine_partials(buf, buf[4096:], 4128, 0, 1, 32)  # no part


@pytest.mark.parametrize("name,kw,R,ns", [("llama8b_128k", dict(max_ctx=3000), 2, 0),
                                          ("llama8b_128k", dict(max_ctx=3000), 8, 0),
                                          ("llama70b_ragged", dict(max_ctx=2500), 3, 0),
                                          ("llava7b_mha", dict(max_ctx=1200, batch=3), 5, 0),
                                          ("tiny_4k", {}, 1, 0),
                                          ("llama8b_128k", dict(max_ctx=3000), 4, 7),
                                          ("llama70b_ragged", dict(max_ctx=2500), 2, 3)])
def test_emulated_context_parallel_matches_oracle(name, kw, R, ns):
    x = inputs.make(name, seed=5, device=DEV, **kw)
    out, dec = cp.emulate(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau, R, n_splits=ns)
    torch.cuda.synchronize()
    assert dec.dec.workspace.device_error() == 0
    ref = H.oracle_full(x, x.tau)
    H.assert_route_equal(dec.dec.route_mask.cpu(), dec.dec.active_list.cpu(), ref.mask, ref.active_list)
    H.check_against_oracle(x, out.cpu(), dec.dec.route_mask.cpu(), what=f"{name} R={R} n_splits={ns}")


def test_emulated_context_parallel_512k_sampled():
    """512K positions over 8 shards, half the groups sinks: sampled units against
    the oracle, and the sharded output close to the single-GPU one."""
    x = inputs.make("llama8b_512k", seed=6, device=DEV, sink_fraction=0.5)
    out, dec = cp.emulate(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau, 8)
    torch.cuda.synchronize()
    mask = dec.dec.route_mask.cpu()
    act = [u for u in range(8) if mask[u] == 0]
    H.check_against_oracle(x, out.cpu(), mask, units=act[:2] + [0], what="512K over 8 shards")
    single = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len).step(
        x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau)
    torch.cuda.synchronize()
    assert (out.float() - single.float()).abs().max().item() <= 2e-2
