"""The bench's graph-timing helpers on a small case (GPU).

Every event that a captured graph records must outlive the graph: the helpers
tie their events to the graph object. These tests replay graphs after the
capturing call has returned, which is when a dropped event would be recorded
after its destruction."""
import gc

import pytest
import torch

import bench
from kv_cache_routing_sr_b200 import inputs, native
from tests.conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


def test_back_to_back_block_timing_small():
    xs = [inputs.make("tiny_4k", seed=s, device="cuda", max_ctx=512) for s in (1, 2, 3)]
    x = xs[0]
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    for fused in (False, True):
        ms, k = bench.time_back_to_back(native, dec, xs, x.tau, 6, 3, fused)
        gc.collect()
        assert k == 6 and ms > 0
    assert dec.workspace.device_error() == 0
    # the last of 3 graph steps runs on xs[2]: it must equal a fresh eager step
    x2 = xs[2]
    ref = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len).step(
        x2.q, x2.k_cache, x2.v_cache, x2.k0, x2.v0, x2.seq_lens, x2.tau)
    dec2 = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    bench.time_back_to_back(native, dec2, xs, x.tau, 3, 3, False)
    torch.cuda.synchronize()
    assert torch.equal(dec2.out.view(torch.int16), ref.view(torch.int16))


def test_isolated_step_graph_events_outlive_the_call():
    x = inputs.make("tiny_4k", seed=4, device="cuda", max_ctx=512)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    g, ev = bench._captured_steps(native, dec, x, x.tau, 3, None, True, False)
    del ev
    gc.collect()
    g.replay()
    torch.cuda.synchronize()
    assert all(e[0].elapsed_time(e[2]) > 0 for e in g.sr_events)


def test_append_back_to_back_small():
    """The back-to-back append timing: every input set's visits append at its
    last slots, the lengths end at the full context after the timed replay, the
    routing keeps the planted groups, and no device error is raised."""
    xs = [inputs.make("tiny_4k", seed=s, device="cuda", max_ctx=512) for s in (5, 6, 7)]
    x = xs[0]
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    steps = 7
    visits = -(-steps // len(xs))
    seqs = [bench.AppendSequence(native, inputs, xi, visits) for xi in xs]
    ms = bench.time_append_back_to_back(native, dec, xs, seqs, x.tau, steps, 3)
    gc.collect()
    assert ms > 0
    assert dec.workspace.device_error() == 0
    for i, (xi, a) in enumerate(zip(xs, seqs)):
        done = len(range(i, steps, len(xs)))  # this set's visits in one replay
        assert torch.equal(a.seq_lens, a.seq_saved + done)
        assert torch.equal(a.seq_saved, xi.seq_lens - visits)
    # the last step ran on set (steps - 1) % 3: its planted sinks are groups 0-3
    assert int(dec.active_list[0]) == 4
    assert dec.route_mask.cpu().tolist() == [1, 1, 1, 1, 0, 0, 0, 0]
