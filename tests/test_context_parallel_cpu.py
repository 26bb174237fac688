"""Context parallelism, host side (CPU): the sharding plan, the decomposition
it relies on (in the oracle's fp64 arithmetic), and the exchange on two gloo
ranks."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import oracle
from kv_cache_routing_sr_b200 import context_parallel as cp


@pytest.mark.parametrize("lens,R", [([131072], 8), ([7, 8, 100], 7), ([5], 5), ([65536, 99999, 131072, 70001], 3)])
def test_shard_bounds_partition_every_sequence(lens, R):
    bounds = cp.shard_bounds(lens, R)
    assert len(bounds) == R
    for b, L in enumerate(lens):
        spans = [bounds[r][b] for r in range(R)]
        assert spans[0][0] == 0 and spans[-1][1] == L
        for (s0, e0), (s1, e1) in zip(spans, spans[1:]):
            assert e0 == s1  # contiguous, disjoint
        sizes = [e - s for s, e in spans]
        assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_shard_bounds_refuse_short_sequences():
    with pytest.raises(ValueError):
        cp.shard_bounds([3, 100], 4)


def test_row_layout_is_aligned():
    for B, Hq in ((1, 32), (3, 1), (7, 9), (16384, 8)):
        n = B * Hq
        f = cp.row_floats(B, Hq)
        assert f % 4 == 0 and f >= n * 128 + n and f - (n * 128 + n) < 4


def test_shard_cache_copies_each_shard():
    B, Hkv, L = 2, 3, 10
    c = torch.arange(B * Hkv * L * 128, dtype=torch.float32).view(B, Hkv, L, 128).to(torch.bfloat16)
    bounds = cp.shard_bounds([10, 7], 3)
    for r in range(3):
        s = cp.shard_cache(c, bounds[r])
        for b, (s0, e0) in enumerate(bounds[r]):
            assert torch.equal(s[b, :, :e0 - s0], c[b, :, s0:e0])
            assert (s[b, :, e0 - s0:].float() == 0).all()


def test_lse_combination_of_shards_is_full_attention_in_fp64():
    """The identity the sharded step rests on, in the oracle's arithmetic: the
    oracle's outputs on each shard, combined with weights exp(lse_r - lse),
    equal the oracle's output on the whole cache (lse_r from the shard's scaled
    logits in fp64)."""
    g = torch.Generator().manual_seed(0)
    B, Hkv, M, L, R = 2, 2, 4, 50, 3
    q = torch.randn(B, Hkv * M, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, L, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, L, 128, generator=g).to(torch.bfloat16)
    lens = torch.tensor([50, 31], dtype=torch.int32)
    mask = torch.zeros(B * Hkv, dtype=torch.uint8)
    full, _ = oracle.decode(q, k, v, v[:, :, 0].contiguous(), lens, mask)
    bounds = cp.shard_bounds(lens.tolist(), R)
    outs, lses = [], []
    for r in range(R):
        ks, vs = cp.shard_cache(k, bounds[r]), cp.shard_cache(v, bounds[r])
        sl = torch.tensor([e - s for s, e in bounds[r]], dtype=torch.int32)
        o, _ = oracle.decode(q, ks, vs, vs[:, :, 0].contiguous(), sl, mask)
        outs.append(o)
        lse = torch.empty(B, Hkv * M, dtype=torch.float64)
        for b in range(B):
            for h in range(Hkv * M):
                logits = ks[b, h // M, :int(sl[b])].double() @ q[b, h].double() / 128 ** 0.5
                lse[b, h] = torch.logsumexp(logits, 0)
        lses.append(lse)
    lse = torch.stack(lses)
    wts = torch.exp(lse - torch.logsumexp(lse, 0))
    comb = (wts.unsqueeze(-1) * torch.stack(outs)).sum(0)
    assert (comb - full).abs().max().item() < 1e-12


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    stride = cp.row_floats(1, 32)
    row = torch.full((stride,), float(rank + 1))
    row[-1] = rank * 10.0
    gathered = torch.zeros(world * stride)
    cp.gather_rows(row, gathered, world)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, gathered.view(world, stride)[:, 0].tolist(), gathered.view(world, stride)[:, -1].tolist()))


def test_gather_rows_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, first, last in res:
        assert first == [1.0, 2.0] and last == [0.0, 10.0]  # rows in rank order on every rank


def test_gather_rows_single_rank_is_identity():
    row = torch.arange(8, dtype=torch.float32)
    assert torch.equal(cp.gather_rows(row, row, 1), row)
    out = torch.zeros(8)
    cp.gather_rows(row, out, 1)
    assert torch.equal(out, row)
