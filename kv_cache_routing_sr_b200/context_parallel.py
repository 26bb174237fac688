"""Context parallelism: one long sequence's decode attention spread over GPUs.

Every GPU (rank) holds one contiguous shard of each sequence's KV cache. One
decode step on every rank:

1. routing, identical on every rank (the same q, k0 and tau give the same
   active list; nothing is exchanged);
2. ``sr_decode_attention_partial`` over the local shard: per head the fp32
   normalised output o_r and the log-sum-exp lse_r of its logits, written as one
   packed row [o (B*Hq*128) | lse (B*Hq), padded to 4 floats];
3. one all-gather of the rows (NCCL over NVLink: B*Hq*129*4 bytes per rank,
   16.5 KB for a Llama-3.1-8B-shaped layer);
4. ``sr_combine_partials`` on the gathered rows: out = sum_r exp(lse_r - lse) o_r
   with lse = log sum_r exp(lse_r), which is softmax attention over the whole
   sequence; every rank ends with the full output.

This is the cross-GPU form of the split-K reduction the SinkRouter README
describes inside one kernel (decode-time procedure list: split-K flash decoding
with an in-kernel reduction): the partials of a GPU's shard are reduced across
GPUs by the same log-sum-exp rule.

``emulate`` runs the R ranks' shards one after another on one GPU, writing each
shard's row straight into the gathered buffer (the exchange is then a no-op),
and combines them: the same kernels and buffers as the multi-GPU step, without
any rank waiting for another.
"""
from __future__ import annotations

import torch

from . import native


def shard_bounds(seq_lens, world: int):
    """[rank][b] -> (start, end): rank r holds positions
    [r*L_b // R, (r+1)*L_b // R) of sequence b, so the shards are contiguous,
    disjoint, cover [0, L_b) and differ in size by at most one. Every shard must
    hold at least one position (L_b >= R)."""
    lens = [int(x) for x in seq_lens]
    if world < 1:
        raise ValueError("world size must be >= 1")
    if any(L < world for L in lens):
        raise ValueError(f"every sequence needs at least {world} positions for {world} shards")
    return [[(r * L // world, (r + 1) * L // world) for L in lens] for r in range(world)]


def row_floats(batch: int, n_q_heads: int) -> int:
    """Floats of one rank's packed row: o [B*Hq*128] then lse [B*Hq], padded
    so that consecutive rows stay 16-byte aligned."""
    n = batch * n_q_heads
    return n * native.HEAD_DIM + (n + 3) // 4 * 4


def shard_cache(cache: torch.Tensor, bounds_r) -> torch.Tensor:
    """A rank's contiguous shard [B, Hkv, max shard length, 128] of a full
    cache [B, Hkv, Lmax, 128] (positions past a sequence's shard are zero)."""
    B, Hkv, _, d = cache.shape
    ls = max(e - s for s, e in bounds_r)
    out = torch.zeros((B, Hkv, ls, d), dtype=cache.dtype, device=cache.device)
    for b, (s, e) in enumerate(bounds_r):
        out[b, :, :e - s] = cache[b, :, s:e]
    return out


def gather_rows(row: torch.Tensor, gathered: torch.Tensor, world: int, group=None):
    """All-gather of the ranks' rows into gathered [world * len(row)] in rank
    order (the exchange step; no-op for one rank, where gathered is row)."""
    if world == 1:
        if gathered.data_ptr() != row.data_ptr():
            gathered.copy_(row)
        return gathered
    import torch.distributed as dist
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, row, group=group)
    else:
        dist.all_gather(list(gathered.view(world, -1).unbind(0)), row, group=group)
    return gathered


class ContextParallelDecoder:
    """One rank's buffers and the four steps above. k_shard / v_shard are this
    rank's [B, Hkv, shard_max_len, 128] caches and shard_lens [B] int32 (device)
    the lengths of its shards; q, k0, v0 and tau are the same on every rank."""

    def __init__(self, batch, n_q_heads, n_kv_heads, shard_max_len, world: int = 1, group=None, device="cuda",
                 max_splits: int = 0):
        self.B, self.Hq, self.world, self.group = batch, n_q_heads, world, group
        self.dec = native.Decoder(batch, n_q_heads, n_kv_heads, shard_max_len, max_splits=max_splits, device=device)
        self.stride = row_floats(batch, n_q_heads)
        self.gathered = torch.zeros(world * self.stride, dtype=torch.float32, device=device)
        self.row = self.gathered[:self.stride] if world == 1 else torch.zeros(self.stride, dtype=torch.float32,
                                                                               device=device)

    def _views(self, buf):
        n = self.B * self.Hq
        return (buf[:n * native.HEAD_DIM].view(self.B, self.Hq, native.HEAD_DIM),
                buf[n * native.HEAD_DIM:n * native.HEAD_DIM + n].view(self.B, self.Hq))

    def local(self, q, k_shard, v_shard, k0, v0, shard_lens, tau, n_splits: int = 0, row=None):
        """Steps 1 and 2: route, then the partial scan into `row` (default:
        this rank's row)."""
        row = self.row if row is None else row
        native.route(q, k0, tau, self.dec.route_mask, self.dec.active_list)
        o, lse = self._views(row)
        native.decode_attention_partial(q, k_shard, v_shard, k0, v0, shard_lens, self.dec.active_list, o, lse,
                                        n_splits, self.dec.workspace)

    def finish(self):
        """Steps 3 and 4: exchange the rows and combine them into self.out."""
        gather_rows(self.row, self.gathered, self.world, self.group)
        n = self.B * self.Hq
        return native.combine_partials(self.gathered, self.gathered[n * native.HEAD_DIM:], self.stride, self.world,
                                       self.B, self.Hq, out=self.dec.out)

    def step(self, q, k_shard, v_shard, k0, v0, shard_lens, tau, n_splits: int = 0):
        self.local(q, k_shard, v_shard, k0, v0, shard_lens, tau, n_splits)
        return self.finish()

    @property
    def out(self):
        return self.dec.out


def emulate(q, k_cache, v_cache, k0, v0, seq_lens, tau, world: int, n_splits: int = 0):
    """All `world` ranks' shards on this GPU, one after another, each writing
    its row of the gathered buffer, then the combine. Returns (out, decoder)."""
    B, Hq, _ = q.shape
    Hkv = k_cache.shape[1]
    bounds = shard_bounds(seq_lens.tolist(), world)
    shards = []
    for r in range(world):
        lens = torch.tensor([e - s for s, e in bounds[r]], dtype=torch.int32, device=q.device)
        shards.append((shard_cache(k_cache, bounds[r]), shard_cache(v_cache, bounds[r]), lens))
    smax = max(k.shape[2] for k, _, _ in shards)
    # one decoder with every rank's row: each shard's scan writes its row of the
    # gathered buffer in place, so the exchange (finish) is never needed
    cp = ContextParallelDecoder(B, Hq, Hkv, smax, world=world, device=q.device, max_splits=n_splits)
    for r, (ks, vs, lens) in enumerate(shards):
        cp.local(q, ks, vs, k0, v0, lens, tau, n_splits, row=cp.gathered[r * cp.stride:(r + 1) * cp.stride])
    n = B * Hq
    out = native.combine_partials(cp.gathered, cp.gathered[n * native.HEAD_DIM:], cp.stride, world, B, Hq,
                                  out=cp.dec.out)
    return out, cp
