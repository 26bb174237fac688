"""sr_decode_attention_static_scratch against sr_decode_attention (GPU).

The static-scratch entry point serves callers that cannot allocate device
memory (a plugin that only receives its input and output buffers, a runtime
that forbids allocation on the decode path): the kernel's scratch is a fixed
array inside the library instead of a caller workspace. Its output must agree
with the workspace entry point, call after call, and oversized shapes must be
refused. This file is collected last on purpose, so that a run stopping at the
first failure has already run every other test; it also passes alone.
"""
import ctypes
import os
import re

import pytest
import torch

from kv_cache_routing_sr_b200 import inputs, native
from tests import gpu_helpers as H
from tests.conftest import cuda_available

gpu = [pytest.mark.gpu, pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]
SOURCE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "kv_cache_routing_sr_b200",
                      "csrc", "sr_static_scratch.cu")

CASES = [
    ("llama70b_ragged", dict(max_ctx=3000, poison_padding=True), 0),  # M = 8, ragged, NaN padding
    ("llava7b_mha", dict(max_ctx=1200, batch=3), 0),  # M = 1: split groups in the merge
    ("llama8b_128k", dict(max_ctx=6000), 5),  # M = 4, forced splits
    ("tiny_4k", {}, 0),
]


def _compare(x, got, ref, mask):
    """Sinks bit-exact; active units within the parity tolerances."""
    M = x.n_q_heads // x.n_kv_heads
    act = mask.view(x.batch, x.n_kv_heads).repeat_interleave(M, dim=1) == 0
    sink = ~act
    assert torch.equal(got[sink].view(torch.int16), ref[sink].view(torch.int16))
    if act.any():
        H.assert_active_close(got[act], ref[act].double(), "static scratch vs workspace entry point")


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("name,kw,n_splits", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_matches_workspace_entry_point(name, kw, n_splits):
    x = inputs.make(name, seed=21, device="cuda", **kw)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len, max_splits=n_splits)
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):  # two calls in a row: the shared array must not carry state over
        ref = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau, n_splits=n_splits).clone()
        out = torch.full_like(x.q, float("nan"))
        native.decode_attention_static_scratch(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens,
                                               dec.active_list, out, n_splits=n_splits, device_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"device error bits {int(err.item())} on call {call}"
        _compare(x, out.cpu(), ref.cpu(), dec.route_mask.cpu())
        # against the oracle as well, for the sampled units
        H.check_against_oracle(x, out.cpu(), dec.route_mask.cpu(),
                               units=[u for u in range(x.batch * x.n_kv_heads)][:4])


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_static_scratch_near_the_limit_and_allocates_nothing():
    """123 sequences x 8 KV heads x 8 query heads with automatic splits needs
    just under the array's 8 MiB; the result must match the workspace entry
    point, torch's allocator must see no change across calls, and one more
    sequence must be refused."""
    x = inputs.make("llama70b_ragged", seed=24, device="cuda", max_ctx=192, batch=123)
    dec = native.Decoder(x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len)
    ref = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau).clone()
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = torch.full_like(x.q, float("nan"))
    native.decode_attention_static_scratch(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, dec.active_list,
                                           out, device_error=err)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    for _ in range(2):
        native.decode_attention_static_scratch(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens,
                                               dec.active_list, out, device_error=err)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    assert int(err.item()) == 0
    _compare(x, out.cpu(), ref.cpu(), dec.route_mask.cpu())
    lib = native.load()
    fake = ctypes.c_void_p(0x10000)
    d = native.Dims(124, 64, 8, 128, 192)
    st = lib.sr_decode_attention_static_scratch(ctypes.byref(d), fake, fake, fake, None, fake, fake, fake, 0,
                                                fake, None, None)
    assert st == native.SR_ERR_WORKSPACE


def test_static_scratch_source_names_no_allocator():
    """The entry point's translation unit calls no allocating CUDA routine (a
    CPU check of the source; the GPU test above checks torch's allocator)."""
    src = open(SOURCE).read()
    code = re.sub(r"//[^\n]*", "", src)  # comments may mention the routines they avoid
    for name in ("cudaMalloc", "cudaFree", "cudaMallocAsync", "cudaMallocManaged", "cudaMallocHost",
                 "cudaHostAlloc", "cuMemAlloc", "malloc(", "new "):
        assert name not in code, f"{name} in sr_static_scratch.cu"


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_static_scratch_reports_device_errors():
    x = inputs.make("tiny_4k", seed=22, device="cuda", max_ctx=256)
    _, active = native.route(x.q, x.k0, x.tau)
    x.seq_lens.fill_(100_000)  # beyond Lmax: clamped and reported
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.decode_attention_static_scratch(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, active,
                                           device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & native.SR_DEVERR_SEQ_LEN
    x.seq_lens.fill_(256)
    native.decode_attention_static_scratch(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, active,
                                           device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0  # each call starts from a cleared error word


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_static_scratch_refuses_shapes_beyond_the_array():
    lib = native.load()
    # 1024 sequences x 8 KV heads with 8 query heads each needs ~38 MB of scratch
    d = native.Dims(1024, 64, 8, 128, 4096)
    fake = ctypes.c_void_p(0x10000)
    st = lib.sr_decode_attention_static_scratch(ctypes.byref(d), fake, fake, fake, None, fake, fake, fake, 0,
                                                fake, None, None)
    assert st == native.SR_ERR_WORKSPACE
    # a forced split count can also exceed it
    d = native.Dims(4, 64, 8, 128, 131072)
    st = lib.sr_decode_attention_static_scratch(ctypes.byref(d), fake, fake, fake, None, fake, fake, fake, 4096,
                                                fake, None, None)
    assert st == native.SR_ERR_WORKSPACE
