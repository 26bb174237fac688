"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same (bf16) inputs, and compare.

Tolerances. Route masks and active lists: bit-exact. Sink outputs: bit-exact
copies of v0. Active outputs (the specification's bar): max |gpu - oracle| <=
1e-2 and mean <= 1e-3, plus a relative-L2 bound per (sequence, head) of 1e-2
derived from the arithmetic: the kernel rounds the softmax weights to bf16
before the PV product (relative 2^-9 per weight, independent signs, so about
2^-9/sqrt(3) = 1.1e-3 relative on a sum of random values) and rounds the
output to bf16 (at most 2^-9 = 2e-3 relative); fp32 accumulation and exp2 add
about 1e-6. The sum, ~2.5e-3, is kept below 1e-2 with a 4x margin while a
missing or duplicated tile still breaks it (one 64-row tile out of 131072
rows moves the output by ~2% relative).
"""
from __future__ import annotations

import torch

import oracle
from kv_cache_routing_sr_b200 import native

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
REL_L2 = 1e-2


def gpu_step(x, n_splits=0, tau=None, decoder=None):
    B, Hq, Hkv, Lmax = x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len
    dec = decoder or native.Decoder(B, Hq, Hkv, Lmax, max_splits=n_splits)
    out = dec.step(x.q, x.k_cache, x.v_cache, x.k0, x.v0, x.seq_lens, x.tau if tau is None else tau,
                   n_splits=n_splits)
    torch.cuda.synchronize()
    return dec.route_mask.cpu(), dec.active_list.cpu(), out.cpu(), dec


def tau32(tau: float) -> float:
    """The GPU compares in fp32: hand the oracle the same fp32 threshold."""
    return float(torch.tensor(tau, dtype=torch.float32))


def unit_subproblem(x, u):
    """The one-unit problem (B=1, Hkv=1) holding unit u's data, on the CPU."""
    Hkv, M = x.n_kv_heads, x.n_q_heads // x.n_kv_heads
    b, g = divmod(u, Hkv)
    q = x.q[b:b + 1, g * M:(g + 1) * M].cpu()
    k = x.k_cache[b:b + 1, g:g + 1].cpu()
    v = x.v_cache[b:b + 1, g:g + 1].cpu()
    k0 = x.k0[b:b + 1, g:g + 1].cpu()
    v0 = x.v0[b:b + 1, g:g + 1].cpu()
    sl = x.seq_lens[b:b + 1].cpu()
    return q, k, v, k0, v0, sl


def oracle_units(x, units, mask, n_threads=8):
    """Oracle outputs [len(units), M, d] (fp64) for the listed units under the
    given route mask (one sub-problem per unit, computed in parallel)."""
    outs = []
    for u in units:
        q, k, v, k0, v0, sl = unit_subproblem(x, u)
        m = mask[u:u + 1].to(torch.uint8)
        o, _ = oracle.decode(q, k, v, v0, sl, m, n_threads=1)
        outs.append(o[0])
    return torch.stack(outs) if outs else torch.empty(0)


def oracle_full(x, tau, n_threads=8):
    cpu = x.to("cpu")
    return oracle.routed_attention(cpu.q, cpu.k_cache, cpu.v_cache, cpu.k0, cpu.v0, cpu.seq_lens, tau32(tau),
                                   n_threads=n_threads)


def assert_route_equal(mask_gpu, active_gpu, mask_ref, active_ref):
    assert torch.equal(mask_gpu, mask_ref), "route mask differs from the oracle"
    n = int(active_ref[0])
    assert int(active_gpu[0]) == n, f"active count {int(active_gpu[0])} != {n}"
    assert torch.equal(active_gpu[1:1 + n], active_ref[1:1 + n]), "active list differs from the oracle"


def assert_sink_exact(out_gpu_unit, v0_unit):
    """out_gpu_unit [M, d] bf16 must equal v0 [d] bit for bit in every head."""
    exp = v0_unit.cpu().view(torch.int16).expand_as(out_gpu_unit.view(torch.int16))
    assert torch.equal(out_gpu_unit.view(torch.int16), exp), "sink output is not v0 bit for bit"


def active_error(out_gpu, ref):
    """(max abs, mean abs, worst per-head relative L2) of bf16 outputs vs fp64."""
    g = out_gpu.double().reshape(-1, out_gpu.shape[-1])
    r = ref.double().reshape(-1, ref.shape[-1])
    diff = (g - r)
    rel = (diff.norm(dim=-1) / r.norm(dim=-1).clamp_min(1e-30)).max().item()
    return diff.abs().max().item(), diff.abs().mean().item(), rel


def assert_active_close(out_gpu, ref, what=""):
    assert torch.isfinite(out_gpu.float()).all(), f"non-finite output {what}"
    mx, mean, rel = active_error(out_gpu, ref)
    assert mx <= MAX_ABS, f"max abs error {mx} {what}"
    assert mean <= MEAN_ABS, f"mean abs error {mean} {what}"
    assert rel <= REL_L2, f"relative L2 error {rel} {what}"
    return mx, mean, rel


def check_against_oracle(x, out_gpu, mask_gpu, units=None, what=""):
    """Compare every listed unit (default: all) of a GPU result with the oracle:
    sinks bit-exact, active units within tolerance."""
    Hkv, M = x.n_kv_heads, x.n_q_heads // x.n_kv_heads
    U = x.batch * Hkv
    units = list(range(U)) if units is None else list(units)
    act = [u for u in units if mask_gpu[u] == 0]
    for u in units:
        if mask_gpu[u]:
            b, g = divmod(u, Hkv)
            assert_sink_exact(out_gpu[b, g * M:(g + 1) * M], x.v0[b, g])
    if act:
        ref = oracle_units(x, act, mask_gpu)
        got = torch.stack([out_gpu[u // Hkv, (u % Hkv) * M:(u % Hkv + 1) * M] for u in act])
        return assert_active_close(got, ref, what)
    return None
