"""fp64 CPU oracle for SinkRouter routed decode attention (ctypes wrapper).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package. The
product path (``kv_cache_routing_sr_b200``) never imports it and shares no code
with it.

The arithmetic lives in ``sr_oracle.c`` (plain C, fp64). This module compiles
it with gcc, loads it, and marshals torch CPU tensors in and out. What each
function computes, and which passage of the pages it follows, is documented in
the C source:

* ``route``  -- per KV-head group cosine routing against the position-0 key
  (SinkRouter README, decode-time procedure list; routing controls).
* ``decode`` -- sink groups return the position-0 value; active groups run
  plain softmax attention over the whole cache (README decode list; pith.science
  review of arXiv 2604.16883, Figure 1 caption, eq. (1)).
* ``rope_append`` -- the step before: rotary embedding of the query and of the
  new key, cache append, position-0 capture (README decode list).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "sr_oracle.c")
LIBRARY = os.path.join(_HERE, "libsr_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the oracle with gcc into ``output`` and return its path."""
    cmd = ["gcc", *CFLAGS, source, "-o", output, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return output


def _needs_build(lib: str, src: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


class Oracle:
    """A loaded build of the oracle (the committed one, or a test's variant)."""

    def __init__(self, library: str = LIBRARY):
        self.path = library
        self._lib = ctypes.CDLL(library)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f64p = ctypes.POINTER(ctypes.c_double)
        ci = ctypes.c_int
        self._lib.sr_oracle_route.argtypes = [ci, ci, ci, ci, u16p, u16p, ctypes.c_double,
                                              u8p, i32p, f64p]
        self._lib.sr_oracle_route.restype = ci
        self._lib.sr_oracle_decode.argtypes = [ci, ci, ci, ci, ci, u16p, u16p, u16p, u16p,
                                               i32p, u8p, i32p, ci, f64p, f64p, ci]
        self._lib.sr_oracle_decode.restype = ci
        f32p = ctypes.POINTER(ctypes.c_float)
        self._lib.sr_oracle_rope_append.argtypes = [ci, ci, ci, ci, ci, ci, u16p, u16p, u16p, f32p, f32p, i32p,
                                                    u16p, u16p, u16p, u16p, u16p]
        self._lib.sr_oracle_rope_append.restype = ci

    @staticmethod
    def _bits(t: torch.Tensor):
        t = t.detach().to("cpu").contiguous()
        if t.dtype != torch.bfloat16:
            raise TypeError(f"oracle inputs are bf16, got {t.dtype}")
        v = t.view(torch.int16)
        return v, ctypes.cast(v.data_ptr(), ctypes.POINTER(ctypes.c_uint16))

    @staticmethod
    def _ptr(t: torch.Tensor, ctype):
        return ctypes.cast(t.data_ptr(), ctypes.POINTER(ctype))

    def route(self, q: torch.Tensor, k0: torch.Tensor, tau: float):
        """Route every KV-head group.

        q [B, Hq, d] bf16, k0 [B, Hkv, d] bf16. Returns (mask uint8 [B*Hkv],
        active_list int32 [1+B*Hkv], score float64 [B*Hkv]). Entries of
        active_list past 1+count are left at -1.
        """
        B, Hq, d = q.shape
        Hkv = k0.shape[1]
        qv, qp = self._bits(q)
        kv, kp = self._bits(k0)
        mask = torch.zeros(B * Hkv, dtype=torch.uint8)
        active = torch.full((1 + B * Hkv,), -1, dtype=torch.int32)
        score = torch.zeros(B * Hkv, dtype=torch.float64)
        st = self._lib.sr_oracle_route(B, Hq, Hkv, d, qp, kp, float(tau),
                                       self._ptr(mask, ctypes.c_uint8),
                                       self._ptr(active, ctypes.c_int32),
                                       self._ptr(score, ctypes.c_double))
        if st != 0:
            raise ValueError(f"sr_oracle_route failed with status {st}")
        return mask, active, score

    def decode(self, q, k_cache, v_cache, v0, seq_lens, mask, units=None, n_threads=1):
        """Routed decode attention in fp64.

        q [B,Hq,d], k_cache/v_cache [B,Hkv,Lmax,d], v0 [B,Hkv,d] (bf16);
        seq_lens [B] int32; mask [B*Hkv] uint8 (1 = sink). ``units`` restricts
        the work to those flat group indices (others stay NaN in the result).
        Returns (out float64 [B,Hq,d], p0 float64 [B,Hq]); p0 is NaN for sink
        heads.
        """
        B, Hq, d = q.shape
        Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
        qv, qp = self._bits(q)
        kv, kp = self._bits(k_cache)
        vv, vp = self._bits(v_cache)
        v0v, v0p = self._bits(v0)
        sl = seq_lens.detach().to("cpu", torch.int32).contiguous()
        mk = mask.detach().to("cpu", torch.uint8).contiguous()
        if units is None:
            up, nu = None, 0
        else:
            ut = torch.as_tensor(units, dtype=torch.int32).contiguous()
            up, nu = self._ptr(ut, ctypes.c_int32), int(ut.numel())
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float64)
        p0 = torch.full((B, Hq), float("nan"), dtype=torch.float64)
        st = self._lib.sr_oracle_decode(B, Hq, Hkv, d, Lmax, qp, kp, vp, v0p,
                                        self._ptr(sl, ctypes.c_int32),
                                        self._ptr(mk, ctypes.c_uint8),
                                        up, nu, self._ptr(out, ctypes.c_double),
                                        self._ptr(p0, ctypes.c_double), int(n_threads))
        if st != 0:
            raise ValueError(f"sr_oracle_decode failed with status {st}")
        return out, p0

    def rope_append(self, q_in, k_new, v_new, rope_cos, rope_sin, seq_lens, k_cache, v_cache, k0, v0):
        """The step before the scan, on CPU copies of the inputs: RoPE of q and
        of the new key at slot seq_lens[b], the append, the position-0 capture
        and the length update. q_in [B,Hq,d], k_new / v_new [B,Hkv,d] (bf16);
        rope_cos / rope_sin fp32 [max_pos, d/2]; seq_lens int32 [B]; caches
        [B,Hkv,Lmax,d], k0 / v0 [B,Hkv,d] (bf16). Returns (status, q_out, k_cache,
        v_cache, k0, v0, seq_lens): status 0 = ok, 1 = some slot out of range
        (that sequence untouched, its q_out rows zero)."""
        B, Hq, d = q_in.shape
        Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
        max_pos = rope_cos.shape[0]
        kc = k_cache.detach().to("cpu").contiguous().clone()
        vc = v_cache.detach().to("cpu").contiguous().clone()
        k0c = k0.detach().to("cpu").contiguous().clone()
        v0c = v0.detach().to("cpu").contiguous().clone()
        sl = seq_lens.detach().to("cpu", torch.int32).contiguous().clone()
        q_out = torch.empty((B, Hq, d), dtype=torch.bfloat16)
        cs = rope_cos.detach().to("cpu", torch.float32).contiguous()
        sn = rope_sin.detach().to("cpu", torch.float32).contiguous()
        qv, qp = self._bits(q_in)
        kv, kp = self._bits(k_new)
        vv, vp = self._bits(v_new)

        def u16(t):
            return ctypes.cast(t.view(torch.int16).data_ptr(), ctypes.POINTER(ctypes.c_uint16))

        st = self._lib.sr_oracle_rope_append(B, Hq, Hkv, d, Lmax, max_pos, qp, kp, vp,
                                             self._ptr(cs, ctypes.c_float), self._ptr(sn, ctypes.c_float),
                                             self._ptr(sl, ctypes.c_int32), u16(kc), u16(vc), u16(k0c), u16(v0c),
                                             u16(q_out))
        return st, q_out, kc, vc, k0c, v0c, sl


@dataclass
class OracleResult:
    mask: torch.Tensor
    active_list: torch.Tensor
    score: torch.Tensor
    out: torch.Tensor
    p0: torch.Tensor


_default = None


def load() -> Oracle:
    """The committed oracle, compiled on first use when missing or stale."""
    global _default
    if _default is None:
        if _needs_build(LIBRARY, SOURCE):
            build()
        _default = Oracle(LIBRARY)
    return _default


def route(q, k0, tau):
    return load().route(q, k0, tau)


def decode(q, k_cache, v_cache, v0, seq_lens, mask, units=None, n_threads=1):
    return load().decode(q, k_cache, v_cache, v0, seq_lens, mask, units, n_threads)


def routed_attention(q, k_cache, v_cache, k0, v0, seq_lens, tau, units=None, n_threads=1):
    """Route, then decode: the whole step the GPU path computes."""
    o = load()
    mask, active, score = o.route(q, k0, tau)
    out, p0 = o.decode(q, k_cache, v_cache, v0, seq_lens, mask, units, n_threads)
    return OracleResult(mask, active, score, out, p0)
