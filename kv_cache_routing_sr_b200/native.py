"""ctypes binding of libsinkrouter.so (the C ABI in include/sinkrouter.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels. torch provides device memory and the current stream. There is no
CPU fallback: a missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import functools
import os

import torch

from . import build as _build

LIBRARY = _build.LIBRARY

SR_OK, SR_ERR_INVALID_ARG, SR_ERR_UNSUPPORTED, SR_ERR_WORKSPACE, SR_ERR_CUDA = range(5)
SR_DEVERR_SEQ_LEN, SR_DEVERR_ACTIVE_LIST, SR_DEVERR_TIMEOUT = 1, 2, 4
SR_MAX_UNITS = 16384
SR_MAX_SPLITS = 4096
HEAD_DIM = 128


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_seq_len", ctypes.c_int32)]


class SinkRouterError(RuntimeError):
    def __init__(self, fn: str, status: int, lib):
        msg = lib.sr_status_string(status).decode()
        if status == SR_ERR_CUDA:
            msg += " -- " + lib.sr_last_cuda_error().decode()
        super().__init__(f"{fn}: {msg}")
        self.status = status


_lib = None

EXPORTS = ["sr_route", "sr_decode_workspace_bytes", "sr_workspace_init", "sr_decode_attention",
           "sr_status_string", "sr_get_device_error", "sr_clear_device_error", "sr_decode_grid_size",
           "sr_last_cuda_error", "sr_decode_attention_static_scratch", "sr_route_decode_attention",
           "sr_decode_attention_lse", "sr_rope_append_route", "sr_decode_attention_partial",
           "sr_combine_partials", "sr_selftest_bounded_wait", "sr_position0_weight"]


def load(path: str | None = None):
    """Load (once) and type the library: `path`, else the file named by the
    SINKROUTER_LIBRARY environment variable (another build of the same
    sources), else the in-tree library, which is compiled first if it is
    absent (nvcc, sm_100a). Any other missing path, or a failed compile,
    raises: there is no other implementation to fall back to."""
    global _lib
    if _lib is not None:
        return _lib
    if path is None:
        path = os.environ.get("SINKROUTER_LIBRARY") or LIBRARY
    if not os.path.exists(path) and os.path.abspath(path) == os.path.abspath(LIBRARY):
        from . import build as _build
        try:
            _build.build()
        except Exception as e:
            raise RuntimeError(f"libsinkrouter.so is missing and compiling it failed: {e}") from e
    if not os.path.exists(path):
        raise RuntimeError(f"libsinkrouter.so not found at {path}: build it with "
                           "`python -m kv_cache_routing_sr_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, i32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    dp = ctypes.POINTER(Dims)
    lib.sr_route.argtypes = [dp, vp, vp, ctypes.c_float, vp, vp, vp]
    lib.sr_route.restype = ctypes.c_int
    lib.sr_decode_workspace_bytes.argtypes = [dp, i32]
    lib.sr_decode_workspace_bytes.restype = u64
    lib.sr_workspace_init.argtypes = [vp, u64, vp]
    lib.sr_workspace_init.restype = ctypes.c_int
    lib.sr_decode_attention.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, u64, vp]
    lib.sr_decode_attention.restype = ctypes.c_int
    lib.sr_status_string.argtypes = [ctypes.c_int]
    lib.sr_status_string.restype = ctypes.c_char_p
    lib.sr_get_device_error.argtypes = [vp, ctypes.POINTER(i32), vp]
    lib.sr_get_device_error.restype = ctypes.c_int
    lib.sr_clear_device_error.argtypes = [vp, vp]
    lib.sr_clear_device_error.restype = ctypes.c_int
    lib.sr_decode_grid_size.argtypes = []
    lib.sr_decode_grid_size.restype = i32
    lib.sr_last_cuda_error.argtypes = []
    lib.sr_last_cuda_error.restype = ctypes.c_char_p
    lib.sr_decode_attention_static_scratch.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp]
    lib.sr_decode_attention_static_scratch.restype = ctypes.c_int
    lib.sr_route_decode_attention.argtypes = [dp, vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, vp, vp, vp, vp,
                                              u64, vp]
    lib.sr_route_decode_attention.restype = ctypes.c_int
    lib.sr_decode_attention_lse.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, u64, vp]
    lib.sr_decode_attention_lse.restype = ctypes.c_int
    lib.sr_position0_weight.argtypes = [dp, vp, vp, vp, vp, vp]
    lib.sr_position0_weight.restype = ctypes.c_int
    lib.sr_rope_append_route.argtypes = [dp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                         vp, vp, vp]
    lib.sr_rope_append_route.restype = ctypes.c_int
    lib.sr_decode_attention_partial.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, u64, vp]
    lib.sr_decode_attention_partial.restype = ctypes.c_int
    lib.sr_combine_partials.argtypes = [dp, i32, vp, vp, ctypes.c_int64, vp, vp]
    lib.sr_combine_partials.restype = ctypes.c_int
    lib.sr_selftest_bounded_wait.argtypes = [i32, vp, vp, vp]
    lib.sr_selftest_bounded_wait.restype = ctypes.c_int
    _lib = lib
    return lib


def _on_tensor_device(fn):
    """Run fn with the device of its first (tensor) argument current: the
    library launches on the current device, and the default stream passed to it
    must be that device's."""
    @functools.wraps(fn)
    def wrapper(t, *args, **kwargs):
        with torch.cuda.device(t.device):
            return fn(t, *args, **kwargs)
    return wrapper


def _check(fn: str, status: int):
    if status != SR_OK:
        raise SinkRouterError(fn, status, load())


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def dims_of(batch: int, n_q_heads: int, n_kv_heads: int, max_seq_len: int, head_dim: int = HEAD_DIM) -> Dims:
    return Dims(batch, n_q_heads, n_kv_heads, head_dim, max_seq_len)


def workspace_bytes(batch, n_q_heads, n_kv_heads, max_seq_len, max_splits: int = 0) -> int:
    d = dims_of(batch, n_q_heads, n_kv_heads, max_seq_len)
    n = load().sr_decode_workspace_bytes(ctypes.byref(d), int(max_splits))
    if n == 0:
        raise ValueError("unsupported dims or max_splits for the decode workspace")
    return int(n)


class Workspace:
    """A zero-initialised decode workspace in torch-allocated device memory,
    usable from any stream once constructed."""

    def __init__(self, batch, n_q_heads, n_kv_heads, max_seq_len, max_splits: int = 0, device=None):
        self.nbytes = workspace_bytes(batch, n_q_heads, n_kv_heads, max_seq_len, max_splits)
        self.buffer = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buffer.data_ptr()) % 256
        self.view = self.buffer[off:off + self.nbytes]
        with torch.cuda.device(self.buffer.device):
            _check("sr_workspace_init", load().sr_workspace_init(ctypes.c_void_p(self.view.data_ptr()),
                                                                 self.nbytes, _stream()))
            # the zeroing must be complete before any stream uses the workspace
            # (side streams do not wait for the stream it was issued on)
            torch.cuda.current_stream().synchronize()

    @property
    def ptr(self) -> int:
        return self.view.data_ptr()

    def device_error(self) -> int:
        code = ctypes.c_int32(0)
        with torch.cuda.device(self.buffer.device):
            _check("sr_get_device_error", load().sr_get_device_error(ctypes.c_void_p(self.ptr),
                                                                     ctypes.byref(code), _stream()))
        return int(code.value)

    def clear_device_error(self):
        with torch.cuda.device(self.buffer.device):
            _check("sr_clear_device_error", load().sr_clear_device_error(ctypes.c_void_p(self.ptr), _stream()))


@_on_tensor_device
def route(q: torch.Tensor, k0: torch.Tensor, tau: float, route_mask=None, active_list=None, stream=None):
    """sr_route: returns (route_mask uint8 [B*Hkv], active_list int32 [1+B*Hkv])."""
    B, Hq, d = q.shape
    Hkv = k0.shape[1]
    if route_mask is None:
        route_mask = torch.empty(B * Hkv, dtype=torch.uint8, device=q.device)
    if active_list is None:
        active_list = torch.empty(1 + B * Hkv, dtype=torch.int32, device=q.device)
    dims = dims_of(B, Hq, Hkv, 1, d)
    st = load().sr_route(ctypes.byref(dims), _dev(q, "q", torch.bfloat16), _dev(k0, "k0", torch.bfloat16),
                         float(tau), _dev(route_mask, "route_mask", torch.uint8),
                         _dev(active_list, "active_list", torch.int32), _stream(stream))
    _check("sr_route", st)
    return route_mask, active_list


@_on_tensor_device
def decode_attention(q, k_cache, v_cache, k0, v0, seq_lens, active_list, out=None, n_splits: int = 0,
                     workspace: Workspace | None = None, stream=None, lse=None):
    """sr_decode_attention: returns out bf16 [B, Hq, 128]. With ``lse`` (an fp32
    CUDA tensor [B, Hq]) it calls sr_decode_attention_lse, which also writes the
    per-head log-sum-exp of the logits (NaN for sink heads)."""
    B, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = Workspace(B, Hq, Hkv, Lmax, n_splits, device=q.device)
    dims = dims_of(B, Hq, Hkv, Lmax, d)
    k0p = _dev(k0, "k0", torch.bfloat16) if k0 is not None else None
    common = (ctypes.byref(dims), _dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
              _dev(v_cache, "v_cache", torch.bfloat16), k0p, _dev(v0, "v0", torch.bfloat16),
              _dev(seq_lens, "seq_lens", torch.int32), _dev(active_list, "active_list", torch.int32),
              int(n_splits), _dev(out, "out", torch.bfloat16))
    tail = (ctypes.c_void_p(workspace.ptr), workspace.nbytes, _stream(stream))
    if lse is None:
        _check("sr_decode_attention", load().sr_decode_attention(*common, *tail))
    else:
        _check("sr_decode_attention_lse",
               load().sr_decode_attention_lse(*common, _dev(lse, "lse", torch.float32), *tail))
    return out


@_on_tensor_device
def position0_weight(q, k_cache, lse, p0=None, stream=None):
    """sr_position0_weight: p0 fp32 [B, Hq], the full-attention weight of
    position 0 of every head, from the lse of sr_decode_attention_lse."""
    B, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if p0 is None:
        p0 = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    dims = dims_of(B, Hq, Hkv, Lmax, d)
    _check("sr_position0_weight",
           load().sr_position0_weight(ctypes.byref(dims), _dev(q, "q", torch.bfloat16),
                                      _dev(k_cache, "k_cache", torch.bfloat16), _dev(lse, "lse", torch.float32),
                                      _dev(p0, "p0", torch.float32), _stream(stream)))
    return p0


@_on_tensor_device
def decode_attention_partial(q, k_cache, v_cache, k0, v0, seq_lens, active_list, o_part=None, lse_part=None,
                             n_splits: int = 0, workspace: Workspace | None = None, stream=None):
    """sr_decode_attention_partial: the scan over this cache's positions with
    fp32 normalised outputs o_part [B, Hq, 128] and natural-log lse_part [B, Hq]
    (NaN for sink heads), ready for combine_partials. Returns (o_part, lse_part)."""
    B, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if o_part is None:
        o_part = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = Workspace(B, Hq, Hkv, Lmax, n_splits, device=q.device)
    dims = dims_of(B, Hq, Hkv, Lmax, d)
    k0p = _dev(k0, "k0", torch.bfloat16) if k0 is not None else None
    st = load().sr_decode_attention_partial(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
        _dev(v_cache, "v_cache", torch.bfloat16), k0p, _dev(v0, "v0", torch.bfloat16),
        _dev(seq_lens, "seq_lens", torch.int32), _dev(active_list, "active_list", torch.int32), int(n_splits),
        _dev(o_part, "o_part", torch.float32), _dev(lse_part, "lse_part", torch.float32),
        ctypes.c_void_p(workspace.ptr), workspace.nbytes, _stream(stream))
    _check("sr_decode_attention_partial", st)
    return o_part, lse_part


@_on_tensor_device
def combine_partials(o_parts, lse_parts, part_stride: int, n_parts: int, batch: int, n_q_heads: int, out=None,
                     stream=None):
    """sr_combine_partials over n_parts parts laid out part_stride floats apart:
    o_parts / lse_parts are fp32 CUDA tensors whose storage starts at part 0's
    o_part / lse_part. Returns out bf16 [B, Hq, 128]."""
    if out is None:
        out = torch.empty((batch, n_q_heads, HEAD_DIM), dtype=torch.bfloat16, device=o_parts.device)
    for t, name in ((o_parts, "o_parts"), (lse_parts, "lse_parts")):
        if not t.is_cuda or t.dtype != torch.float32:
            raise ValueError(f"{name} must be a float32 CUDA tensor")
    dims = dims_of(batch, n_q_heads, n_q_heads, 1)  # only B, Hq and head_dim are read
    st = load().sr_combine_partials(ctypes.byref(dims), int(n_parts), o_parts.data_ptr(), lse_parts.data_ptr(),
                                    int(part_stride), _dev(out, "out", torch.bfloat16), _stream(stream))
    _check("sr_combine_partials", st)
    return out


@_on_tensor_device
def decode_attention_static_scratch(q, k_cache, v_cache, k0, v0, seq_lens, active_list, out=None,
                                    n_splits: int = 0, device_error=None, stream=None):
    """sr_decode_attention_static_scratch: the decode step with the library's
    fixed scratch array instead of a workspace (no device allocation by the
    library). ``device_error``: optional int32 CUDA tensor of one element that
    receives the launch's device error bits. Returns out bf16 [B, Hq, 128]."""
    B, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    dims = dims_of(B, Hq, Hkv, Lmax, d)
    k0p = _dev(k0, "k0", torch.bfloat16) if k0 is not None else None
    errp = _dev(device_error, "device_error", torch.int32) if device_error is not None else None
    st = load().sr_decode_attention_static_scratch(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
        _dev(v_cache, "v_cache", torch.bfloat16), k0p, _dev(v0, "v0", torch.bfloat16),
        _dev(seq_lens, "seq_lens", torch.int32), _dev(active_list, "active_list", torch.int32),
        int(n_splits), _dev(out, "out", torch.bfloat16), errp, _stream(stream))
    _check("sr_decode_attention_static_scratch", st)
    return out


@_on_tensor_device
def route_decode_attention(q, k_cache, v_cache, k0, v0, seq_lens, tau, out=None, route_mask=None,
                           active_list=None, n_splits: int = 0, workspace: Workspace | None = None, stream=None):
    """sr_route_decode_attention: routing and decode in one launch. Returns out;
    route_mask / active_list (optional tensors) receive the route result."""
    B, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = Workspace(B, Hq, Hkv, Lmax, n_splits, device=q.device)
    dims = dims_of(B, Hq, Hkv, Lmax, d)
    mp = _dev(route_mask, "route_mask", torch.uint8) if route_mask is not None else None
    ap = _dev(active_list, "active_list", torch.int32) if active_list is not None else None
    st = load().sr_route_decode_attention(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
        _dev(v_cache, "v_cache", torch.bfloat16), _dev(k0, "k0", torch.bfloat16), _dev(v0, "v0", torch.bfloat16),
        _dev(seq_lens, "seq_lens", torch.int32), float(tau), int(n_splits), mp, ap,
        _dev(out, "out", torch.bfloat16), ctypes.c_void_p(workspace.ptr), workspace.nbytes, _stream(stream))
    _check("sr_route_decode_attention", st)
    return out


@_on_tensor_device
def rope_append_route(q_in, k_new, v_new, rope_cos, rope_sin, seq_lens, k_cache, v_cache, k0, v0, tau,
                      q_out=None, route_mask=None, active_list=None, device_error=None, stream=None):
    """sr_rope_append_route: RoPE of the query and the new key at slot
    seq_lens[b], append of the new key / value, position-0 capture, routing and
    the length update, in one launch. Updates k_cache, v_cache, k0, v0 and
    seq_lens in place; returns (q_out, route_mask, active_list). q_out may be
    q_in (rotated in place)."""
    B, Hq, d = q_in.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if q_out is None:
        q_out = torch.empty_like(q_in)
    if route_mask is None:
        route_mask = torch.empty(B * Hkv, dtype=torch.uint8, device=q_in.device)
    if active_list is None:
        active_list = torch.empty(1 + B * Hkv, dtype=torch.int32, device=q_in.device)
    if rope_cos.shape != rope_sin.shape or rope_cos.dim() != 2 or rope_cos.shape[1] != d // 2:
        raise ValueError("rope_cos / rope_sin must both be [max_pos, head_dim / 2]")
    err = 0 if device_error is None else _dev(device_error, "device_error", torch.int32)
    dims = dims_of(B, Hq, Hkv, Lmax, d)
    st = load().sr_rope_append_route(
        ctypes.byref(dims), _dev(q_in, "q_in", torch.bfloat16), _dev(k_new, "k_new", torch.bfloat16),
        _dev(v_new, "v_new", torch.bfloat16), _dev(rope_cos, "rope_cos", torch.float32),
        _dev(rope_sin, "rope_sin", torch.float32), int(rope_cos.shape[0]), _dev(seq_lens, "seq_lens", torch.int32),
        _dev(k_cache, "k_cache", torch.bfloat16), _dev(v_cache, "v_cache", torch.bfloat16),
        _dev(k0, "k0", torch.bfloat16), _dev(v0, "v0", torch.bfloat16), float(tau),
        _dev(q_out, "q_out", torch.bfloat16), _dev(route_mask, "route_mask", torch.uint8),
        _dev(active_list, "active_list", torch.int32), err or None, _stream(stream))
    _check("sr_rope_append_route", st)
    return q_out, route_mask, active_list


def selftest_bounded_wait(limit_us: int, device="cuda", stream=None):
    """sr_selftest_bounded_wait: a wait on an mbarrier nothing arrives on, with
    a bound of limit_us. Returns (status, waited_ns) after synchronising; the
    expected status is SR_DEVERR_TIMEOUT."""
    status = torch.full((1,), -1, dtype=torch.int32, device=device)
    waited = torch.zeros(1, dtype=torch.int64, device=device)
    with torch.cuda.device(status.device):
        _check("sr_selftest_bounded_wait",
               load().sr_selftest_bounded_wait(int(limit_us), _dev(status, "status", torch.int32),
                                               _dev(waited, "waited_ns", torch.int64), _stream(stream)))
    torch.cuda.synchronize(device)
    return int(status.item()), int(waited.item())


def grid_size() -> int:
    return int(load().sr_decode_grid_size())


class Decoder:
    """Owns the route buffers and the workspace for repeated decode steps of
    one layer shape: step() = sr_route then sr_decode_attention, both async on
    the current stream."""

    def __init__(self, batch, n_q_heads, n_kv_heads, max_seq_len, max_splits: int = 0, device="cuda"):
        self.shape = (batch, n_q_heads, n_kv_heads, max_seq_len)
        U = batch * n_kv_heads
        self.route_mask = torch.empty(U, dtype=torch.uint8, device=device)
        self.active_list = torch.empty(1 + U, dtype=torch.int32, device=device)
        self.out = torch.empty(batch, n_q_heads, HEAD_DIM, dtype=torch.bfloat16, device=device)
        self.workspace = Workspace(batch, n_q_heads, n_kv_heads, max_seq_len, max_splits, device=device)

    def step(self, q, k_cache, v_cache, k0, v0, seq_lens, tau, n_splits: int = 0, stream=None):
        route(q, k0, tau, self.route_mask, self.active_list, stream)
        decode_attention(q, k_cache, v_cache, k0, v0, seq_lens, self.active_list, self.out, n_splits,
                         self.workspace, stream)
        return self.out

    def append_step(self, q_in, k_new, v_new, rope_cos, rope_sin, k_cache, v_cache, k0, v0, seq_lens, tau,
                    n_splits: int = 0, device_error=None, stream=None):
        """A whole decode step from the un-rotated projections:
        sr_rope_append_route (RoPE, append, capture, route, lengths) then
        sr_decode_attention on the rotated query. The caches, k0 / v0 and
        seq_lens are updated in place; the rotated query is kept in self.q."""
        if getattr(self, "q", None) is None or self.q.shape != q_in.shape:
            self.q = torch.empty_like(q_in)
        rope_append_route(q_in, k_new, v_new, rope_cos, rope_sin, seq_lens, k_cache, v_cache, k0, v0, tau,
                          self.q, self.route_mask, self.active_list, device_error, stream)
        decode_attention(self.q, k_cache, v_cache, k0, v0, seq_lens, self.active_list, self.out, n_splits,
                         self.workspace, stream)
        return self.out

    def step_fused(self, q, k_cache, v_cache, k0, v0, seq_lens, tau, n_splits: int = 0, stream=None):
        """The same step in one launch (sr_route_decode_attention)."""
        route_decode_attention(q, k_cache, v_cache, k0, v0, seq_lens, tau, self.out, self.route_mask,
                               self.active_list, n_splits, self.workspace, stream)
        return self.out


class StepGraph:
    """One decode step captured in a CUDA graph: sr_route then
    sr_decode_attention (either may be left out) on fixed tensors, replayed with
    one graph launch. The programmatic dependency between the two kernels is
    kept as a graph edge, and the host cost per step is a single launch.

    The tensors are bound at capture: replay reads whatever they hold then."""

    def __init__(self, decoder: "Decoder", q, k_cache, v_cache, k0, v0, seq_lens, tau, n_splits: int = 0,
                 with_route: bool = True, with_decode: bool = True):
        self.decoder = decoder
        self.graph = torch.cuda.CUDAGraph()
        args = (q, k_cache, v_cache, k0, v0, seq_lens)

        def body():
            if with_route:
                route(q, k0, tau, decoder.route_mask, decoder.active_list)
            if with_decode:
                decode_attention(q, k_cache, v_cache, k0, v0, seq_lens, decoder.active_list, decoder.out,
                                 n_splits, decoder.workspace)

        side = torch.cuda.Stream(device=q.device)
        side.wait_stream(torch.cuda.current_stream(q.device))
        with torch.cuda.stream(side):  # warm-up outside the capture (module load, attributes)
            decoder.step(*args, tau, n_splits)
        torch.cuda.current_stream(q.device).wait_stream(side)
        with torch.cuda.graph(self.graph):
            body()
        self._args = args  # keep the bound tensors alive as long as the graph

    def replay(self):
        self.graph.replay()
        return self.decoder.out
