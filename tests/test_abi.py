"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, and its host-side validation rejects bad arguments before any
CUDA call (so these run on a CPU-only machine)."""
import ctypes
import os
import re

import pytest

from kv_cache_routing_sr_b200 import build, native

HEADER = os.path.join(build.INCLUDE, "sinkrouter.h")
FAKE = 0x10000  # aligned, never dereferenced: validation fails before any launch


@pytest.fixture(scope="module")
def lib():
    if build.needs_build():
        build.build()
    return native.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sr_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for must in ("sr_route", "sr_decode_attention", "sr_decode_workspace_bytes", "sr_status_string",
                 "sr_get_device_error"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in sinkrouter.h but not exported"
    assert set(native.EXPORTS) <= set(declared_functions())


def test_status_strings(lib):
    for s in range(5):
        assert lib.sr_status_string(s).decode().startswith("SR_")


def dims(B=1, Hq=32, Hkv=8, d=128, L=4096):
    return native.Dims(B, Hq, Hkv, d, L)


def test_workspace_bytes(lib):
    d = dims()
    auto = lib.sr_decode_workspace_bytes(ctypes.byref(d), 0)
    forced = lib.sr_decode_workspace_bytes(ctypes.byref(d), 64)
    assert auto > 0 and forced >= auto and auto % 256 == 0
    # 1024 + 8 slots * 4 heads * (128 + 2) fp32 + counters + header
    assert auto >= (1024 + 8) * 4 * 130 * 4
    assert lib.sr_decode_workspace_bytes(ctypes.byref(dims(d=64)), 0) == 0
    assert lib.sr_decode_workspace_bytes(ctypes.byref(dims(Hq=24, Hkv=8)), 0) == 0  # M=3
    assert lib.sr_decode_workspace_bytes(ctypes.byref(dims(Hq=30, Hkv=8)), 0) == 0  # Hq % Hkv
    assert lib.sr_decode_workspace_bytes(ctypes.byref(d), -1) == 0
    assert lib.sr_decode_workspace_bytes(None, 0) == 0


@pytest.mark.parametrize("bad,expect", [
    (dict(d=64), native.SR_ERR_UNSUPPORTED),
    (dict(Hq=128, Hkv=8), native.SR_ERR_UNSUPPORTED),  # M = 16
    (dict(Hq=24, Hkv=8), native.SR_ERR_UNSUPPORTED),  # M = 3
    (dict(B=4097, Hkv=8, Hq=32), native.SR_ERR_UNSUPPORTED),  # units > SR_MAX_UNITS
    (dict(B=0), native.SR_ERR_INVALID_ARG),
    (dict(Hq=30, Hkv=8), native.SR_ERR_INVALID_ARG),
    (dict(L=0), native.SR_ERR_INVALID_ARG),
])
def test_rejects_bad_dims(lib, bad, expect):
    d = dims(**bad)
    st = lib.sr_route(ctypes.byref(d), FAKE, FAKE, ctypes.c_float(0.6), FAKE, FAKE, None)
    assert st == expect
    st = lib.sr_decode_attention(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE,
                                 1 << 30, None)
    assert st == expect


def test_rejects_bad_pointers(lib):
    d = dims()
    assert lib.sr_route(ctypes.byref(d), None, FAKE, ctypes.c_float(0.6), FAKE, FAKE, None) == native.SR_ERR_INVALID_ARG
    assert lib.sr_route(ctypes.byref(d), FAKE + 2, FAKE, ctypes.c_float(0.6), FAKE, FAKE, None) == native.SR_ERR_INVALID_ARG
    assert lib.sr_route(ctypes.byref(d), FAKE, FAKE, ctypes.c_float(float("nan")), FAKE, FAKE, None) == native.SR_ERR_INVALID_ARG
    call = lambda **kw: lib.sr_decode_attention(  # noqa: E731
        ctypes.byref(d), kw.get("q", FAKE), FAKE, FAKE, None, FAKE, kw.get("seq", FAKE), FAKE, kw.get("ns", 0),
        kw.get("out", FAKE), kw.get("ws", FAKE), kw.get("wsb", 1 << 30), None)
    assert call(q=None) == native.SR_ERR_INVALID_ARG
    assert call(out=FAKE + 8) == native.SR_ERR_INVALID_ARG
    assert call(seq=FAKE + 2) == native.SR_ERR_INVALID_ARG
    assert call(ns=-1) == native.SR_ERR_INVALID_ARG
    assert call(ns=native.SR_MAX_SPLITS + 1) == native.SR_ERR_INVALID_ARG
    assert call(ws=None) == native.SR_ERR_WORKSPACE
    assert call(ws=FAKE + 128) == native.SR_ERR_WORKSPACE
    need = lib.sr_decode_workspace_bytes(ctypes.byref(d), 0)
    assert call(wsb=need - 1) == native.SR_ERR_WORKSPACE
    # forced splits need units * n_splits slots (here more than the automatic mode)
    need_forced = lib.sr_decode_workspace_bytes(ctypes.byref(d), 1024)
    assert need_forced > need
    assert call(ns=1024, wsb=need_forced - 1) == native.SR_ERR_WORKSPACE
    assert lib.sr_get_device_error(None, None, None) == native.SR_ERR_WORKSPACE
    assert lib.sr_workspace_init(FAKE + 4, 256, None) == native.SR_ERR_WORKSPACE


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(native, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        native.load(str(tmp_path / "nope.so"))


def test_fused_entry_validation(lib):
    d = dims()
    c = lambda **kw: lib.sr_route_decode_attention(  # noqa: E731
        ctypes.byref(d), FAKE, FAKE, FAKE, kw.get("k0", FAKE), FAKE, FAKE, ctypes.c_float(kw.get("tau", 0.6)),
        kw.get("ns", 0), None, kw.get("act", None), FAKE, kw.get("ws", FAKE), kw.get("wsb", 1 << 30), None)
    assert c(k0=None) == native.SR_ERR_INVALID_ARG  # the fused call routes, so k0 is required
    assert c(tau=float("nan")) == native.SR_ERR_INVALID_ARG
    assert c(act=FAKE + 2) == native.SR_ERR_INVALID_ARG
    assert c(ns=-3) == native.SR_ERR_INVALID_ARG
    assert c(ws=None) == native.SR_ERR_WORKSPACE
    assert c(wsb=16) == native.SR_ERR_WORKSPACE
    bad = dims(d=96)
    assert lib.sr_route_decode_attention(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.6),
                                         0, None, None, FAKE, FAKE, 1 << 30, None) == native.SR_ERR_UNSUPPORTED


def test_rope_append_route_validation(lib):
    """Host-side refusals of sr_rope_append_route: nothing is launched."""
    d = dims()

    def c(**kw):
        a = dict(q_in=FAKE, k_new=FAKE, v_new=FAKE, cos=FAKE, sin=FAKE, max_pos=64, seq=FAKE, kc=FAKE, vc=FAKE,
                 k0=FAKE, v0=FAKE, tau=0.6, q_out=FAKE, mask=FAKE, act=FAKE, err=None, dims=d)
        a.update(kw)
        return lib.sr_rope_append_route(ctypes.byref(a["dims"]), a["q_in"], a["k_new"], a["v_new"], a["cos"],
                                        a["sin"], a["max_pos"], a["seq"], a["kc"], a["vc"], a["k0"], a["v0"],
                                        ctypes.c_float(a["tau"]), a["q_out"], a["mask"], a["act"], a["err"], None)

    for name in ("q_in", "k_new", "v_new", "cos", "sin", "seq", "kc", "vc", "k0", "v0", "q_out", "mask", "act"):
        assert c(**{name: None}) == native.SR_ERR_INVALID_ARG, name
    for name in ("q_in", "k_new", "v_new", "cos", "sin", "kc", "vc", "k0", "v0", "q_out"):
        assert c(**{name: FAKE + 8}) == native.SR_ERR_INVALID_ARG, name  # 16-byte rows
    assert c(seq=FAKE + 2) == native.SR_ERR_INVALID_ARG
    assert c(err=FAKE + 2) == native.SR_ERR_INVALID_ARG
    assert c(max_pos=0) == native.SR_ERR_INVALID_ARG
    assert c(tau=float("nan")) == native.SR_ERR_INVALID_ARG
    assert c(dims=dims(d=64)) == native.SR_ERR_UNSUPPORTED


def test_bounded_wait_selftest_validation(lib):
    """Host-side refusals of sr_selftest_bounded_wait: nothing is launched."""
    c = lambda lim, st=FAKE, w=FAKE: lib.sr_selftest_bounded_wait(lim, st, w, None)  # noqa: E731
    assert c(0) == native.SR_ERR_INVALID_ARG
    assert c(2000001) == native.SR_ERR_INVALID_ARG
    assert c(1000, st=None) == native.SR_ERR_INVALID_ARG
    assert c(1000, st=FAKE + 2) == native.SR_ERR_INVALID_ARG
    assert c(1000, w=None) == native.SR_ERR_INVALID_ARG
    assert c(1000, w=FAKE + 4) == native.SR_ERR_INVALID_ARG
