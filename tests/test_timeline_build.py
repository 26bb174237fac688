"""The phase-timeline build (-DSR_TIMELINE) still compiles and exports its
readers, without a GPU: it is how the per-CTA phase timings of the decode and
routing kernels are taken, and nothing else exercises it on every change. The
default library must export none of them."""
import ctypes

import pytest

from kv_cache_routing_sr_b200 import build, native

READERS = ("sr_timeline_tl_decode", "sr_timeline_tl_decode_clear", "sr_timeline_tl_route",
           "sr_timeline_tl_route_clear", "sr_timeline_last_exit_addr", "sr_timeline_set_exit_ptr")


def have_nvcc():
    try:
        build.nvcc()
        return True
    except RuntimeError:
        return False


@pytest.mark.skipif(not have_nvcc(), reason="needs nvcc")
def test_timeline_build_compiles_and_exports_its_readers(tmp_path):
    out = build.build(output=str(tmp_path / "libsr_timeline.so"), defines=["SR_TIMELINE"])
    lib = ctypes.CDLL(out)
    for name in READERS:
        assert hasattr(lib, name), name
    # the instrumented build keeps the whole ABI
    for name in native.EXPORTS:
        assert hasattr(lib, name), name


def test_default_library_has_no_timeline():
    if build.needs_build():
        build.build()
    lib = ctypes.CDLL(build.LIBRARY)
    for name in READERS:
        assert not hasattr(lib, name), name
