"""Host-side pieces of the bench on CPU: the ncu traffic figure is used only
while the decode kernel's source is the one it was captured on, and the
rotated input sets of the back-to-back protocol exceed L2 several times."""
import hashlib
import re
import types

import bench


def test_profiled_traffic_follows_the_committed_summary():
    text = open(bench.PROFILE_SUMMARY).read()
    want = float(re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M).group(1))
    recorded = re.search(r"^decode_source_sha256:\s*([0-9a-f]+)", text, re.M).group(1)
    current = hashlib.sha256(open(bench.DECODE_SOURCE, "rb").read()).hexdigest()
    got = bench.profiled_traffic()
    if current == recorded:
        assert got == want
    else:
        assert got is None


def test_profiled_traffic_is_dropped_for_another_source(tmp_path, monkeypatch):
    other = tmp_path / "sr_decode.cu"
    other.write_text("// a different kernel\n")
    monkeypatch.setattr(bench, "DECODE_SOURCE", str(other))
    assert bench.profiled_traffic() is None


def test_input_sets_exceed_l2_three_times():
    l2 = 126 << 20
    for numel in (1 << 20, 64 << 20, 512 << 20):  # bf16 elements of one cache
        x = types.SimpleNamespace(k_cache=types.SimpleNamespace(numel=lambda n=numel: n))
        n = bench.n_input_sets(x)
        per_set = numel * 2 * 2  # K and V, bf16
        assert n >= 3
        assert n * per_set > 3 * l2 or n == 32
