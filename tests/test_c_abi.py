"""The C ABI from plain C: tests/c_abi/sr_abi_client.c is compiled with gcc
against include/sinkrouter.h and linked with libsinkrouter.so and the CUDA
runtime (for its own device buffers), with no Python in its path. On CPU it
checks status strings, workspace sizing and argument validation; on a GPU it
runs one routed decode step through sr_route + sr_decode_attention, and its
outputs are compared with the oracle."""
from __future__ import annotations

import os
import struct
import subprocess

import numpy as np
import pytest
import torch

from kv_cache_routing_sr_b200 import build, inputs
from tests import gpu_helpers as H

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def client(tmp_path_factory):
    if build.needs_build():
        build.build()
    out = str(tmp_path_factory.mktemp("c_abi") / "sr_abi_client")
    lib_dir = os.path.dirname(build.LIBRARY)
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Wextra", "-Werror", f"-I{build.INCLUDE}", f"-I{CUDA}/include",
           os.path.join(HERE, "c_abi", "sr_abi_client.c"), f"-L{lib_dir}", "-lsinkrouter", f"-L{CUDA}/lib64",
           "-lcudart", f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{CUDA}/lib64", "-o", out]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def test_c_client_host_checks(client):
    r = subprocess.run([client, "host"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "host checks ok" in r.stdout


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().tobytes()


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", [("tiny_4k", dict(max_ctx=1000)), ("llava7b_mha", dict(max_ctx=700, batch=2)),
                                     ("llama70b_ragged", dict(max_ctx=1500))])
def test_c_client_decode_step_matches_oracle(client, tmp_path, name, kw):
    x = inputs.make(name, seed=13, device="cpu", **kw)
    B, Hq, Hkv, L = x.batch, x.n_q_heads, x.n_kv_heads, x.max_seq_len
    tau_bits = struct.unpack("<i", struct.pack("<f", x.tau))[0]
    inp, outp = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        f.write(struct.pack("<5i", B, Hq, Hkv, L, tau_bits))
        for t in (x.q, x.k_cache, x.v_cache, x.k0, x.v0):
            f.write(_bits(t))
        f.write(x.seq_lens.to(torch.int32).numpy().tobytes())
    r = subprocess.run([client, "gpu", str(inp), str(outp)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    raw = open(outp, "rb").read()
    nq, U = B * Hq * 128 * 2, B * Hkv
    out = torch.from_numpy(np.frombuffer(raw[:nq], dtype=np.int16).copy()).view(torch.bfloat16).view(B, Hq, 128)
    mask = torch.from_numpy(np.frombuffer(raw[nq:nq + U], dtype=np.uint8).copy())
    act = torch.from_numpy(np.frombuffer(raw[nq + U:nq + U + 4 * (U + 1)], dtype=np.int32).copy())
    derr = struct.unpack("<i", raw[-4:])[0]
    assert derr == 0
    ref = H.oracle_full(x, x.tau)
    H.assert_route_equal(mask, act, ref.mask, ref.active_list)
    H.check_against_oracle(x, out, mask, what=f"C client {name}")
