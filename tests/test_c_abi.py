"""The C ABI from plain C (tests/c_abi/abi_decode.c): include/hq.h compiles as
C99, a C client links against libhq.so and the CUDA runtime alone, and on a
GPU its prefix install and decode step give bit-for-bit the output the
Python binding gives on the same inputs."""
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "abi_decode.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(out):
    from hybrid_precision_attention_b200 import build
    lib = build.build()
    cmd = ["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SRC, lib, "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + os.path.dirname(lib), "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def test_c_client_compiles_and_links(tmp_path):
    assert os.path.exists(_build(str(tmp_path / "abi_decode")))


@pytest.mark.gpu
def test_c_client_matches_the_python_binding(tmp_path):
    import torch
    from hybrid_precision_attention_b200 import hq
    exe = _build(str(tmp_path / "abi_decode"))
    dump = str(tmp_path / "dump.bin")
    r = subprocess.run([exe, dump], capture_output=True, text=True)
    assert r.returncode == 0, (r.stdout, r.stderr)
    B, Hq, Hkv, D, W, L, NQ = 1, 8, 2, 128, 16, 200, 64
    a = np.fromfile(dump, dtype=np.float16)
    sizes = [B * Hkv * L * D] * 2 + [B * Hq * NQ * D, B * Hq * D, B * Hkv * D, B * Hkv * D, B * Hq * D]
    parts = np.split(a, np.cumsum(sizes)[:-1])
    k, v = parts[0].reshape(B, Hkv, L, D), parts[1].reshape(B, Hkv, L, D)
    qt, q1 = parts[2].reshape(B, Hq, NQ, D), parts[3].reshape(B, Hq, D)
    k1, v1 = parts[4].reshape(B, Hkv, D), parts[5].reshape(B, Hkv, D)
    c_out = parts[6].reshape(B, Hq, D)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    cache = hq.HybridCache(B, Hq, Hkv, 256, W, 500)
    hq.hq_select_vlines(cache, dev(k), dev(qt))
    hq.hq_pack_merge(cache, dev(k), dev(v))
    scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    out = hq.hq_decode_attn(cache, dev(q1), dev(k1), dev(v1), sm_scale=scale)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), c_out.view(np.uint16))
