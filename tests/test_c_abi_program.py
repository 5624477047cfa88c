"""The C ABI from a plain C program (tests/c_abi_layer.c: CUDA runtime allocations and
a stream, no PyTorch): it builds against include/poem.h and libpoem.so on any host,
and on a GPU its outputs equal the Python binding's for the same layer."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import poem_synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    from block_sparse_attention_poem_b200 import build

    lib = build.build()
    exe = str(tmp_path / "c_abi_layer")
    cmd = [shutil.which("gcc") or "gcc", "-std=c11", "-O2", "-Wall", "-Werror",
           "-I" + os.path.join(ROOT, "include"), "-I" + os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c_abi_layer.c"), "-o", exe,
           "-L" + os.path.dirname(lib), "-lpoem", "-Wl,-rpath," + os.path.dirname(lib),
           "-L" + os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_program_builds_against_the_header_and_library(tmp_path):
    exe = _build(tmp_path)
    assert os.path.exists(exe)


@pytest.mark.gpu
def test_c_program_matches_the_python_binding(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_poem_b200 as poem

    exe = _build(tmp_path)
    n, hq, hkv, d, B, tau = 2048, 4, 2, 128, 128, 0.05
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=21)
    for name in ("q", "k", "v"):
        poem_synth.bf16_bits(x[name]).tofile(str(tmp_path / f"{name}.bin"))
    r = subprocess.run([exe, str(tmp_path), str(n), str(hq), str(hkv), str(d), str(B), str(tau)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    o_c = np.fromfile(str(tmp_path / "o.bin"), dtype=np.uint16).reshape(n, hq, d)
    rp_c = np.fromfile(str(tmp_path / "row_ptr.bin"), dtype=np.int32)
    ci_c = np.fromfile(str(tmp_path / "col_idx.bin"), dtype=np.int32)
    layer = poem.prefill_layer(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), tau, block=B)
    for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    rp = layer.row_ptr.cpu().numpy()
    assert np.array_equal(rp, rp_c)
    assert np.array_equal(layer.col_idx[: int(rp[-1])].cpu().numpy(), ci_c)
    assert np.array_equal(poem_synth.bf16_bits(layer.o.cpu()), o_c)
