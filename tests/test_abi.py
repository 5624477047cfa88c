"""The C-ABI library loads and exports every entry point of include/poem.h, and
the host-side argument checks reject bad calls before any device work.  These
tests make no CUDA call and need no GPU."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "poem.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def poem():
    from block_sparse_attention_poem_b200 import build

    build.build()
    import block_sparse_attention_poem_b200 as m

    return m


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("poem_workspace_size", "poem_score", "poem_select", "poem_select_mass_only", "bsa_fwd",
              "poem_check", "poem_set_wait_limit_ns", "poem_status_string", "poem_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(poem):
    lib = ctypes.CDLL(poem.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) <= set(poem.EXPORTED)


def test_checks_build_exports_the_same_symbols(poem):
    """The debug build (bounds checks compiled in), when built, exports every entry point."""
    from block_sparse_attention_poem_b200 import build

    path = build.LIBS["checks"]
    if not os.path.exists(path):
        pytest.skip("libpoem_checks.so not built")
    lib = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_rejects_an_unknown_library_variant(tmp_path):
    import subprocess
    import sys

    env = dict(os.environ, POEM_LIBRARY_VARIANT="fast")
    r = subprocess.run([sys.executable, "-c", "import block_sparse_attention_poem_b200"], cwd=ROOT, env=env,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "POEM_LIBRARY_VARIANT" in r.stderr


def _shape(poem, **kw):
    base = dict(n_tokens=1024, n_q_heads=4, n_kv_heads=2, head_dim=128, block=128, n_sample=16, softmax_scale=0.0,
                q_offset=0, q_stride_tok=512, q_stride_head=128, kv_stride_tok=256, kv_stride_head=128,
                o_stride_tok=512, o_stride_head=128)
    base.update(kw)
    return poem.Shape(**base)


def _ws(poem, shape):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    st = poem._lib.poem_workspace_size(ctypes.byref(shape), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return st, a.value, b.value, c.value


def test_workspace_sizes(poem):
    st, s, sel, f = _ws(poem, _shape(poem))
    assert st == 0
    T, hq = 8, 4
    assert s >= 256 + hq * T * 16 * 128 * 4 + hq * T * 16 * 4
    assert sel >= 256 + hq * T * 4 + hq * T * (T + 1) // 2 * 4
    assert f >= 256


@pytest.mark.parametrize("kw,status", [
    (dict(n_tokens=1000), 1),            # N % block
    (dict(n_q_heads=3), 1),              # Hq % Hkv
    (dict(n_tokens=0), 1),
    (dict(head_dim=96), 2),
    (dict(block=32), 2),
    (dict(q_stride_tok=500), 1),         # not a multiple of 8 elements
    (dict(softmax_scale=float("nan")), 1),
    (dict(softmax_scale=-1.0), 1),
])
def test_shape_validation(poem, kw, status):
    st, *_ = _ws(poem, _shape(poem, **kw))
    assert st == status, poem.poem_status_string(st)


def test_null_and_misaligned_pointers_rejected(poem):
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    st = poem._lib.bsa_fwd(ctypes.byref(sh), None, ok, ok, ok, ok, None, ok, None, ok, 4096, None)
    assert st == 1
    st = poem._lib.bsa_fwd(ctypes.byref(sh), mis, ok, ok, ok, ok, None, ok, None, ok, 4096, None)
    assert st == 1
    st = poem._lib.poem_score(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, 16, None)
    assert st == 6  # workspace too small
    st = poem._lib.poem_score(ctypes.byref(_shape(poem, n_sample=8)), ok, ok, ok, ok, ok, ok, 1 << 30, None)
    assert st == 2
    assert "16-byte" in poem.poem_last_error() or "n_sample" in poem.poem_last_error()


def test_grouped_forward_validates_like_bsa_fwd(poem):
    """bsa_fwd_grouped shares bsa_fwd's host checks: null or misaligned pointers,
    a too-small workspace and unsupported shapes fail before any launch."""
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    f = poem._lib.bsa_fwd_grouped
    assert f(ctypes.byref(sh), None, ok, ok, ok, ok, ok, None, ok, 4096, None) == 1
    assert f(ctypes.byref(sh), ok, mis, ok, ok, ok, ok, None, ok, 4096, None) == 1
    assert f(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, ctypes.c_void_p((1 << 20) + 4), ok, 4096, None) == 1  # lse
    assert f(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, None, ok, 8, None) == 6
    assert f(ctypes.byref(_shape(poem, head_dim=96)), ok, ok, ok, ok, ok, ok, None, ok, 4096, None) == 2


@pytest.mark.parametrize("tau", [-0.1, float("nan"), float("inf")])
def test_select_rejects_bad_tau(poem, tau):
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    st = poem._lib.poem_select(ctypes.byref(sh), ok, ok, ctypes.c_float(tau), ok, ok, 100, None, ok, 1 << 30, None)
    assert st == 1


def test_select_rejects_small_workspace_and_negative_capacity(poem):
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    assert poem._lib.poem_select(ctypes.byref(sh), ok, ok, ctypes.c_float(0.05), ok, ok, 100, None, ok, 8, None) == 6
    assert poem._lib.poem_select(ctypes.byref(sh), ok, ok, ctypes.c_float(0.05), ok, ok, -1, None, ok, 1 << 30,
                                 None) == 1


def test_select_noalloc_host_refusals_set_the_message(poem):
    """poem_select_noalloc refuses bad arguments on the host, before resolving its
    scratch array, and leaves a message for every refusal."""
    f = poem._lib.poem_select_noalloc
    ok = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 4)
    poem._lib.poem_select(ctypes.byref(_shape(poem)), ok, ok, ctypes.c_float(-1.0), ok, ok, 100, None, ok, 1 << 30,
                          None)  # leaves an unrelated message behind
    cases = [
        (_shape(poem, n_tokens=1024 * 128, n_q_heads=32, n_kv_heads=8, q_stride_tok=4096, kv_stride_tok=1024),
         ok, 0.05, 100, 6, "static maximum"),
        (_shape(poem), ok, float("nan"), 100, 1, "poem_select_noalloc: tau"),
        (_shape(poem), ok, 0.05, -1, 1, "col_capacity"),
        (_shape(poem), mis, 0.05, 100, 1, "aligned"),
        (_shape(poem, head_dim=96), ok, 0.05, 100, 2, "head_dim"),
    ]
    for sh, ih, tau, cap, status, text in cases:
        poem._lib.poem_select(ctypes.byref(_shape(poem)), ok, ok, ctypes.c_float(-1.0), ok, ok, 100, None, ok,
                              1 << 30, None)
        assert f(ctypes.byref(sh), ih, ok, ctypes.c_float(tau), ok, ok, cap, None, None) == status
        assert text in poem.poem_last_error(), (text, poem.poem_last_error())


def test_status_strings(poem):
    for code, name in poem.STATUS.items():
        assert poem.poem_status_string(code) == name


def test_pooled_workspace_size(poem):
    sh = _shape(poem)
    a = ctypes.c_size_t()
    assert poem._lib.poem_pooled_workspace_size(ctypes.byref(sh), ctypes.byref(a)) == 0
    T, hq, hkv, d = 8, 4, 2, 128
    assert a.value >= 256 + (hq + 3 * hkv) * T * d * 4
    assert poem._lib.poem_pooled_workspace_size(ctypes.byref(_shape(poem, head_dim=96)), ctypes.byref(a)) == 2


def test_score_pooled_rejects_bad_pointers_and_workspace(poem):
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 4)
    assert poem._lib.poem_score_pooled(ctypes.byref(sh), ok, ok, ok, None, ok, ok, 1 << 30, None) == 1
    assert poem._lib.poem_score_pooled(ctypes.byref(sh), ok, mis, ok, ok, ok, ok, 1 << 30, None) == 1
    assert poem._lib.poem_score_pooled(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, 300, None) == 6


@pytest.mark.parametrize("w,gamma,rho", [(-1.0, 0.9, 0.5), (math.inf, 0.9, 0.5), (math.nan, 0.9, 0.5),
                                         (1.0, math.nan, 0.5), (1.0, 0.9, 1.01), (1.0, 0.9, -0.5),
                                         (1.0, 0.9, math.nan)])
def test_select_practical_rejects_bad_parameters(poem, w, gamma, rho):
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    st = poem._lib.poem_select_practical(ctypes.byref(sh), ok, ok, w, gamma, rho, ok, ok, 100, None, ok, 1 << 30,
                                         None)
    assert st == 1


def test_select_practical_rejects_null_deviation_and_small_workspace(poem):
    sh = _shape(poem)
    ok = ctypes.c_void_p(1 << 20)
    assert poem._lib.poem_select_practical(ctypes.byref(sh), ok, None, 1.0, 0.9, 0.5, ok, ok, 100, None, ok, 1 << 30,
                                           None) == 1
    assert poem._lib.poem_select_practical(ctypes.byref(sh), ok, ok, 1.0, 0.9, 0.5, ok, ok, 100, None, ok, 8,
                                           None) == 6


def test_query_offset_shape(poem):
    import torch

    q = torch.zeros(256, 2, 128, dtype=torch.bfloat16)
    k = torch.zeros(256 + 384, 1, 128, dtype=torch.bfloat16)
    sh = poem.make_shape(q, k, block=128)
    assert sh.q_offset == 384 and sh.n_tokens == 256
    st, s, sel, f = _ws(poem, sh)
    assert st == 0
    Tq, t0, hq = 2, 3, 2
    entries = hq * (Tq * t0 + Tq * (Tq + 1) // 2)
    assert entries == poem.n_score_entries(hq, Tq, t0) == 18  # per head: rows of 4 and 5 blocks
    assert sel >= 256 + hq * Tq * 4 + entries * 4
    assert poem.score_row_offset(Tq, t0, 1, 1) == 9 + 4
    for bad in (64, -128):  # not a multiple of block / negative
        st, *_ = _ws(poem, _shape(poem, q_offset=bad))
        assert st == 1
    with pytest.raises(ValueError):
        poem.make_shape(k, q)  # fewer keys than queries


def test_select_rejects_lists_beyond_int32_offsets(poem):
    # 128 heads x 8192 tiles: 128 * 8192 * 8193 / 2 > 2^31 - 1 entries
    sh = _shape(poem, n_tokens=8192 * 128, n_q_heads=128, n_kv_heads=8, q_stride_tok=128 * 128,
                o_stride_tok=128 * 128, kv_stride_tok=8 * 128)
    ok = ctypes.c_void_p(1 << 20)
    st = poem._lib.poem_select(ctypes.byref(sh), ok, ok, ctypes.c_float(0.05), ok, ok, 100, None, ok, 1 << 62, None)
    assert st == 2
    assert "int32" in poem.poem_last_error()


def test_binding_rejects_k_v_with_different_layouts(poem):
    import torch

    q = torch.zeros(256, 2, 128, dtype=torch.bfloat16)
    k = torch.zeros(256, 1, 128, dtype=torch.bfloat16)
    v = torch.zeros(256, 2, 160, dtype=torch.bfloat16)[:, :1, :128]  # same shape, other strides
    with pytest.raises(ValueError):
        poem._check_kv(k, v)
    poem._check_kv(k, k.clone())


def test_binding_checks_buffer_types_and_sizes(poem):
    import torch

    sh = _shape(poem)  # 4 q heads, 8 tiles: 32 rows, 144 entries
    rows, ne = poem._dims(sh)
    assert (rows, ne) == (32, 144)
    cpu_f = torch.zeros(ne, dtype=torch.float32)
    with pytest.raises(TypeError):  # not on a CUDA device
        poem._need(cpu_f, torch.float32, ne, "I_hat")
    with pytest.raises(TypeError):
        poem._need(torch.zeros(ne, dtype=torch.float64), torch.float32, ne, "I_hat")
    with pytest.raises(TypeError):
        poem._need(None, torch.int32, rows + 1, "row_ptr")
    poem._need(None, torch.int32, rows, "order", optional=True)


def test_binding_without_the_library_fails_at_import(tmp_path):
    """No fallback: a copy of the package without libpoem.so refuses to import."""
    import shutil
    import subprocess
    import sys

    src = os.path.join(ROOT, "block_sparse_attention_poem_b200")
    dst = tmp_path / "block_sparse_attention_poem_b200"
    dst.mkdir()
    for name in os.listdir(src):
        if name.endswith(".py"):
            shutil.copy(os.path.join(src, name), dst / name)
    r = subprocess.run([sys.executable, "-c", "import block_sparse_attention_poem_b200"], cwd=tmp_path,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)}, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "libpoem.so not built" in r.stderr
