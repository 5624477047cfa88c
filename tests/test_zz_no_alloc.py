"""poem_select_noalloc: block selection for callers that cannot allocate device
memory (a runtime that reserved all of HBM up front, or a plug-in that is only
handed pointers).  The entry point keeps its scratch in a fixed array inside the
library; this file checks, through the C ABI, that two calls in a row give the
same lists, row pointers and work order as poem_select with a caller-allocated
workspace, and that shapes beyond the fixed scratch are refused.

Kept in its own file, collected last, so that a failure here comes after every
other test has run."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def poem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_poem_b200 import build

    build.build()
    import block_sparse_attention_poem_b200 as m

    return m


def _shape(poem, hq, hkv, T, B=128, d=128):
    return poem.Shape(T * B, hq, hkv, d, B, 16, 0.0, 0, hq * d, d, hkv * d, d, hq * d, d)


def _scores(seed, hq, T):
    rng = np.random.default_rng(seed)
    ne = hq * T * (T + 1) // 2
    Ih = (rng.pareto(2.0, ne) * 1e-3).astype(np.float32)
    Ih[rng.random(ne) < 0.1] = np.float32(1e-3)  # ties
    mh = np.empty(ne, dtype=np.float32)
    off = 0
    for _ in range(hq):
        for i in range(T):
            w = rng.random(i + 1) ** 4
            mh[off:off + i + 1] = (w / w.sum()).astype(np.float32)
            off += i + 1
    return torch.from_numpy(Ih).cuda(), torch.from_numpy(mh).cuda()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_poem_select_on_two_calls(poem):
    hq, hkv, T = 4, 2, 64
    shape = _shape(poem, hq, hkv, T)
    rows = hq * T
    ne = hq * T * (T + 1) // 2
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed, tau in ((0, 0.02), (1, 0.1)):   # two calls in a row, different inputs
        Ih, mh = _scores(seed, hq, T)
        # the existing entry point, with a caller-allocated workspace
        rp_ref = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
        ci_ref = torch.full((ne,), -1, dtype=torch.int32, device="cuda")
        or_ref = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
        _, sel_b, _ = poem.poem_workspace_size(shape)
        ws = poem.alloc_workspace(sel_b)
        poem.poem_select(shape, Ih, mh, tau, rp_ref, ci_ref, ws, order=or_ref)
        poem.poem_check(ws)
        # the no-alloc entry point, called through the C ABI
        rp = torch.full((rows + 1,), -1, dtype=torch.int32, device="cuda")
        ci = torch.full((ne,), -1, dtype=torch.int32, device="cuda")
        order = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
        st = poem._lib.poem_select_noalloc(ctypes.byref(shape), _p(Ih), _p(mh), ctypes.c_float(tau), _p(rp), _p(ci),
                                           ci.numel(), _p(order), stream)
        assert st == 0, poem.poem_status_string(st)
        torch.cuda.synchronize()
        nnz = int(rp_ref[-1])
        assert torch.equal(rp, rp_ref)
        assert torch.equal(ci[:nnz], ci_ref[:nnz])
        assert torch.equal(order, or_ref)
        assert int(rp[-1]) <= ci.numel()


def test_noalloc_refuses_shapes_beyond_its_fixed_scratch(poem):
    shape = _shape(poem, 32, 8, 1024)   # needs ~67 MB of selection scratch
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    st = poem._lib.poem_select_noalloc(ctypes.byref(shape), _p(dummy), _p(dummy), ctypes.c_float(0.05), _p(dummy),
                                       _p(dummy), dummy.numel(), None, None)
    assert poem.STATUS[st] == "POEM_ERR_WORKSPACE"
    assert "static maximum" in poem.poem_last_error()


def test_noalloc_refusals_leave_a_message(poem):
    """Every refusal sets poem_last_error, so a caller never reads an earlier call's text."""
    shape = _shape(poem, 4, 2, 8)
    buf = torch.zeros(4096, dtype=torch.int32, device="cuda")
    f = torch.zeros(4096, dtype=torch.float32, device="cuda")
    poem._lib.poem_select_noalloc(ctypes.byref(_shape(poem, 32, 8, 1024)), _p(f), _p(f), ctypes.c_float(0.05),
                                  _p(buf), _p(buf), buf.numel(), None, None)
    assert "static maximum" in poem.poem_last_error()
    st = poem._lib.poem_select_noalloc(ctypes.byref(shape), _p(f), _p(f), ctypes.c_float(float("nan")), _p(buf),
                                       _p(buf), buf.numel(), None, None)
    assert poem.STATUS[st] == "POEM_ERR_INVALID_ARG"
    msg = poem.poem_last_error()
    assert msg and "tau" in msg
    st = poem._lib.poem_select_noalloc(ctypes.byref(shape), _p(f), _p(f), ctypes.c_float(0.05), _p(buf), _p(buf),
                                       -1, None, None)
    assert poem.STATUS[st] == "POEM_ERR_INVALID_ARG"
    assert "col_capacity" in poem.poem_last_error()
    st = poem._lib.poem_select_noalloc(ctypes.byref(shape), None, _p(f), ctypes.c_float(0.05), _p(buf), _p(buf),
                                       buf.numel(), None, None)
    assert poem.STATUS[st] == "POEM_ERR_INVALID_ARG"
    assert "aligned" in poem.poem_last_error()
