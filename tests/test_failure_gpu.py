"""Failure detection on the GPU without a fault: every device wait in the library
is bounded.  With the limit set to zero the waits run out, the kernels record
POEM_ERR_TIMEOUT in the workspace error word, drain their in-flight copies and
MMAs, release tensor memory and return; poem_check reports the status and the
context stays usable (the next call with the normal limit is correct)."""
import pytest
import torch

import oracle
import poem_synth
from _parity import FWD_MAX_ABS, FWD_MEAN_ABS, compare_fwd, problem_from

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


@pytest.fixture(scope="module")
def poem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_poem_b200 import build

    build.build()
    oracle.build()
    import block_sparse_attention_poem_b200 as m

    yield m
    m.poem_set_wait_limit_ns(DEFAULT_LIMIT_NS)


def test_expired_waits_report_timeout_and_context_recovers(poem):
    n, hq, hkv, d, B = 2048, 4, 1, 128, 128
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=5)
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    rp, ci = poem_synth.random_block_lists(hq, T, 0.5, seed=5)
    rpd, cid = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
    layer = poem.alloc_layer(q, k, block=B)
    o = torch.empty_like(q)
    try:
        poem.poem_set_wait_limit_ns(0)
        poem.bsa_fwd(q, k, v, rpd, cid, o, layer.ws_fwd, shape=layer.shape)
        assert poem.STATUS[poem.poem_check_status(layer.ws_fwd)] == "POEM_ERR_TIMEOUT"
        poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
        assert poem.STATUS[poem.poem_check_status(layer.ws_score)] == "POEM_ERR_TIMEOUT"
    finally:
        poem.poem_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    # the error words were cleared by poem_check; the same calls now succeed
    torch.cuda.synchronize()
    poem.bsa_fwd(q, k, v, rpd, cid, o, layer.ws_fwd, shape=layer.shape)
    assert poem.poem_check_status(layer.ws_fwd) == 0
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, _ = problem_from(x, B).masked_units(units, rp, ci)
    mx, mean = compare_fwd(o, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS
    poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
    assert poem.poem_check_status(layer.ws_score) == 0
    assert torch.isfinite(layer.I_hat).all()


def test_grouped_expired_waits_report_timeout_and_context_recovers(poem):
    """The same for bsa_fwd_grouped (one CTA per SM, two heads over a shared K/V ring)."""
    n, hq, hkv, d, B = 2048, 8, 2, 128, 128
    T = n // B
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=6)
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    rp, ci = poem_synth.random_block_lists(hq, T, 0.5, seed=6)
    rpd, cid = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
    ws = poem.alloc_workspace(256)
    o = torch.empty_like(q)
    try:
        poem.poem_set_wait_limit_ns(0)
        poem.bsa_fwd_grouped(q, k, v, rpd, cid, o, ws, block=B)
        assert poem.STATUS[poem.poem_check_status(ws)] == "POEM_ERR_TIMEOUT"
    finally:
        poem.poem_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    torch.cuda.synchronize()
    poem.bsa_fwd_grouped(q, k, v, rpd, cid, o, ws, block=B)
    assert poem.poem_check_status(ws) == 0
    o_ref = torch.empty_like(q)
    poem.bsa_fwd(q, k, v, rpd, cid, o_ref, ws, block=B)
    assert poem.poem_check_status(ws) == 0
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
