"""GPU tests of the per-head threshold entry points (thresholds calibrated per head
group, as the pages describe) and of capturing a whole prefill layer in a CUDA
graph (the library neither allocates nor synchronises inside its calls)."""
import numpy as np
import pytest
import torch

import oracle
import poem_synth
from _parity import csr_rows, practical_lists_agree

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def poem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_poem_b200 import build

    build.build()
    oracle.build()
    import block_sparse_attention_poem_b200 as m

    return m


def _scores(poem, x, B):
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    layer = poem.alloc_layer(q, k, block=B, practical=True)
    poem.poem_score(q, k, v, layer.I_hat, layer.m_hat, layer.ws_score, shape=layer.shape)
    poem.poem_score_pooled(q, k, v, layer.m_pool, layer.d_pool, layer.ws_pooled, shape=layer.shape)
    poem.poem_check(layer.ws_score)
    poem.poem_check(layer.ws_pooled)
    return layer


def test_select_per_head_matches_oracle(poem):
    n, hq, hkv, d, B = 4096, 4, 1, 128, 128
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=12)
    layer = _scores(poem, x, B)
    taus = [0.02, 0.05, 0.1, 0.5]
    tau_dev = torch.tensor(taus, dtype=torch.float32, device="cuda")
    poem.poem_select_per_head(layer.shape, layer.I_hat, layer.m_hat, tau_dev, layer.row_ptr, layer.col_idx,
                              layer.ws_select, order=layer.order)
    poem.poem_check(layer.ws_select)
    rp = layer.row_ptr.cpu().numpy()
    rows = csr_rows(rp, layer.col_idx[: int(rp[-1])].cpu().numpy())
    Ig = layer.I_hat.cpu().numpy().astype(np.float64)
    mg = layer.m_hat.cpu().numpy().astype(np.float64)
    for h in range(hq):
        for i in range(T):
            o = oracle.tri_offset(T, h, i)
            ref, _ = oracle.select_row(i, Ig[o:o + i + 1], mg[o:o + i + 1], taus[h])
            assert rows[h * T + i] == ref.tolist(), (h, i)
    # a uniform array equals the scalar call
    tau_u = torch.full((hq,), 0.05, dtype=torch.float32, device="cuda")
    rp2, ci2 = torch.empty_like(layer.row_ptr), torch.empty_like(layer.col_idx)
    poem.poem_select_per_head(layer.shape, layer.I_hat, layer.m_hat, tau_u, rp2, ci2, layer.ws_select)
    poem.poem_select(layer.shape, layer.I_hat, layer.m_hat, 0.05, layer.row_ptr, layer.col_idx, layer.ws_select)
    poem.poem_check(layer.ws_select)
    assert torch.equal(rp2, layer.row_ptr) and torch.equal(ci2[: int(rp2[-1])], layer.col_idx[: int(rp2[-1])])


def test_select_per_head_bad_entry_keeps_rows_whole(poem):
    n, hq, hkv, d, B = 2048, 4, 1, 128, 128
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=13)
    layer = _scores(poem, x, B)
    tau_dev = torch.tensor([0.05, float("nan"), 0.1, -1.0], dtype=torch.float32, device="cuda")
    poem.poem_select_per_head(layer.shape, layer.I_hat, layer.m_hat, tau_dev, layer.row_ptr, layer.col_idx,
                              layer.ws_select)
    assert poem.poem_check_status(layer.ws_select) == 1  # POEM_ERR_INVALID_ARG
    assert poem.poem_check_status(layer.ws_select) == 0  # cleared
    rp = layer.row_ptr.cpu().numpy()
    rows = csr_rows(rp, layer.col_idx[: int(rp[-1])].cpu().numpy())
    for h in (1, 3):
        for i in range(T):
            assert rows[h * T + i] == list(range(i + 1))


def test_practical_per_head_matches_oracle(poem):
    n, hq, hkv, d, B = 4096, 4, 1, 128, 128
    T = n // B
    w, rho = 1.0, 0.5
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=14)
    layer = _scores(poem, x, B)
    gammas = [0.8, 0.9, 0.95, 0.99]
    g_dev = torch.tensor(gammas, dtype=torch.float32, device="cuda")
    poem.poem_select_practical_per_head(layer.shape, layer.m_pool, layer.d_pool, w, g_dev, rho, layer.row_ptr,
                                        layer.col_idx, layer.ws_select)
    poem.poem_check(layer.ws_select)
    rp = layer.row_ptr.cpu().numpy()
    rows = csr_rows(rp, layer.col_idx[: int(rp[-1])].cpu().numpy())
    mg = layer.m_pool.cpu().numpy().astype(np.float64)
    dg = layer.d_pool.cpu().numpy().astype(np.float64)
    for h in range(hq):
        # the gamma the kernel used is the float32 entry
        gh = float(np.float32(gammas[h]))
        ref = [[] for _ in range(hq * T)]
        for i in range(T):
            o = oracle.tri_offset(T, h, i)
            ref[h * T + i] = oracle.select_practical_row(i, mg[o:o + i + 1], dg[o:o + i + 1], w, gh, rho)[0].tolist()
        _, bad = practical_lists_agree(rows, ref, mg, dg, hq, T, w, gh, rho, band_m=0.0, band_key=1e-12,
                                       band_acc=1e-12, rows=[h * T + i for i in range(T)])
        assert not bad, (h, bad)


def test_prefill_layer_captured_in_a_cuda_graph(poem):
    """poem_score -> poem_select -> bsa_fwd captured once and replayed on new
    inputs written into the same buffers: identical to eager calls."""
    n, hq, hkv, d, B = 2048, 4, 1, 128, 128
    xa = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=15)
    xb = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=16)
    q, k, v = xa["q"].cuda(), xa["k"].cuda(), xa["v"].cuda()
    layer = poem.alloc_layer(q, k, block=B)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        poem.prefill_layer(q, k, v, 0.05, layer=layer, block=B)  # first calls (one-time setup) outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        poem.prefill_layer(q, k, v, 0.05, layer=layer, block=B)
    for x in (xb, xa):
        q.copy_(x["q"])
        k.copy_(x["k"])
        v.copy_(x["v"])
        g.replay()
        torch.cuda.synchronize()
        for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
            poem.poem_check(ws)
        o_graph = layer.o.clone()
        rp_graph = layer.row_ptr.clone()
        eager = poem.prefill_layer(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), 0.05, block=B)
        torch.cuda.synchronize()
        assert torch.equal(rp_graph, eager.row_ptr)
        assert torch.equal(o_graph, eager.o)
    del g
