"""GPU parity with a query offset (chunked prefill): the queries are the last
n_tokens of the q_offset + n_tokens keys ("Block-Filtered Long-Context
Attention", Section 3.6).  Every step through the C ABI is checked against the
oracle (global tiles), and the chunk's rows against the same rows of the whole
prefill run on the GPU."""
import numpy as np
import pytest
import torch

import oracle
import poem_synth
from _parity import (FWD_MAX_ABS, FWD_MEAN_ABS, compare_fwd, csr_rows, pooled_err_excess,
                     practical_lists_agree, score_err_excess, max_value_norm)

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


def _problem(x, q_offset, B):
    return oracle.Problem(q=poem_synth.bf16_bits(x["q"])[q_offset:], k=poem_synth.bf16_bits(x["k"]),
                          v=poem_synth.bf16_bits(x["v"]), block=B)


def _to_global(poem, arr_gpu, hq, Tq, t0, T):
    """Chunk layout (rows of the query tiles) -> the oracle's global lower-triangular layout."""
    out = np.zeros(hq * T * (T + 1) // 2)
    for h in range(hq):
        for i in range(Tq):
            a = poem.score_row_offset(Tq, t0, h, i)
            b = oracle.tri_offset(T, h, t0 + i)
            out[b:b + t0 + i + 1] = arr_gpu[a:a + t0 + i + 1]
    return out


def _global_csr(rp, ci, hq, Tq, t0):
    """Chunk CSR (rows h*Tq + i) -> CSR over all global tiles (history rows empty)."""
    T = Tq + t0
    counts = np.zeros(hq * T, dtype=np.int64)
    lists = {}
    for h in range(hq):
        for i in range(Tq):
            r = h * Tq + i
            lists[h * T + t0 + i] = ci[rp[r]:rp[r + 1]]
            counts[h * T + t0 + i] = rp[r + 1] - rp[r]
    grp = np.zeros(hq * T + 1, dtype=np.int32)
    grp[1:] = np.cumsum(counts)
    gci = np.concatenate([lists[r] for r in sorted(lists)]).astype(np.int32) if lists else np.zeros(0, np.int32)
    return grp, gci


CASES = [
    # (n_total, q_offset, Hq, Hkv, d, B, seed)
    (2048, 1024, 4, 1, 128, 128, 0),
    (1280, 896, 5, 1, 128, 128, 1),   # 7 history tiles, 3 query tiles, 5-way GQA
    (1024, 192, 2, 2, 64, 64, 2),     # 3 history tiles (odd), d = 64, B = 64
    (1024, 896, 4, 2, 128, 128, 3),   # a single query tile
]


@pytest.mark.parametrize("n,off,hq,hkv,d,B,seed", CASES)
def test_chunk_exact_path_matches_oracle(poem, n, off, hq, hkv, d, B, seed):
    tau = 0.05
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=seed)
    q = x["q"][off:].cuda()
    k, v = x["k"].cuda(), x["v"].cuda()
    T, t0 = n // B, off // B
    Tq = T - t0
    layer = poem.prefill_layer(q, k, v, tau, block=B)
    for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    assert layer.shape.q_offset == off
    prob = _problem(x, off, B)
    units = [(h, t0 + i) for h in range(hq) for i in range(Tq)]
    Ir, mr = prob.score_units(units)
    Ig = _to_global(poem, layer.I_hat.cpu().numpy(), hq, Tq, t0, T)
    mg = _to_global(poem, layer.m_hat.cpu().numpy(), hq, Tq, t0, T)
    idx = np.concatenate([np.arange(oracle.tri_offset(T, h, i), oracle.tri_offset(T, h, i) + i + 1) for h, i in units])
    assert score_err_excess(Ig[idx], Ir[idx], mg[idx], mr[idx], max_value_norm(x["v"])) <= 1.0
    # selection: bit-exact against the oracle's rule on the GPU's own scores
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
    rows = csr_rows(rp, ci)
    for h in range(hq):
        for i in range(Tq):
            o = oracle.tri_offset(T, h, t0 + i)
            ref, _ = oracle.select_row(t0 + i, Ig[o:o + t0 + i + 1], mg[o:o + t0 + i + 1], tau)
            assert rows[h * Tq + i] == ref.tolist(), (h, i)
    # attention: oracle masked attention over the GPU's lists
    grp, gci = _global_csr(rp, ci, hq, Tq, t0)
    O_ref, _ = prob.masked_units(units, grp, gci)
    og = torch.zeros(n, hq, d, dtype=torch.bfloat16)
    og[off:] = layer.o.cpu()
    mx, mean = compare_fwd(og, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS, (mx, mean)


def test_chunk_rows_equal_whole_prefill_rows(poem):
    """Scores and outputs of a chunk equal the corresponding rows of the whole
    prefill (same kernels, same per-row arithmetic)."""
    n, off, hq, hkv, d, B = 2048, 1024, 4, 1, 128, 128
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=4)
    T, t0 = n // B, off // B
    Tq = T - t0
    qf, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    full = poem.prefill_layer(qf, k, v, 0.05, block=B)
    chunk = poem.prefill_layer(qf[off:].contiguous(), k, v, 0.05, block=B)
    for ws in (full.ws_score, full.ws_select, full.ws_fwd, chunk.ws_score, chunk.ws_select, chunk.ws_fwd):
        poem.poem_check(ws)
    If = full.I_hat.cpu().numpy()
    Ic = chunk.I_hat.cpu().numpy()
    for h in range(hq):
        for i in range(Tq):
            a = poem.score_row_offset(Tq, t0, h, i)
            b = oracle.tri_offset(T, h, t0 + i)
            np.testing.assert_allclose(Ic[a:a + t0 + i + 1], If[b:b + t0 + i + 1], rtol=1e-6, atol=0)
    rpf = csr_rows(full.row_ptr.cpu().numpy(), full.col_idx[: int(full.row_ptr[-1])].cpu().numpy())
    rpc = csr_rows(chunk.row_ptr.cpu().numpy(), chunk.col_idx[: int(chunk.row_ptr[-1])].cpu().numpy())
    differ = sum(rpc[h * Tq + i] != rpf[h * T + t0 + i] for h in range(hq) for i in range(Tq))
    assert differ <= 1
    if differ == 0:
        np.testing.assert_array_equal(chunk.o.float().cpu().numpy(), full.o[off:].float().cpu().numpy())


@pytest.mark.parametrize("n,off,hq,hkv,d,B,seed", CASES[:3])
def test_chunk_practical_path_matches_oracle(poem, n, off, hq, hkv, d, B, seed):
    w, gamma, rho = 1.0, 0.9, 0.5
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=seed)
    q = x["q"][off:].cuda()
    k, v = x["k"].cuda(), x["v"].cuda()
    T, t0 = n // B, off // B
    Tq = T - t0
    layer = poem.prefill_layer_practical(q, k, v, w, gamma, rho, block=B)
    for ws in (layer.ws_pooled, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    prob = _problem(x, off, B)
    units = [(h, t0 + i) for h in range(hq) for i in range(Tq)]
    rm, rd = prob.pooled_units(units)
    mg = _to_global(poem, layer.m_pool.cpu().numpy(), hq, Tq, t0, T)
    dg = _to_global(poem, layer.d_pool.cpu().numpy(), hq, Tq, t0, T)
    idx = np.concatenate([np.arange(oracle.tri_offset(T, h, i), oracle.tri_offset(T, h, i) + i + 1) for h, i in units])
    vbar = float(x["v"].float().view(T, B, hkv, d).mean(1).norm(dim=-1).max())
    assert pooled_err_excess(mg[idx], rm[idx], dg[idx], rd[idx], vbar) <= 1.0
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
    rows = csr_rows(rp, ci)
    # lists on the GPU's own estimates against the oracle's practical rule (global rows)
    grows = [[] for _ in range(hq * T)]
    refrows = [[] for _ in range(hq * T)]
    for h in range(hq):
        for i in range(Tq):
            g = t0 + i
            o = oracle.tri_offset(T, h, g)
            grows[h * T + g] = rows[h * Tq + i]
            refrows[h * T + g] = oracle.select_practical_row(g, mg[o:o + g + 1], dg[o:o + g + 1], w, gamma,
                                                             rho)[0].tolist()
    for h in range(hq):
        for i in range(Tq):
            g, row = t0 + i, rows[h * Tq + i]
            assert row == sorted(set(row)) and all(0 <= b <= g for b in row)
            assert {0, g, g - 1} <= set(row)
    _, bad = practical_lists_agree(grows, refrows, mg, dg, hq, T, w, gamma, rho, band_m=0.0, band_key=1e-12,
                                   band_acc=1e-12, rows=[h * T + t0 + i for h in range(hq) for i in range(Tq)])
    assert not bad, bad
