"""GPU parity of the practical (pooled-estimate) selector: poem_score_pooled and
poem_select_practical through the C ABI against the fp64 oracle.

* Estimates: m~ and d~ for every (head, tile, visible block) against the oracle's
  pooled estimates on the same bf16 inputs (fp32 tolerance).
* Lists on identical estimates: the GPU's fp32 m~ / d~ fed to the oracle's
  selector; rows must match exactly except where a last-bit difference of the
  fp64 logarithms or of the fp64 summation order can decide (near-ties across
  the cut at 1e-12, accumulated mass within 1e-12 of gamma).
* End to end: GPU lists against the oracle's selection on the oracle's own
  estimates, with 1e-4 bands at the cut, and bsa_fwd on the GPU lists against
  oracle masked attention.  Sparse lists average few blocks, so outputs reach
  |o| ~ 3 here and the element bound adds bf16 output rounding (2^-8 |o|).
"""
import numpy as np
import pytest
import torch

import oracle
import poem_synth
from _parity import (FWD_MEAN_ABS, check_list_valid, compare_fwd_excess, csr_rows, pooled_err_excess,
                     practical_lists_agree, problem_from, to_dev)

pytestmark = pytest.mark.gpu

EXACT_BANDS = dict(band_m=0.0, band_key=1e-12, band_acc=1e-12)
E2E_BANDS = dict(band_m=1e-4, band_key=1e-4, band_acc=1e-4)

# (w, gamma, rho): plain I-estimate ranking, mass-only rerank, a heavier deviation
# weight, an unreachable threshold (whole shortlist) and a zero threshold.
PARAMS = [(1.0, 0.9, 0.5), (0.0, 0.95, 1.0), (2.0, 0.99, 0.25), (1.0, 1.5, 0.3), (1.0, 0.0, 1.0)]


@pytest.fixture(scope="module")
def poem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_poem_b200 import build

    build.build()
    oracle.build()
    import block_sparse_attention_poem_b200 as m

    return m


def _pooled(poem, x, B):
    q, k, v = to_dev(x)
    shape = poem.make_shape(q, k, block=B)
    T = q.shape[0] // B
    ne = poem.n_score_entries(q.shape[1], T)
    m_pool = torch.full((ne,), float("nan"), device="cuda")
    d_pool = torch.full((ne,), float("nan"), device="cuda")
    ws = poem.alloc_workspace(poem.poem_pooled_workspace_size(shape))
    poem.poem_score_pooled(q, k, v, m_pool, d_pool, ws, shape=shape)
    poem.poem_check(ws)
    return shape, m_pool, d_pool


def _select(poem, shape, m_pool, d_pool, w, gamma, rho, hq, T):
    _, sel_b, _ = poem.poem_workspace_size(shape)
    ws = poem.alloc_workspace(sel_b)
    rp = torch.empty(hq * T + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(max(m_pool.numel(), 4), dtype=torch.int32, device="cuda")
    order = torch.empty(hq * T, dtype=torch.int32, device="cuda")
    poem.poem_select_practical(shape, m_pool, d_pool, w, gamma, rho, rp, ci, ws, order=order)
    poem.poem_check(ws)
    rpn = rp.cpu().numpy()
    assert sorted(order.cpu().numpy().tolist()) == list(range(hq * T))
    return rpn, ci[: int(rpn[-1])].cpu().numpy(), rp, ci


def _vbar_norm(x, B):
    v = x["v"].float()
    n, hkv, d = v.shape
    return float(v.view(n // B, B, hkv, d).mean(1).norm(dim=-1).max())


LAYERS = [
    # (n_tokens, Hq, Hkv, d, block, seed)
    (2048, 4, 1, 128, 128, 0),
    (1280, 5, 1, 128, 128, 1),   # 5-way GQA, ragged tile count
    (1024, 2, 2, 64, 64, 2),
    (1024, 4, 2, 128, 64, 3),
    (1152, 2, 2, 64, 64, 7),     # 18 tiles: a partial group of 8 tiles per CTA
    (128, 4, 1, 128, 128, 8),    # a single tile
]


@pytest.mark.parametrize("n,hq,hkv,d,B,seed", LAYERS)
def test_pooled_estimates_match_oracle(poem, n, hq, hkv, d, B, seed):
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=seed)
    _, m_pool, d_pool = _pooled(poem, x, B)
    rm, rd = problem_from(x, B).pooled_all()
    assert np.isfinite(m_pool.cpu().numpy()).all() and np.isfinite(d_pool.cpu().numpy()).all()
    exc = pooled_err_excess(m_pool.cpu().numpy(), rm, d_pool.cpu().numpy(), rd, _vbar_norm(x, B))
    assert exc <= 1.0, exc


def test_pooled_masses_normalised(poem):
    """iid inputs, B = 64 rows averaged: the estimates stay finite and normalised:
    sum_b m~ = 1 per row and d~ >= 0."""
    x = poem_synth.iid_layer(2048, 4, 2, 128, seed=9)
    _, m_pool, d_pool = _pooled(poem, x, 64)
    m = m_pool.cpu().numpy().astype(np.float64)
    T = 2048 // 64
    for h in range(4):
        for i in range(T):
            off = oracle.tri_offset(T, h, i)
            assert abs(m[off:off + i + 1].sum() - 1.0) <= 1e-5
    assert (d_pool.cpu().numpy() >= 0).all()


@pytest.mark.parametrize("w,gamma,rho", PARAMS)
def test_practical_lists_on_identical_estimates(poem, w, gamma, rho):
    n, hq, hkv, d, B = 4096, 4, 1, 128, 128
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=4)
    T = n // B
    shape, m_pool, d_pool = _pooled(poem, x, B)
    rpn, cin, _, _ = _select(poem, shape, m_pool, d_pool, w, gamma, rho, hq, T)
    gpu_rows = csr_rows(rpn, cin)
    check_list_valid(gpu_rows, T)
    mg = m_pool.cpu().numpy().astype(np.float64)
    dg = d_pool.cpu().numpy().astype(np.float64)
    ref_rp, ref_ci, _ = oracle.select_practical_all(hq, T, mg, dg, w, gamma, rho)
    ref_rows = csr_rows(ref_rp, ref_ci)
    differ, bad = practical_lists_agree(gpu_rows, ref_rows, mg, dg, hq, T, w, gamma, rho, **EXACT_BANDS)
    assert not bad, bad
    assert differ <= max(1, hq * T // 100)


def test_practical_limits(poem):
    """gamma above any reachable mass keeps the whole shortlist; rho = 0 keeps the
    mandatory blocks only; rho = 1 with gamma > 1 keeps every visible block."""
    n, hq, hkv, d, B = 2048, 2, 1, 128, 128
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=5)
    shape, m_pool, d_pool = _pooled(poem, x, B)
    rpn, cin, _, _ = _select(poem, shape, m_pool, d_pool, 1.0, 2.0, 1.0, hq, T)
    assert csr_rows(rpn, cin) == [list(range(r % T + 1)) for r in range(hq * T)]
    rpn, cin, _, _ = _select(poem, shape, m_pool, d_pool, 1.0, 2.0, 0.0, hq, T)
    for r, row in enumerate(csr_rows(rpn, cin)):
        i = r % T
        assert row == sorted({0, i} | ({i - 1} if i >= 1 else set()))


def test_practical_rejects_bad_arguments(poem):
    n, hq, B = 512, 2, 128
    x = poem_synth.iid_layer(n, hq, 1, 128, seed=0)
    shape, m_pool, d_pool = _pooled(poem, x, B)
    T = n // B
    for w, gamma, rho in [(-1.0, 0.9, 0.5), (float("inf"), 0.9, 0.5), (1.0, float("nan"), 0.5), (1.0, 0.9, 1.5),
                          (1.0, 0.9, -0.1)]:
        with pytest.raises(poem.PoemError) as e:
            _select(poem, shape, m_pool, d_pool, w, gamma, rho, hq, T)
        assert e.value.status == 1


@pytest.mark.parametrize("n,hq,hkv,d,B,seed", LAYERS[:2])
def test_practical_end_to_end(poem, n, hq, hkv, d, B, seed):
    w, gamma, rho = 1.0, 0.9, 0.5
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=seed)
    T = n // B
    shape, m_pool, d_pool = _pooled(poem, x, B)
    rpn, cin, rp, ci = _select(poem, shape, m_pool, d_pool, w, gamma, rho, hq, T)
    gpu_rows = csr_rows(rpn, cin)
    prob = problem_from(x, B)
    rm, rd = prob.pooled_all()
    ref_rp, ref_ci, _ = oracle.select_practical_all(hq, T, rm, rd, w, gamma, rho)
    differ, bad = practical_lists_agree(gpu_rows, csr_rows(ref_rp, ref_ci), rm, rd, hq, T, w, gamma, rho,
                                        **E2E_BANDS)
    assert not bad, bad
    q, k, v = to_dev(x)
    o = torch.full_like(q, float("nan"))
    ws = poem.alloc_workspace(256)
    poem.bsa_fwd(q, k, v, rp, ci, o, ws, block=B)
    poem.poem_check(ws)
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, _ = prob.masked_units(units, rpn, cin)
    exc, mean = compare_fwd_excess(o, O_ref, units, B)
    assert exc <= 1.0 and mean <= FWD_MEAN_ABS, (exc, mean)


def test_prefill_layer_practical_128k_sampled(poem):
    """Llama-3.1-8B-shaped layer at 131072 tokens through prefill_layer_practical:
    estimates, lists and outputs checked on a deterministic sample of units."""
    n, hq, hkv, d, B = 131072, 32, 8, 128, 128
    w, gamma, rho = 1.0, 0.9, 0.5
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=500000.0, seed=0)
    q, k, v = to_dev(x)
    layer = poem.prefill_layer_practical(q, k, v, w, gamma, rho, block=B)
    for ws in (layer.ws_pooled, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    units = sorted({(0, 0), (0, 1), (0, 2), (hq - 1, T - 1), (hq // 2, T - 1), (1, T // 2), (7, 300), (20, 1000)})
    prob = problem_from(x, B)
    rm, rd = prob.pooled_units(units)
    mg = layer.m_pool.cpu().numpy()
    dg = layer.d_pool.cpu().numpy()
    idx = np.concatenate([np.arange(oracle.tri_offset(T, h, i), oracle.tri_offset(T, h, i) + i + 1)
                          for h, i in units])
    assert pooled_err_excess(mg[idx], rm[idx], dg[idx], rd[idx], _vbar_norm(x, B)) <= 1.0
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
    gpu_rows = csr_rows(rp, ci)
    check_list_valid(gpu_rows, T)
    ref_rows = {}
    for h, i in units:
        off = oracle.tri_offset(T, h, i)
        ref_rows[h * T + i] = oracle.select_practical_row(i, rm[off:off + i + 1], rd[off:off + i + 1], w, gamma,
                                                          rho)[0].tolist()
    rows = sorted(ref_rows)
    full_ref = [ref_rows.get(r, gpu_rows[r]) for r in range(hq * T)]
    _, bad = practical_lists_agree(gpu_rows, full_ref, rm, rd, hq, T, w, gamma, rho, rows=rows, **E2E_BANDS)
    assert not bad, bad
    O_ref, _ = prob.masked_units(units, rp, ci)
    exc, mean = compare_fwd_excess(layer.o, O_ref, units, B)
    assert exc <= 1.0 and mean <= FWD_MEAN_ABS, (exc, mean)


def test_ranked_budget_matches_oracle(poem):
    """poem_select_ranked_budget with score = exact I_hat at the practical lists'
    budgets: identical to the oracle's fixed-budget ranking on the same scores."""
    n, hq, hkv, d, B = 4096, 4, 1, 128, 128
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=6)
    shape, m_pool, d_pool = _pooled(poem, x, B)
    rpn, _, rp, _ = _select(poem, shape, m_pool, d_pool, 1.0, 0.9, 0.5, hq, T)
    q, k, v = to_dev(x)
    ne = poem.n_score_entries(hq, T)
    I_hat = torch.empty(ne, device="cuda")
    m_hat = torch.empty(ne, device="cuda")
    s_b, sel_b, _ = poem.poem_workspace_size(shape)
    ws_s = poem.alloc_workspace(s_b)
    poem.poem_score(q, k, v, I_hat, m_hat, ws_s, shape=shape)
    poem.poem_check(ws_s)
    ws = poem.alloc_workspace(sel_b)
    rp2 = torch.empty_like(rp)
    ci2 = torch.empty(ne, dtype=torch.int32, device="cuda")
    poem.poem_select_ranked_budget(shape, I_hat, rp, rp2, ci2, ws)
    poem.poem_check(ws)
    rows = csr_rows(rp2.cpu().numpy(), ci2[: int(rp2[-1])].cpu().numpy())
    Ig = I_hat.cpu().numpy().astype(np.float64)
    for h in range(hq):
        for i in range(T):
            r = h * T + i
            n_mand = 1 if i == 0 else (2 if i == 1 else 3)
            budget = int(rpn[r + 1] - rpn[r]) - n_mand
            off = oracle.tri_offset(T, h, i)
            assert rows[r] == oracle.select_mass_only_row(i, Ig[off:off + i + 1], budget).tolist(), (h, i)
