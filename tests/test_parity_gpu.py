"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Sizes span several tiles and the ragged/degenerate cases;
the full-size sampled checks live in test_parity_fullsize_gpu.py."""
import numpy as np
import pytest
import torch

import oracle
import poem_synth
from _parity import (FWD_MAX_ABS, FWD_MEAN_ABS, compare_fwd, csr_rows, lists_agree_at_cut, max_value_norm,
                     problem_from, score_err_excess, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def poem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_poem_b200 import build

    build.build()
    import block_sparse_attention_poem_b200 as m

    return m


@pytest.fixture(scope="module", autouse=True)
def _oracle_built():
    oracle.build()


def _run_fwd(poem, x, row_ptr, col_idx, block, order=None, with_lse=True):
    q, k, v = to_dev(x)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((q.shape[1], q.shape[0]), float("nan"), device="cuda") if with_lse else None
    ws = poem.alloc_workspace(256)
    rp = torch.from_numpy(np.ascontiguousarray(row_ptr, dtype=np.int32)).cuda()
    ci = torch.from_numpy(np.ascontiguousarray(col_idx, dtype=np.int32)).cuda()
    if ci.numel() == 0:
        ci = torch.zeros(4, dtype=torch.int32, device="cuda")
    od = None if order is None else torch.from_numpy(np.ascontiguousarray(order, dtype=np.int32)).cuda()
    poem.bsa_fwd(q, k, v, rp, ci, o, ws, lse=lse, order=od, block=block)
    status = poem.poem_check_status(ws)
    return o, lse, status


# ---------------------------------------------------------------------------
# bsa_fwd on identical (oracle-made) lists
# ---------------------------------------------------------------------------

FWD_CASES = [
    # (n_tokens, Hq, Hkv, d, block, density, seed)
    (1024, 4, 2, 128, 128, 0.4, 0),
    (2048, 4, 1, 128, 128, 0.25, 1),
    (1024, 1, 1, 64, 64, 0.5, 2),
    (1024, 2, 1, 128, 64, 0.3, 3),
    (768, 2, 2, 64, 128, 0.6, 4),
    (640, 5, 1, 128, 128, 1.0, 5),   # dense lists, 5-way GQA
]


@pytest.mark.parametrize("n,hq,hkv,d,B,dens,seed", FWD_CASES)
def test_bsa_fwd_matches_oracle(poem, n, hq, hkv, d, B, dens, seed):
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=seed)
    T = n // B
    rp, ci = poem_synth.random_block_lists(hq, T, dens, seed=seed)
    o, lse, status = _run_fwd(poem, x, rp, ci, B)
    assert status == 0, poem.poem_status_string(status)
    prob = problem_from(x, B)
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, lse_ref = prob.masked_units(units, rp, ci)
    mx, mean = compare_fwd(o, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS, (mx, mean)
    lg = lse.cpu().numpy()
    for u, (h, i) in enumerate(units):
        np.testing.assert_allclose(lg[h, i * B:(i + 1) * B], lse_ref[u], atol=2e-3, rtol=0)


def test_bsa_fwd_all_blocks_equals_dense(poem):
    n, hq, hkv, d, B = 1024, 2, 1, 128, 128
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=7)
    T = n // B
    rp, ci = poem_synth.random_block_lists(hq, T, 1.0, seed=7)
    o, _, status = _run_fwd(poem, x, rp, ci, B)
    assert status == 0
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, _ = problem_from(x, B).dense_units(units)
    mx, mean = compare_fwd(o, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("T", [1, 2, 3])
def test_bsa_fwd_few_tiles(poem, T):
    B = 128
    x = poem_synth.iid_layer(T * B, 2, 1, 128, seed=10 + T)
    rp, ci = poem_synth.random_block_lists(2, T, 0.5, seed=T)
    o, _, status = _run_fwd(poem, x, rp, ci, B)
    assert status == 0
    units = [(h, i) for h in range(2) for i in range(T)]
    O_ref, _ = problem_from(x, B).masked_units(units, rp, ci)
    mx, mean = compare_fwd(o, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS


def test_bsa_fwd_empty_and_diagonal_only_rows(poem):
    n, hq, B = 512, 2, 128
    T = n // B
    x = poem_synth.iid_layer(n, hq, 1, 128, seed=21)
    rows = []
    for h in range(hq):
        for i in range(T):
            if h == 0 and i == 2:
                rows.append([])          # empty row: output 0, lse -inf
            elif h == 1:
                rows.append([i])         # diagonal block only
            else:
                rows.append(list(range(i + 1)))
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.array([b for r in rows for b in r], dtype=np.int32)
    o, lse, status = _run_fwd(poem, x, rp, ci, B)
    assert status == 0
    og = o.float().cpu().numpy()
    assert np.all(og[2 * B:3 * B, 0, :] == 0.0)
    assert np.all(np.isneginf(lse.cpu().numpy()[0, 2 * B:3 * B]))
    units = [(h, i) for h in range(hq) for i in range(T) if not (h == 0 and i == 2)]
    O_ref, _ = problem_from(x, B).masked_units(units, rp, ci)
    mx, mean = compare_fwd(o, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS


def test_bsa_fwd_explicit_order_gives_same_result(poem):
    n, hq, B = 1024, 4, 128
    T = n // B
    x = poem_synth.iid_layer(n, hq, 2, 128, seed=31)
    rp, ci = poem_synth.random_block_lists(hq, T, 0.5, seed=31)
    o1, _, s1 = _run_fwd(poem, x, rp, ci, B)
    order = np.random.default_rng(0).permutation(hq * T).astype(np.int32)
    o2, _, s2 = _run_fwd(poem, x, rp, ci, B, order=order)
    assert s1 == 0 and s2 == 0
    assert torch.equal(o1, o2)


def test_bsa_fwd_rejects_out_of_range_block(poem):
    n, hq, B = 512, 1, 128
    x = poem_synth.iid_layer(n, hq, 1, 128, seed=41)
    rows = [[0], [0, 1], [0, 3, 2], [0, 3]]   # row 2 lists block 3 > tile 2
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.array([b for r in rows for b in r], dtype=np.int32)
    o, _, status = _run_fwd(poem, x, rp, ci, B)
    assert poem.STATUS[status] == "POEM_ERR_BAD_LIST"
    # the valid entries of every row are still computed
    fixed = [[0], [0, 1], [0, 2], [0, 3]]
    rp2 = np.concatenate([[0], np.cumsum([len(r) for r in fixed])]).astype(np.int32)
    ci2 = np.array([b for r in fixed for b in r], dtype=np.int32)
    O_ref, _ = problem_from(x, B).masked_units([(0, i) for i in range(4)], rp2, ci2)
    mx, mean = compare_fwd(o, O_ref, [(0, i) for i in range(4)], B)
    assert mx <= FWD_MAX_ABS


# ---------------------------------------------------------------------------
# poem_select on identical (oracle-produced, fp32-rounded) scores: bit-exact
# ---------------------------------------------------------------------------

def _gpu_select(poem, shape, Ih32, mh32, tau, n_rows, mass_only_ref=None, want_order=True):
    Ih = torch.from_numpy(Ih32).cuda()
    mh = torch.from_numpy(mh32).cuda()
    rp = torch.empty(n_rows + 1, dtype=torch.int32, device="cuda")
    ci = torch.full((Ih32.size,), -1, dtype=torch.int32, device="cuda")
    order = torch.full((n_rows,), -1, dtype=torch.int32, device="cuda") if want_order else None
    _, sel_b, _ = poem.poem_workspace_size(shape)
    ws = poem.alloc_workspace(sel_b)
    if mass_only_ref is None:
        poem.poem_select(shape, Ih, mh, tau, rp, ci, ws, order=order)
    else:
        ref = torch.from_numpy(np.ascontiguousarray(mass_only_ref, dtype=np.int32)).cuda()
        poem.poem_select_mass_only(shape, mh, ref, rp, ci, ws, order=order)
    status = poem.poem_check_status(ws)
    return rp.cpu().numpy(), ci.cpu().numpy(), (order.cpu().numpy() if want_order else None), status


def _fake_shape(poem, hq, hkv, T, B=128):
    n = T * B
    return poem.Shape(n, hq, hkv, 128, B, 16, 0.0, 0, hq * 128, 128, hkv * 128, 128, hq * 128, 128)


@pytest.mark.parametrize("T,hq,hkv,seed", [(16, 4, 1, 0), (300, 2, 1, 1), (1024, 1, 1, 2), (3, 2, 2, 3)])
def test_select_bit_exact_on_identical_scores(poem, T, hq, hkv, seed):
    rng = np.random.default_rng(seed)
    ne = hq * T * (T + 1) // 2
    # heavy-tailed scores with exact ties
    Ih = (rng.pareto(2.0, ne) * 1e-3).astype(np.float32)
    Ih[rng.random(ne) < 0.1] = np.float32(1e-3)
    Ih[rng.random(ne) < 0.05] = 0.0
    mh = np.zeros(ne, dtype=np.float32)
    for h in range(hq):
        for i in range(T):
            off = oracle.tri_offset(T, h, i)
            w = rng.random(i + 1) ** 4
            mh[off:off + i + 1] = (w / w.sum() * 1.3).astype(np.float32)
    shape = _fake_shape(poem, hq, hkv, T)
    prev_rows = None
    for tau in (0.0, 0.002, 0.02, 0.1, 1e6):  # 1e6: only the mandatory blocks survive
        rp, ci, order, status = _gpu_select(poem, shape, Ih, mh, tau, hq * T)
        assert status == 0
        # nested supports: a larger tau keeps a subset of every row (the cut is monotone in tau)
        rows = csr_rows(rp, ci[:rp[-1]])
        if prev_rows is not None:
            assert all(set(a) <= set(b) for a, b in zip(rows, prev_rows))
        prev_rows = rows
        rp_ref, ci_ref, _ = oracle.select_all(hq, T, Ih.astype(np.float64), mh.astype(np.float64), tau)
        assert np.array_equal(rp, rp_ref)
        assert np.array_equal(ci[:rp[-1]], ci_ref)
        # work order: a permutation, grouped by KV head, longest first, ties by row id
        G = hq // hkv
        lens = np.diff(rp)
        for g in range(hkv):
            seg = order[g * G * T:(g + 1) * G * T]
            assert sorted(seg.tolist()) == list(range(g * G * T, (g + 1) * G * T))
            key = [(-lens[r], r) for r in seg]
            assert key == sorted(key)


def _tau_cutting_between(I, m, i, a, b):
    """A float32 tau whose stopping rule keeps candidate a and drops b (b right after
    a in the (I desc, id asc) order) in row i, or None when no such tau exists."""
    cand = sorted(range(1, max(i - 1, 1)), key=lambda c: (-I[c], c))
    if a not in cand or b not in cand or cand.index(b) != cand.index(a) + 1:
        return None
    k = cand.index(a) + 1  # kept candidates: through a

    def thr(kk):  # smallest tau that lets the suffix after kk be dropped
        D = cand[kk:]
        sI, sm = float(sum(I[c] for c in D)), float(sum(m[c] for c in D))
        return sI / (1.0 - sm) if sm < 1.0 else np.inf

    lo, hi = thr(k), thr(k - 1)
    if not (np.isfinite(hi) and lo < hi):
        return None
    tau = float(np.float32(0.5 * (lo + hi)))
    keep, _ = oracle.select_row(i, I[:i + 1], m[:i + 1], tau)
    return tau if (a in keep.tolist() and b not in keep.tolist()) else None


def test_ties_forced_by_duplicated_blocks(poem):
    """Key blocks with identical K and V give bit-identical scores through the whole
    score pass; with tau chosen so that a row's cut falls between the two copies, the
    selector keeps the smaller id and drops the larger (the "Block ordering" tie-break)."""
    n, hq, hkv, d, B = 2048, 2, 1, 128, 128
    T = n // B
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=31)
    pairs = [(2, 10), (3, 5), (7, 9)]
    for a, b in pairs:
        x["k"][b * B:(b + 1) * B] = x["k"][a * B:(a + 1) * B]
        x["v"][b * B:(b + 1) * B] = x["v"][a * B:(a + 1) * B]
    q, k, v = to_dev(x)
    layer = poem.prefill_layer(q, k, v, 0.05, block=B)
    for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    Ig = layer.I_hat.cpu().numpy()
    mg = layer.m_hat.cpu().numpy()
    shape = _fake_shape(poem, hq, hkv, T)
    decisive = 0
    for h in range(hq):
        for i in range(T):
            off = oracle.tri_offset(T, h, i)
            I = Ig[off:off + i + 1].astype(np.float64)
            m = mg[off:off + i + 1].astype(np.float64)
            for a, b in pairs:
                if b >= i - 1:  # b must be a candidate (not mandatory) of tile i
                    continue
                assert Ig[off + a] == Ig[off + b] and mg[off + a] == mg[off + b], (h, i, a, b)
                tau = _tau_cutting_between(I, m, i, a, b)
                if tau is None:
                    continue
                rp, ci, _, st = _gpu_select(poem, shape, Ig, mg, tau, hq * T, want_order=False)
                assert st == 0
                row = csr_rows(rp, ci[:rp[-1]])[h * T + i]
                assert a in row and b not in row, (h, i, a, b, tau)
                decisive += 1
    assert decisive > 0


def test_select_mass_only_matches_oracle(poem):
    T, hq = 64, 2
    rng = np.random.default_rng(5)
    ne = hq * T * (T + 1) // 2
    Ih = rng.random(ne).astype(np.float32)
    mh = (rng.random(ne) ** 3 / 8).astype(np.float32)
    shape = _fake_shape(poem, hq, 1, T)
    rp, ci, _, st = _gpu_select(poem, shape, Ih, mh, 0.05, hq * T)
    assert st == 0
    rpm, cim, _, st = _gpu_select(poem, shape, Ih, mh, 0.05, hq * T, mass_only_ref=rp)
    assert st == 0
    assert np.array_equal(rpm, rp)  # same budget per row
    rows = csr_rows(rpm, cim)
    for h in range(hq):
        for i in range(T):
            off = oracle.tri_offset(T, h, i)
            k = max(0, len(rows[h * T + i]) - min(3, i + 1))
            ref = oracle.select_mass_only_row(i, mh[off:off + i + 1].astype(np.float64), k)
            assert rows[h * T + i] == ref.tolist()


def test_select_capacity_exceeded_reports(poem):
    T, hq = 32, 1
    ne = T * (T + 1) // 2
    Ih = np.ones(ne, dtype=np.float32)
    mh = np.full(ne, 0.01, dtype=np.float32)
    shape = _fake_shape(poem, hq, 1, T)
    Ihd, mhd = torch.from_numpy(Ih).cuda(), torch.from_numpy(mh).cuda()
    rp = torch.empty(T + 1, dtype=torch.int32, device="cuda")
    ci = torch.full((40,), -7, dtype=torch.int32, device="cuda")
    _, sel_b, _ = poem.poem_workspace_size(shape)
    ws = poem.alloc_workspace(sel_b)
    poem.poem_select(shape, Ihd, mhd, 0.0, rp, ci, ws)
    assert poem.STATUS[poem.poem_check_status(ws)] == "POEM_ERR_CAPACITY"
    assert int(rp[-1]) == ne  # tau = 0 keeps everything
    assert torch.all(ci[:40] >= 0)  # the prefix that fits was written


# ---------------------------------------------------------------------------
# poem_score against the oracle
# ---------------------------------------------------------------------------

SCORE_CASES = [
    # (n_tokens, Hq, Hkv, d, block, rope_base, seed)
    (2048, 4, 1, 128, 128, 500000.0, 0),
    (1280, 5, 1, 128, 128, 1000000.0, 1),   # 5-way GQA: packed groups straddle tiles
    (1024, 8, 2, 128, 128, 500000.0, 2),
    (1024, 2, 1, 64, 64, 10000.0, 3),
    # more than 32 tiles: the CTAs beyond tile 32 take both passes' fp16 P V contraction
    (6400, 5, 1, 128, 128, 1000000.0, 4),
    (4096, 2, 1, 64, 64, 10000.0, 5),
    # 8-way GQA: a CTA holds one tile of 8 heads, so tile 0's CTA sweeps a single block
    # (the second softmax warpgroup of each pass gets none) and the sweep lengths take
    # both parities
    (1536, 16, 2, 128, 128, 500000.0, 6),
]


def _gpu_score(poem, x, B):
    q, k, v = to_dev(x)
    shape = poem.make_shape(q, k, block=B)
    T = q.shape[0] // B
    ne = poem.n_score_entries(q.shape[1], T)
    Ih = torch.full((ne,), float("nan"), device="cuda")
    mh = torch.full((ne,), float("nan"), device="cuda")
    s_b, _, _ = poem.poem_workspace_size(shape)
    ws = poem.alloc_workspace(s_b)
    poem.poem_score(q, k, v, Ih, mh, ws, shape=shape)
    status = poem.poem_check_status(ws)
    return Ih.cpu().numpy(), mh.cpu().numpy(), status


@pytest.mark.parametrize("n,hq,hkv,d,B,base,seed", SCORE_CASES)
def test_score_matches_oracle(poem, n, hq, hkv, d, B, base, seed):
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, rope_base=base, seed=seed)
    Ig, mg, status = _gpu_score(poem, x, B)
    assert status == 0
    T = n // B
    Ir, mr = problem_from(x, B).score_all()
    assert np.all(np.isfinite(Ig)) and np.all(np.isfinite(mg))
    assert score_err_excess(Ig, Ir, mg, mr, max_value_norm(x["v"])) <= 1.0


def test_score_single_head_fp32_recipe(poem):
    """Single-head N = 1024, d = 64, B = 64 recipe (K scaled for logit std 2),
    fed to both sides as the same bf16-rounded values."""
    x = poem_synth.single_head(1024, 64, seed=0)
    xb = {k: t.to(torch.bfloat16) for k, t in x.items()}
    Ig, mg, status = _gpu_score(poem, xb, 64)
    assert status == 0
    Ir, mr = problem_from(xb, 64).score_all()
    assert score_err_excess(Ig, Ir, mg, mr, max_value_norm(xb["v"])) <= 1.0


def test_score_shift_invariance(poem):
    """Adding one vector to every value leaves I_hat unchanged (reading note,
    Section 4.1 shift check); m_hat does not depend on V at all."""
    x = poem_synth.heavy_block_layer(1024, 4, 1, 128, block=128, seed=9)
    c = torch.randn(128, generator=torch.Generator().manual_seed(1)) * 3
    xs = dict(x)
    # shift in fp32 then round; compare against the oracle on the shifted values
    xs["v"] = (x["v"].float() + c).to(torch.bfloat16)
    I0, m0, _ = _gpu_score(poem, x, 128)
    I1, m1, _ = _gpu_score(poem, xs, 128)
    Ir1, mr1 = problem_from(xs, 128).score_all()
    assert score_err_excess(I1, Ir1, m1, mr1, max_value_norm(xs["v"])) <= 1.0
    assert np.array_equal(m0, m1)


def test_score_values_beyond_fp16_range_take_the_bf16_contraction(poem):
    """Both score passes run the P V contraction of CTAs whose tiles are all >= 32 with
    one fp16 P on an fp16 copy of V.  A finite |v| above the fp16 maximum (65504) sets the range
    flag in the score workspace (byte 8) and every CTA takes the bf16 hi/lo
    contraction; both give oracle scores (64 tiles: CTAs on both sides of tile 32)."""
    x = poem_synth.heavy_block_layer(8192, 4, 1, 128, block=128, seed=21)
    for scale, flag in ((1.0, 0), (2.0 ** -8, 0), (2.0 ** 16, 1)):
        xs = dict(x)
        xs["v"] = (x["v"].float() * scale).to(torch.bfloat16)  # a power of two: exact in bf16
        q, k, v = to_dev(xs)
        shape = poem.make_shape(q, k, block=128)
        ne = poem.n_score_entries(4, 64)
        Ih = torch.full((ne,), float("nan"), device="cuda")
        mh = torch.full((ne,), float("nan"), device="cuda")
        s_b, _, _ = poem.poem_workspace_size(shape)
        ws = poem.alloc_workspace(s_b)
        poem.poem_score(q, k, v, Ih, mh, ws, shape=shape)
        assert poem.poem_check_status(ws) == 0
        assert int(ws[8:12].view(torch.int32).item()) == flag, scale
        Ir, mr = problem_from(xs, 128).score_all()
        assert score_err_excess(Ih.cpu().numpy(), Ir, mh.cpu().numpy(), mr, max_value_norm(xs["v"])) <= 1.0, scale


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("tau", [0.02, 0.05, 0.1])
def test_prefill_layer_end_to_end(poem, tau):
    n, hq, hkv, d, B = 2048, 4, 1, 128, 128
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=11)
    q, k, v = to_dev(x)
    layer = poem.prefill_layer(q, k, v, tau, block=B)
    for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
        poem.poem_check(ws)
    T = n // B
    prob = problem_from(x, B)
    Ir, mr = prob.score_all()
    rp_ref, ci_ref, _ = oracle.select_all(hq, T, Ir, mr, tau)
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx.cpu().numpy()
    differ, bad = lists_agree_at_cut(csr_rows(rp, ci), csr_rows(rp_ref, ci_ref), Ir, mr, hq, T, tau)
    assert not bad, bad
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, _ = prob.masked_units(units, rp, ci)
    mx, mean = compare_fwd(layer.o, O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS
    # the error at the sampled queries obeys tau (and at the loosest tau some block is dropped)
    if tau >= 0.1:
        assert rp[-1] < hq * T * (T + 1) // 2
    for (h, i) in [(0, T - 1), (2, T // 2)]:
        keep = csr_rows(rp, ci)[h * T + i]
        for j in range(16):
            t = i * B + j * (B // 16)
            od, _ = prob.dense_row(h, t)
            ot, _ = prob.masked_row(h, t, keep)
            assert np.linalg.norm(od - ot) <= tau * (1 + 1e-3) + 1e-6


def test_strided_views_match_contiguous(poem):
    """Q, K, V as padded views (head stride and token stride larger than dense) and a
    padded O: the layer equals the contiguous run bit for bit, and the padding of O
    is never written."""
    n, hq, hkv, d, B, tau = 2048, 4, 2, 128, 128, 0.05
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=23)
    q, k, v = to_dev(x)
    ref = poem.prefill_layer(q, k, v, tau, block=B)
    for ws in (ref.ws_score, ref.ws_select, ref.ws_fwd):
        poem.poem_check(ws)

    def padded(t, extra_heads, extra_dim):
        big = torch.zeros(t.shape[0], t.shape[1] + extra_heads, t.shape[2] + extra_dim, dtype=t.dtype,
                          device=t.device)
        big[:, : t.shape[1], : t.shape[2]] = t
        return big[:, : t.shape[1], : t.shape[2]]

    qv, kv, vv = padded(q, 1, 64), padded(k, 2, 32), padded(v, 2, 32)  # K and V share one layout (ABI)
    assert qv.stride() != q.stride() and not qv.is_contiguous()
    lay = poem.prefill_layer(qv, kv, vv, tau, block=B)
    for ws in (lay.ws_score, lay.ws_select, lay.ws_fwd):
        poem.poem_check(ws)
    assert torch.equal(lay.I_hat, ref.I_hat) and torch.equal(lay.row_ptr, ref.row_ptr)
    assert torch.equal(lay.o, ref.o)
    # a padded O written through its own strides
    ob = torch.full((n, hq, d + 32), 7.0, dtype=torch.bfloat16, device="cuda")
    ov = ob[:, :, :d]
    poem.bsa_fwd(qv, kv, vv, ref.row_ptr, ref.col_idx, ov, ref.ws_fwd, block=B)
    poem.poem_check(ref.ws_fwd)
    assert torch.equal(ov, ref.o)
    assert bool((ob[:, :, d:] == 7.0).all())
    # the practical path reads strided inputs too (pooling)
    p_ref = poem.prefill_layer_practical(q, k, v, 1.0, 0.95, 0.5, block=B)
    p_str = poem.prefill_layer_practical(qv, kv, vv, 1.0, 0.95, 0.5, block=B)
    for ws in (p_ref.ws_pooled, p_str.ws_pooled):
        poem.poem_check(ws)
    assert torch.equal(p_ref.m_pool, p_str.m_pool) and torch.equal(p_ref.d_pool, p_str.d_pool)
