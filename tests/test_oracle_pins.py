"""Pins of the fp64 oracle against facts the method description fixes.

Nothing here compares the oracle with itself: every check is a worked value
printed in the description (golden fixture), an exact identity or bound of
Section 4.1 / Equations (3)-(4) checked by brute force over every subset, a
textbook special case computed by a library routine (PyTorch float64 SDPA), or
a property of the selection rule verified in exact rational arithmetic.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "toy_three_block.json")


def _frac(s):
    return float(Fraction(s))


def _toy(oracle, shift=0.0):
    q = np.array([[[0.0]], [[0.0]], [[1.0]]])  # only the last query (t = 2) is used
    k = np.array([[[math.log(2.0)]], [[0.0]], [[0.0]]])
    v = np.array([[[2.0]], [[0.0]], [[4.0]]]) + shift
    return oracle.Problem(q=q, k=k, v=v, block=1, n_sample=1, scale=1.0)


# ---------------------------------------------------------------------------
# Worked example (Section 4.1) and the shift check
# ---------------------------------------------------------------------------

def test_toy_dense_output_and_removals(oracle_mod):
    g = json.load(open(GOLDEN))
    p = _toy(oracle_mod)
    o, _ = p.dense_row(0, 2)
    assert o[0] == pytest.approx(_frac(g["dense_output"]), abs=1e-14)
    names = g["block_names"]
    for rem in g["removals"]:
        keep = [b for b, n in enumerate(names) if n not in rem["remove"]]
        ot, _ = p.masked_row(0, 2, keep)
        assert ot[0] == pytest.approx(_frac(rem["sparse_output"]), abs=1e-14), rem
        assert abs(o[0] - ot[0]) == pytest.approx(_frac(rem["abs_error"]), abs=1e-14), rem


def test_toy_block_stats_and_scores(oracle_mod):
    g = json.load(open(GOLDEN))
    p = _toy(oracle_mod)
    m, vb, I, o = p.block_stats(0, 2)
    np.testing.assert_allclose(m, [_frac(x) for x in g["masses"]], atol=1e-14)
    np.testing.assert_allclose(vb[:, 0], [_frac(x) for x in g["values"]], atol=1e-14)
    np.testing.assert_allclose(I, [_frac(x) for x in g["scores_I"]], atol=1e-14)
    # Eq. (4) for D = {B, C}: (I_B + I_C) / (1 - m_B - m_C) = 2, actual error 0.
    bound = (I[1] + I[2]) / (1 - m[1] - m[2])
    assert bound == pytest.approx(_frac(g["bound_remove_BC"]), abs=1e-14)
    # Singleton removals: I_b / (1 - m_b) equals the exact error.
    for b in range(3):
        keep = [c for c in range(3) if c != b]
        ot, _ = p.masked_row(0, 2, keep)
        assert abs(o[0] - ot[0]) == pytest.approx(I[b] / (1 - m[b]), abs=1e-14)


def test_toy_shift_invariance(oracle_mod):
    g = json.load(open(GOLDEN))["shift"]
    p0 = _toy(oracle_mod)
    p = _toy(oracle_mod, shift=_frac(g["c"]))
    o, _ = p.dense_row(0, 2)
    assert o[0] == pytest.approx(_frac(g["dense_output"]), abs=1e-13)
    ot, _ = p.masked_row(0, 2, [0, 2])
    assert ot[0] == pytest.approx(_frac(g["remove_B_sparse_output"]), abs=1e-13)
    assert abs(o[0] - ot[0]) == pytest.approx(_frac(g["remove_B_abs_error"]), abs=1e-13)
    # Deviations, hence the I_b scores, do not move under the shift.
    _, _, I0, _ = p0.block_stats(0, 2)
    _, _, I1, _ = p.block_stats(0, 2)
    np.testing.assert_allclose(I1, I0, atol=1e-13)


# ---------------------------------------------------------------------------
# Equation (3) identity, Equation (4) bound and the 2 R delta worst case,
# by brute force over every discarded subset of tiny random problems
# ---------------------------------------------------------------------------

def _tiny(oracle, seed, n=16, hq=2, hkv=1, d=4, block=4):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(n, hq, d)) * 1.5
    k = rng.normal(size=(n, hkv, d)) * 1.5
    v = rng.normal(size=(n, hkv, d))
    return oracle.Problem(q=q, k=k, v=v, block=block, n_sample=block // 2 if block > 1 else 1)


@pytest.mark.parametrize("seed,block,d", [(0, 2, 3), (1, 4, 4), (2, 3, 2)])
def test_eq3_identity_eq4_bound_worst_case_brute_force(oracle_mod, seed, block, d):
    n = 12 if block == 3 else 16
    p = _tiny(oracle_mod, seed, n=n, d=d, block=block)
    R = np.max(np.linalg.norm(p.v, axis=-1))
    checked = 0
    for h in range(p.n_q_heads):
        for t in range(n):
            m, vb, I, o = p.block_stats(h, t)
            nb = len(m)
            for r in range(1, nb + 1):
                for D in itertools.combinations(range(nb), r):
                    delta = sum(m[b] for b in D)
                    if delta >= 1.0 - 1e-12:
                        continue
                    keep = [b for b in range(nb) if b not in D]
                    ot, _ = p.masked_row(h, t, keep)
                    err = o - ot
                    rhs = sum(m[b] * (vb[b] - o) for b in D) / (1.0 - delta)
                    # fp64 rounding is amplified by 1 / (1 - delta)
                    tol = 1e-12 / (1.0 - delta)
                    np.testing.assert_allclose(err, rhs, atol=tol, rtol=0)
                    bound = sum(I[b] for b in D) / (1.0 - delta)
                    assert np.linalg.norm(err) <= bound + tol
                    assert np.linalg.norm(err) <= 2.0 * R * delta + tol
                    checked += 1
    assert checked > 100


def test_mass_and_deviation_sums(oracle_mod):
    p = _tiny(oracle_mod, 5, n=16, d=4, block=4)
    for h in range(p.n_q_heads):
        for t in range(16):
            m, vb, I, o = p.block_stats(h, t)
            assert m.sum() == pytest.approx(1.0, abs=1e-14)
            # sum_b m_b v_b = o, so the signed deviations cancel.
            np.testing.assert_allclose((m[:, None] * (vb - o)).sum(0), 0.0, atol=1e-13)
            np.testing.assert_allclose(I, m * np.linalg.norm(vb - o, axis=1), atol=1e-14)


# ---------------------------------------------------------------------------
# Dense and masked attention against a library routine
# ---------------------------------------------------------------------------

def _sdpa_f64(q, k, v, scale):
    hq, hkv = q.shape[1], k.shape[1]
    G = hq // hkv
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, 0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    s = (qt @ kt.transpose(1, 2)) * scale
    n = q.shape[0]
    s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    return o.permute(1, 0, 2).numpy(), torch.logsumexp(s, -1).numpy()


def test_dense_and_all_blocks_match_sdpa_f64(oracle_mod):
    rng = np.random.default_rng(11)
    n, hq, hkv, d, B = 64, 4, 2, 8, 8
    q = rng.normal(size=(n, hq, d))
    k = rng.normal(size=(n, hkv, d)) * 2
    v = rng.normal(size=(n, hkv, d))
    p = oracle_mod.Problem(q=q, k=k, v=v, block=B, n_sample=4)
    ref_o, ref_lse = _sdpa_f64(q, k, v, 1.0 / math.sqrt(d))
    T = n // B
    units = [(h, i) for h in range(hq) for i in range(T)]
    O, lse = p.dense_units(units)
    # all-blocks CSR
    rows = [list(range(i + 1)) for h in range(hq) for i in range(T)]
    row_ptr = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    col_idx = np.concatenate(rows).astype(np.int32)
    Om, lsem = p.masked_units(units, row_ptr, col_idx)
    for u, (h, i) in enumerate(units):
        sl = slice(i * B, (i + 1) * B)
        np.testing.assert_allclose(O[u], ref_o[sl, h], atol=1e-12)
        np.testing.assert_allclose(Om[u], ref_o[sl, h], atol=1e-12)
        np.testing.assert_allclose(lse[u], ref_lse[h, sl], atol=1e-12)
        np.testing.assert_allclose(lsem[u], ref_lse[h, sl], atol=1e-12)


def test_masked_matches_sdpa_with_block_mask(oracle_mod):
    rng = np.random.default_rng(12)
    n, hq, hkv, d, B = 48, 2, 1, 8, 8
    q, k, v = rng.normal(size=(n, hq, d)), rng.normal(size=(n, hkv, d)), rng.normal(size=(n, hkv, d))
    p = oracle_mod.Problem(q=q, k=k, v=v, block=B, n_sample=4)
    T = n // B
    lists = {(h, i): sorted(set([i]) | set(rng.choice(i + 1, size=(i + 1) // 2, replace=False).tolist()))
             for h in range(hq) for i in range(T)}
    units = list(lists)
    row_ptr = np.zeros(hq * T + 1, dtype=np.int32)
    for (h, i), l in lists.items():
        row_ptr[h * T + i + 1] = len(l)
    row_ptr = np.cumsum(row_ptr).astype(np.int32)
    col_idx = np.concatenate([lists[(h, i)] for h in range(hq) for i in range(T)]).astype(np.int32)
    O, _ = p.masked_units(units, row_ptr, col_idx)
    for u, (h, i) in enumerate(units):
        mask = torch.zeros(B, n, dtype=torch.bool)
        for b in lists[(h, i)]:
            mask[:, b * B:(b + 1) * B] = True
        causal = torch.arange(n)[None, :] <= (i * B + torch.arange(B))[:, None]
        mask &= causal
        qt = torch.from_numpy(q[i * B:(i + 1) * B, h])[None]
        kt = torch.from_numpy(k[:, 0])[None]
        vt = torch.from_numpy(v[:, 0])[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask[None], scale=1 / math.sqrt(d))
        np.testing.assert_allclose(O[u], ref[0].numpy(), atol=1e-12)


def test_bf16_inputs_widen_exactly(oracle_mod):
    import poem_synth

    x = poem_synth.iid_layer(32, 2, 1, 8, seed=3)
    p16 = oracle_mod.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                             v=poem_synth.bf16_bits(x["v"]), block=8, n_sample=4)
    p64 = oracle_mod.Problem(q=poem_synth.to_f64(x["q"]), k=poem_synth.to_f64(x["k"]),
                             v=poem_synth.to_f64(x["v"]), block=8, n_sample=4)
    for t in (0, 7, 31):
        a, la = p16.dense_row(1, t)
        b, lb = p64.dense_row(1, t)
        assert np.array_equal(a, b) and la == lb


# ---------------------------------------------------------------------------
# Score aggregation: sampled rows and max
# ---------------------------------------------------------------------------

def test_score_uses_exactly_the_strided_sampled_rows(oracle_mod):
    rng = np.random.default_rng(21)
    n, d, B, S = 32, 4, 8, 4
    q, k, v = rng.normal(size=(n, 1, d)), rng.normal(size=(n, 1, d)), rng.normal(size=(n, 1, d))
    p = oracle_mod.Problem(q=q, k=k, v=v, block=B, n_sample=S)
    T = n // B
    Ih, mh = p.score_all()
    stride = B // S
    for i in range(T):
        off = oracle_mod.tri_offset(T, 0, i)
        rows = [p.block_stats(0, i * B + j * stride) for j in range(S)]
        Is = np.stack([r[2] for r in rows])
        ms = np.stack([r[0] for r in rows])
        for b in range(i + 1):
            # the aggregate is attained by one sampled row and bounds all of them
            assert np.any(Is[:, b] == Ih[off + b]) and np.all(Is[:, b] <= Ih[off + b])
            assert np.any(ms[:, b] == mh[off + b]) and np.all(ms[:, b] <= mh[off + b])
    # Perturbing a query that is not sampled leaves the scores unchanged;
    # perturbing a sampled one changes them.
    q2 = q.copy()
    q2[1 * B + 1] += 3.0  # offset 1 is not a multiple of the stride 2
    Ih2, _ = oracle_mod.Problem(q=q2, k=k, v=v, block=B, n_sample=S).score_all()
    assert np.array_equal(Ih2, Ih)
    q3 = q.copy()
    q3[1 * B + 2] += 3.0
    Ih3, _ = oracle_mod.Problem(q=q3, k=k, v=v, block=B, n_sample=S).score_all()
    assert not np.array_equal(Ih3, Ih)


# ---------------------------------------------------------------------------
# Selection rule
# ---------------------------------------------------------------------------

def _dyadic(rng, n, lo, hi, denom=1024):
    return np.array([rng.integers(lo * denom, hi * denom) / denom for _ in range(n)], dtype=np.float64)


def test_select_minimal_k_exact_arithmetic(oracle_mod):
    rng = np.random.default_rng(31)
    for trial in range(300):
        i = int(rng.integers(0, 14))
        Ih = _dyadic(rng, i + 1, 0, 1)
        if trial % 5 == 0 and i > 3:
            Ih[2] = Ih[3]  # force ties
        mh = _dyadic(rng, i + 1, 0, 1) / max(1, i)
        tau = float(rng.choice([0.0, 0.01, 0.05, 0.1, 0.5, 2.0]))
        keep, kcut = oracle_mod.select_row(i, Ih, mh, tau)
        cand = list(range(1, i - 1))
        ranked = sorted(cand, key=lambda b: (-Fraction(Ih[b]), b))

        def ok(k):
            D = ranked[k:]
            SI = sum((Fraction(Ih[b]) for b in D), Fraction(0))
            SM = sum((Fraction(mh[b]) for b in D), Fraction(0))
            return SM < 1 and SI <= Fraction(tau) * (1 - SM)

        k_ref = next(k for k in range(len(cand) + 1) if ok(k))
        assert kcut == k_ref
        mand = {0, i} | ({i - 1} if i >= 1 else set())
        expect = sorted(mand | set(ranked[:k_ref]))
        assert keep.tolist() == expect


def test_select_nested_in_tau(oracle_mod):
    rng = np.random.default_rng(41)
    for _ in range(200):
        i = int(rng.integers(3, 40))
        Ih = rng.random(i + 1) * rng.choice([0.01, 0.1, 1.0])
        mh = rng.random(i + 1) / (i + 1)
        prev = None
        for tau in (0.1, 0.05, 0.02):
            keep, _ = oracle_mod.select_row(i, Ih, mh, tau)
            if prev is not None:
                assert set(prev) <= set(keep)
            prev = keep


def test_select_tau_zero_keeps_every_positive_candidate(oracle_mod):
    i = 9
    Ih = np.array([0.3, 0.2, 0.0, 0.5, 0.0, 0.1, 0.4, 0.2, 0.7, 0.9])
    mh = np.full(i + 1, 0.05)
    keep, _ = oracle_mod.select_row(i, Ih, mh, 0.0)
    assert keep.tolist() == [0, 1, 3, 5, 6, 7, 8, 9]


def test_select_ties_prefer_smaller_id(oracle_mod):
    i = 8
    Ih = np.array([0, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0, 0], dtype=float)
    mh = np.full(i + 1, 0.01)
    # tau such that exactly two of the six tied candidates must be kept
    tau = 4 * 0.5 / (1 - 4 * 0.01) + 1e-9
    keep, k = oracle_mod.select_row(i, Ih, mh, tau)
    assert k == 2 and keep.tolist() == [0, 1, 2, 7, 8]


def test_select_small_tiles_all_mandatory(oracle_mod):
    for i in range(3):
        keep, k = oracle_mod.select_row(i, np.ones(i + 1), np.full(i + 1, 0.5), 0.0)
        assert keep.tolist() == list(range(i + 1)) and k == 0


def test_mass_only_keeps_same_number(oracle_mod):
    rng = np.random.default_rng(51)
    for _ in range(100):
        i = int(rng.integers(3, 30))
        Ih, mh = rng.random(i + 1), rng.random(i + 1) / i
        keep, k = oracle_mod.select_row(i, Ih, mh, 0.05)
        km = oracle_mod.select_mass_only_row(i, mh, k)
        assert len(km) == len(keep)
        cand = sorted(range(1, i - 1), key=lambda b: (-mh[b], b))
        assert set(km) == {0, i, i - 1} | set(cand[:k])


def test_selection_bounds_error_at_every_sampled_query(oracle_mod):
    """End-to-end invariant of the stopping rule: with max-aggregated I_b and
    m_b, every sampled query's error under the kept list is at most tau."""
    import poem_synth

    x = poem_synth.heavy_block_layer(256, 4, 2, 16, block=16, rope_base=10000.0, seed=7,
                                     beta_range=(2.0, 3.0))
    p = oracle_mod.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                           v=poem_synth.bf16_bits(x["v"]), block=16, n_sample=4)
    T = p.n_tiles
    Ih, mh = p.score_all()
    worst = 0.0
    dropped = 0
    for tau in (0.02, 0.1, 0.5):
        for h in range(4):
            for i in range(T):
                off = oracle_mod.tri_offset(T, h, i)
                keep, k = oracle_mod.select_row(i, Ih[off:off + i + 1], mh[off:off + i + 1], tau)
                dropped += (i + 1) - len(keep)
                for j in range(4):
                    t = i * 16 + j * 4
                    o, _ = p.dense_row(h, t)
                    ot, _ = p.masked_row(h, t, keep)
                    err = np.linalg.norm(o - ot)
                    worst = max(worst, err / tau)
                    assert err <= tau * (1 + 1e-9) + 1e-12
    assert dropped > 0  # the rule really drops blocks on this input
    assert worst > 0.0
