"""Pins of the practical (estimated-score) selector in the oracle.

The estimators of practical POEM are not printed on the pages, so the pooled
reading cannot be checked against printed values.  What can be pinned: with one
token per block and one query per tile, pooling is exact and the estimates must
equal the exact definitions of Section 4.1 / Equation (4); the selection rule is
checked in exact rational arithmetic (shortlist by mass, rerank, pooled-mass
threshold), for nesting in the threshold, and for its limits."""
import math
from fractions import Fraction

import numpy as np
import pytest


def test_pooled_estimates_equal_exact_scores_with_one_token_per_block(oracle_mod):
    rng = np.random.default_rng(3)
    for seed in range(3):
        n, d = 12, 3
        q = rng.normal(size=(n, 2, d)) * 1.3
        k = rng.normal(size=(n, 1, d)) * 1.3
        v = rng.normal(size=(n, 1, d))
        p = oracle_mod.Problem(q=q, k=k, v=v, block=1, n_sample=1)
        mp, dp = p.pooled_all()
        for h in range(2):
            for i in range(n):
                m, vb, I, o = p.block_stats(h, i)
                off = oracle_mod.tri_offset(n, h, i)
                np.testing.assert_allclose(mp[off:off + i + 1], m, atol=1e-14)
                np.testing.assert_allclose(mp[off:off + i + 1] * dp[off:off + i + 1], I, atol=1e-13)


def test_pooled_toy_example(oracle_mod):
    # the three-block toy (one token per block): m~ = (1/2, 1/4, 1/4), d~ = (0, 2, 2)
    q = np.array([[[0.0]], [[0.0]], [[1.0]]])
    k = np.array([[[math.log(2.0)]], [[0.0]], [[0.0]]])
    v = np.array([[[2.0]], [[0.0]], [[4.0]]])
    p = oracle_mod.Problem(q=q, k=k, v=v, block=1, n_sample=1, scale=1.0)
    mp, dp = p.pooled_units([(0, 2)])
    off = oracle_mod.tri_offset(3, 0, 2)
    np.testing.assert_allclose(mp[off:off + 3], [0.5, 0.25, 0.25], atol=1e-15)
    np.testing.assert_allclose(dp[off:off + 3], [0.0, 2.0, 2.0], atol=1e-14)


def test_pooled_means_with_larger_blocks(oracle_mod):
    rng = np.random.default_rng(9)
    n, d, B = 32, 4, 8
    q, k, v = rng.normal(size=(n, 1, d)), rng.normal(size=(n, 1, d)), rng.normal(size=(n, 1, d))
    p = oracle_mod.Problem(q=q, k=k, v=v, block=B, n_sample=4)
    mp, dp = p.pooled_all()
    T = n // B
    for i in range(T):
        qm = q[i * B:(i + 1) * B, 0].mean(0)
        km = np.stack([k[b * B:(b + 1) * B, 0].mean(0) for b in range(i + 1)])
        vm = np.stack([v[b * B:(b + 1) * B, 0].mean(0) for b in range(i + 1)])
        off = oracle_mod.tri_offset(T, 0, i)
        # the pooled masses are a softmax of the pooled logits: log-ratios are exact
        lm = np.log(mp[off:off + i + 1])
        lg = km @ qm / math.sqrt(d)
        np.testing.assert_allclose(lm - lm[0], lg - lg[0], atol=1e-12)
        assert mp[off:off + i + 1].sum() == pytest.approx(1.0, abs=1e-14)
        # sum_b m~_b (v~_b - o~) = 0, so o~ is recovered from the deviations' weights
        assert np.all(dp[off:off + i + 1] >= 0)


def _rational_practical(i, m, dv, w, gamma, rho):
    cand = list(range(1, i - 1))
    s1 = sorted(cand, key=lambda b: (-Fraction(m[b]), b))
    n1 = min(len(cand), math.ceil(rho * len(cand)))
    short = s1[:n1]

    def key(b):
        if m[b] <= 0 or (w > 0 and dv[b] <= 0):
            return -math.inf
        return math.log(m[b]) + (w * math.log(dv[b]) if w > 0 else 0.0)

    s2 = sorted(short, key=lambda b: (-key(b), b))
    mand = {0, i} | ({i - 1} if i >= 1 else set())
    acc = sum(Fraction(m[b]) for b in mand)
    kept = set(mand)
    kk = 0
    while kk < len(s2) and acc < Fraction(gamma):
        acc += Fraction(m[s2[kk]])
        kept.add(s2[kk])
        kk += 1
    return sorted(kept), kk


def test_practical_selection_rule(oracle_mod):
    rng = np.random.default_rng(17)
    for trial in range(300):
        i = int(rng.integers(0, 20))
        raw = rng.integers(1, 64, size=i + 1).astype(float)
        raw[rng.random(i + 1) < 0.15] = 8.0  # ties
        m = raw / raw.sum()
        dv = rng.integers(0, 16, size=i + 1) / 8.0
        w = float(rng.choice([0.0, 0.5, 1.0, 2.0]))
        gamma = float(rng.choice([0.5, 0.8, 0.95, 1.5]))
        rho = float(rng.choice([0.0, 0.3, 1.0]))
        keep, k = oracle_mod.select_practical_row(i, m, dv, w, gamma, rho)
        ref, kref = _rational_practical(i, m, dv, w, gamma, rho)
        assert keep.tolist() == ref and k == kref, (i, w, gamma, rho)


def test_practical_nested_in_gamma_and_limits(oracle_mod):
    rng = np.random.default_rng(23)
    for _ in range(100):
        i = int(rng.integers(3, 40))
        m = rng.random(i + 1) ** 3
        m /= m.sum()
        dv = rng.random(i + 1)
        prev = None
        for gamma in (0.5, 0.9, 0.99):
            keep, _ = oracle_mod.select_practical_row(i, m, dv, 1.0, gamma, 0.5)
            if prev is not None:
                assert set(prev) <= set(keep)
            prev = keep
        # gamma above 1 keeps the whole shortlist; rho = 0 keeps only mandatory blocks
        all_short, _ = oracle_mod.select_practical_row(i, m, dv, 1.0, 2.0, 1.0)
        assert all_short.tolist() == list(range(i + 1))
        mand_only, _ = oracle_mod.select_practical_row(i, m, dv, 1.0, 2.0, 0.0)
        assert mand_only.tolist() == sorted({0, i - 1, i})
