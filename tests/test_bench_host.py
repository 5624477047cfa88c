"""Host arithmetic of the benchmark (CPU): the FLOP counts that the roofline figures
divide by, checked against brute-force counts of causal (query, key) pairs."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _pairs_brute(row_ptr, col_idx, n_tiles, B, q_tile0):
    """Visible (query, key) pairs of every listed block, one by one: query t of local
    tile i sits at key position (q_tile0 + i) B + t and sees keys at or before it."""
    pairs = 0
    for r in range(len(row_ptr) - 1):
        g = r % n_tiles + q_tile0
        for b in col_idx[row_ptr[r]:row_ptr[r + 1]]:
            for t in range(B):
                qpos = g * B + t
                pairs += sum(1 for u in range(b * B, (b + 1) * B) if u <= qpos)
    return pairs


def _random_lists(n_heads, n_tiles, q_tile0, rng, p=0.5):
    rows = []
    for _ in range(n_heads):
        for i in range(n_tiles):
            g = q_tile0 + i
            keep = [b for b in range(g + 1) if rng.random() < p]
            rows.append(keep)
    row_ptr = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    col_idx = np.array([b for x in rows for b in x], dtype=np.int32)
    return row_ptr, col_idx


def test_retained_flops_counts_causal_pairs():
    rng = np.random.default_rng(5)
    for B, d in ((4, 8), (8, 16)):
        for q_tile0 in (0, 3):
            for p in (0.3, 1.0):
                row_ptr, col_idx = _random_lists(2, 5, q_tile0, rng, p)
                want = 4 * d * _pairs_brute(row_ptr, col_idx, 5, B, q_tile0)
                assert bench.retained_flops(row_ptr, col_idx, 5, d, B, q_tile0) == want


def test_retained_flops_empty_rows_and_no_diagonal():
    # rows without their diagonal block count full blocks only; empty rows count nothing
    row_ptr = np.array([0, 0, 1, 1, 3], dtype=np.int32)
    col_idx = np.array([0, 0, 1], dtype=np.int32)
    n_tiles, B, d = 4, 4, 2
    want = 4 * d * _pairs_brute(row_ptr, col_idx, n_tiles, B, 0)
    assert bench.retained_flops(row_ptr, col_idx, n_tiles, d, B) == want


def test_dense_flops_is_every_causal_pair():
    for n, hq, d in ((8, 2, 4), (13, 3, 8)):
        pairs = sum(t + 1 for t in range(n))
        assert bench.dense_flops(n, hq, d) == 4 * d * hq * pairs


def test_all_blocks_listed_equals_dense():
    n_tiles, B, d, hq = 6, 8, 16, 3
    rows = [list(range(i % n_tiles + 1)) for i in range(hq * n_tiles)]
    row_ptr = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    col_idx = np.array([b for x in rows for b in x], dtype=np.int32)
    assert bench.retained_flops(row_ptr, col_idx, n_tiles, d, B) == bench.dense_flops(n_tiles * B, hq, d)


def test_sampled_oracle_cross_check_scores_a_planted_error():
    """The benchmark's cross-check on sampled units: rows taken from the oracle itself
    give zero errors and equal lists; a 0.3% error planted in one score row shows up
    as ~3 tolerances, and a shifted output row as its shift."""
    import oracle
    import poem_synth

    oracle.build()
    n, hq, hkv, d, B, tau = 2048, 2, 1, 64, 128, 0.05
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=3)
    prob = oracle.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                          v=poem_synth.bf16_bits(x["v"]), block=B, n_sample=16)

    def rows_from_oracle(h, i, plant=False):
        Ih, mh = prob.score_units([(h, i)])
        off = oracle.tri_offset(T, h, i)
        I, m = Ih[off:off + i + 1].copy(), mh[off:off + i + 1].copy()
        keep, _ = oracle.select_row(i, I, m, tau)
        rp = np.zeros(hq * T + 1, dtype=np.int32)
        rp[h * T + i + 1:] = len(keep)
        O, _ = prob.masked_units([(h, i)], rp, np.asarray(keep, dtype=np.int32))
        o = np.asarray(O[0])[:B].copy()
        if plant:
            I[np.argmax(I)] *= 1.003
            o[0, 0] += 0.25
        return I, m, np.asarray(keep, dtype=np.int32), o

    clean = bench.cpu_baseline(x, n, hq, hkv, d, B, tau, 1e9, gpu_rows=rows_from_oracle)["parity"]
    assert clean["units"] >= 2 and clean["lists_equal"] == clean["units"]
    assert clean["score_tol_ratio_max"] == 0.0 and clean["o_max_abs"] == 0.0
    bad = bench.cpu_baseline(x, n, hq, hkv, d, B, tau, 1e9,
                             gpu_rows=lambda h, i: rows_from_oracle(h, i, plant=True))["parity"]
    assert 2.0 < bad["score_tol_ratio_max"] < 3.1
    assert abs(bad["o_max_abs"] - 0.25) < 1e-9


def test_oracle_sample_reaches_the_last_tile_and_balances_pairs():
    """The CPU-baseline sample: at least 16 units at 128K, the last tile included,
    every tile pair (i, T-1-i) holding T + 1 visible blocks."""
    T = 1024
    units = bench.oracle_sample_units(32, T, 16)
    tiles = sorted(i for _, i in units)
    assert len(units) >= 16 and tiles[-1] == T - 1 and tiles[0] == 0
    lo = [i for i in tiles if i < T // 2]
    hi = sorted((i for i in tiles if i >= T // 2), reverse=True)
    assert len(lo) == len(hi) and all(a + b == T - 1 for a, b in zip(lo, hi))
    assert units == sorted(units, key=lambda u: -u[1])
    assert len(set(units)) == len(units) and all(0 <= h < 32 for h, _ in units)
