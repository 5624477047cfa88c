"""Oracle pins for a query offset (chunked prefill: the queries are the last
len(q) of the len(k) tokens, the convention of the "Block-Filtered Long-Context
Attention" page, Section 3.6).  A chunk's rows must equal the rows of the same
positions in the whole prefill -- scores, pooled estimates, dense and masked
attention -- and asking with misplaced query rows must change them (so the
offset is really applied)."""
import numpy as np
import pytest

import oracle
import poem_synth


@pytest.fixture(scope="module")
def layers():
    oracle.build()
    x = poem_synth.heavy_block_layer(1024, 4, 2, 32, block=64, seed=11, heavy_prob=0.3)
    full = oracle.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                          v=poem_synth.bf16_bits(x["v"]), block=64)
    off = 640  # 10 of 16 tiles are history
    chunk = oracle.Problem(q=poem_synth.bf16_bits(x["q"])[off:], k=poem_synth.bf16_bits(x["k"]),
                           v=poem_synth.bf16_bits(x["v"]), block=64)
    return full, chunk, off


def test_chunk_geometry(layers):
    full, chunk, off = layers
    assert chunk.n_tokens == 1024 and chunk.q_offset == off and chunk.q_tile0 == 10 and chunk.n_tiles == 16


def test_chunk_scores_equal_full_rows(layers):
    full, chunk, off = layers
    units = [(h, i) for h in range(4) for i in (10, 12, 15)]
    If, mf = full.score_units(units)
    Ic, mc = chunk.score_units(units)
    for h, i in units:
        o = oracle.tri_offset(16, h, i)
        np.testing.assert_array_equal(Ic[o:o + i + 1], If[o:o + i + 1])
        np.testing.assert_array_equal(mc[o:o + i + 1], mf[o:o + i + 1])


def test_chunk_pooled_equal_full_rows(layers):
    full, chunk, off = layers
    units = [(h, i) for h in range(4) for i in (10, 15)]
    mf, df = full.pooled_units(units)
    mc, dc = chunk.pooled_units(units)
    np.testing.assert_array_equal(mf, mc)
    np.testing.assert_array_equal(df, dc)


def test_chunk_attention_equal_full_rows(layers):
    full, chunk, off = layers
    units = [(1, 11), (3, 15)]
    Of, lf = full.dense_units(units)
    Oc, lc = chunk.dense_units(units)
    np.testing.assert_array_equal(Of, Oc)
    np.testing.assert_array_equal(lf, lc)
    rp, ci = poem_synth.random_block_lists(4, 16, 0.4, seed=2)
    Mf, _ = full.masked_units(units, rp, ci)
    Mc, _ = chunk.masked_units(units, rp, ci)
    np.testing.assert_array_equal(Mf, Mc)


def test_offset_is_applied(layers):
    """Feeding the chunk's query rows as if they started at position 0 gives
    different rows: the offset is not a no-op."""
    full, chunk, off = layers
    wrong = oracle.Problem(q=chunk.q, k=chunk.k[: len(chunk.q)], v=chunk.v[: len(chunk.q)], block=64)
    o1, _ = chunk.dense_row(0, off + 5)
    o2, _ = wrong.dense_row(0, 5)
    assert np.abs(o1 - o2).max() > 1e-3
