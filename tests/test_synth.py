"""Seeded input generators: determinism and the structure the recipes state."""
import numpy as np
import torch

import poem_synth


def test_generators_are_deterministic():
    a = poem_synth.heavy_block_layer(512, 4, 2, 32, block=64, seed=3)
    b = poem_synth.heavy_block_layer(512, 4, 2, 32, block=64, seed=3)
    c = poem_synth.heavy_block_layer(512, 4, 2, 32, block=64, seed=4)
    assert poem_synth.digest(a["q"], a["k"], a["v"]) == poem_synth.digest(b["q"], b["k"], b["v"])
    assert poem_synth.digest(a["q"], a["k"], a["v"]) != poem_synth.digest(c["q"], c["k"], c["v"])
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (512, 4, 32) and a["k"].shape == (512, 2, 32)


def test_single_head_recipe():
    x = poem_synth.single_head(1024, 64, seed=0)
    assert x["q"].shape == (1024, 1, 64) and x["q"].dtype == torch.float32
    logits = (x["q"][:, 0] @ x["k"][:, 0].T) / 8.0
    assert 1.8 < float(logits.std()) < 2.2


def test_heavy_keys_get_the_logit_boost():
    x = poem_synth.heavy_block_layer(2048, 4, 1, 128, block=128, rope_base=500000.0, seed=1, heavy_prob=0.3,
                                     beta_range=(5.0, 5.0))
    heavy = x["heavy"][0]
    assert 0 < int(heavy.sum()) < 16
    q = x["q"].float()[1024:1040, 0]
    k = x["k"].float()[:, 0]
    s = (q @ k.T) / np.sqrt(128)
    tok_heavy = heavy.repeat_interleave(128)
    gap = float(s[:, tok_heavy].mean() - s[:, ~tok_heavy].mean())
    assert 3.0 < gap < 6.0


def test_random_block_lists_structure():
    rp, ci = poem_synth.random_block_lists(2, 20, 0.25, seed=5)
    for r in range(40):
        i = r % 20
        row = ci[rp[r]:rp[r + 1]]
        assert row[0] == 0 and row[-1] == i and np.all(np.diff(row) > 0)
        assert len(row) == max(len({0, i}), int(round(0.25 * (i + 1))))
    rp1, ci1 = poem_synth.random_block_lists(2, 20, 1.0, seed=5)
    assert rp1[-1] == 2 * 20 * 21 // 2


def test_contrast_layer_structure():
    x = poem_synth.contrast_layer(4096, 4, 2, 64, block=128, seed=2, heavy_prob=0.3)
    y = poem_synth.heavy_block_layer(4096, 4, 2, 64, block=128, seed=2, heavy_prob=0.3)
    assert torch.equal(x["q"], y["q"]) and torch.equal(x["k"], y["k"])
    v = x["v"].float().view(32, 128, 2, 64).mean(1)  # block means [T, Hkv, d]
    for g in range(2):
        heavy, flat, sign, dev = x["heavy"][g], x["flat"][g], x["pair_sign"][g], x["deviant"][g]
        assert not (flat & ~heavy).any() and not (dev & heavy).any()
        assert int((sign == 1).sum()) == int((sign == -1).sum())
        pos = torch.nonzero(sign == 1).flatten()
        neg = torch.nonzero(sign == -1).flatten()
        for a, b in zip(pos.tolist(), neg.tolist()):
            # opposite offsets: the pair's block means nearly cancel
            assert float((v[a, g] + v[b, g]).norm()) < 1.6 < float(v[a, g].norm())
        if dev.any():
            assert float(v[dev, g].norm(dim=-1).min()) > 4.0
