"""Helpers shared by the GPU parity tests: moving seeded inputs between the CUDA
path and the oracle, and the list-comparison rule at the selection cut."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import poem_synth

# Tolerances (hot-path contract): bsa_fwd on an identical list, unit-scale V.
FWD_MAX_ABS = 1e-2
FWD_MEAN_ABS = 1e-3
# I_hat / m_hat relative error, with a floor relative to the row maximum.
SCORE_REL = 1e-3
# Lists: only blocks whose oracle score lies within this relative band of the
# cut score may differ.
CUT_BAND = 1e-4


def problem_from(x: dict, block: int, n_sample: int = 16) -> oracle.Problem:
    return oracle.Problem(q=poem_synth.bf16_bits(x["q"]), k=poem_synth.bf16_bits(x["k"]),
                          v=poem_synth.bf16_bits(x["v"]), block=block, n_sample=n_sample)


def to_dev(x: dict):
    return x["q"].cuda(), x["k"].cuda(), x["v"].cuda()


def csr_rows(row_ptr, col_idx):
    rp = np.asarray(row_ptr)
    ci = np.asarray(col_idx)
    return [ci[rp[r]:rp[r + 1]].tolist() for r in range(len(rp) - 1)]


def compare_fwd(o_gpu: torch.Tensor, O_ref: np.ndarray, units, block: int):
    """o_gpu [N, Hq, d] bf16 vs oracle O [n_units, B, d]; returns (max_abs, mean_abs)."""
    og = o_gpu.float().cpu().numpy()
    errs = []
    for u, (h, i) in enumerate(units):
        errs.append(np.abs(og[i * block:(i + 1) * block, h, :] - O_ref[u]))
    e = np.concatenate([x.ravel() for x in errs])
    return float(e.max()), float(e.mean())


def score_rel_err(gpu: np.ndarray, ref: np.ndarray, n_q_heads: int, n_tiles: int):
    """Max relative error of packed scores, floored at 1e-3 of each row's max."""
    worst = 0.0
    for h in range(n_q_heads):
        for i in range(n_tiles):
            off = oracle.tri_offset(n_tiles, h, i)
            r = ref[off:off + i + 1]
            g = gpu[off:off + i + 1]
            floor = 1e-3 * max(float(r.max()), 1e-30)
            worst = max(worst, float(np.max(np.abs(g - r) / np.maximum(r, floor))))
    return worst


def lists_agree_at_cut(gpu_rows, ref_rows, Ihat_ref, mhat_ref, n_q_heads, n_tiles, tau):
    """Rows must match exactly, except for blocks whose reference score lies within
    CUT_BAND (relative) of the row's cut score, or -- when the reference slack of
    the stopping test at the cut is within CUT_BAND * tau -- one block at the cut.
    Returns (n_rows_differing, list of violations)."""
    bad = []
    differ = 0
    for h in range(n_q_heads):
        for i in range(n_tiles):
            r = h * n_tiles + i
            a, b = set(gpu_rows[r]), set(ref_rows[r])
            if a == b:
                continue
            differ += 1
            off = oracle.tri_offset(n_tiles, h, i)
            Ih = np.asarray(Ihat_ref[off:off + i + 1], dtype=np.float64)
            mh = np.asarray(mhat_ref[off:off + i + 1], dtype=np.float64)
            cand = sorted(range(1, i - 1), key=lambda x: (-Ih[x], x))
            k = len([x for x in cand if x in b])
            cut_scores = [Ih[cand[k - 1]]] if k > 0 else []
            if k < len(cand):
                cut_scores.append(Ih[cand[k]])
            sym = a ^ b
            in_band = all(any(abs(Ih[x] - c) <= CUT_BAND * max(c, 1e-30) for c in cut_scores) for x in sym)
            if in_band:
                continue
            # slack rule: S_I - tau (1 - S_m) near zero at k-1 or k; one block may move
            ok_slack = False
            for kk in (k - 1, k, k + 1):
                if 0 <= kk <= len(cand):
                    D = cand[kk:]
                    SI = float(sum(Ih[x] for x in D))
                    SM = float(sum(mh[x] for x in D))
                    if abs(SI - tau * (1 - SM)) <= CUT_BAND * tau and len(sym) <= 1:
                        ok_slack = True
            if not ok_slack:
                bad.append((h, i, sorted(a - b), sorted(b - a)))
    return differ, bad
