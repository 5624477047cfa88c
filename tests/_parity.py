"""Helpers shared by the GPU parity tests: moving seeded inputs between the CUDA
path and the oracle, and the list-comparison rule at the selection cut."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import poem_synth

# Tolerances: bsa_fwd on an identical list, unit-scale V.
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


# bsa_fwd writes O in bf16: rounding to nearest bf16 (8-bit significand) moves a
# value x by at most 2^-8 |x|, which alone exceeds FWD_MAX_ABS once |x| > 2.56.
BF16_ROUND_REL = 2.0 ** -8


def compare_fwd_excess(o_gpu: torch.Tensor, O_ref: np.ndarray, units, block: int):
    """Like compare_fwd, but the element bound adds the bf16 output rounding:
    |o_gpu - o_ref| <= FWD_MAX_ABS + BF16_ROUND_REL |o_ref|.  Returns (largest
    violation ratio (<= 1 passes), mean_abs)."""
    og = o_gpu.float().cpu().numpy()
    worst, tot, cnt = 0.0, 0.0, 0
    for u, (h, i) in enumerate(units):
        ref = O_ref[u]
        e = np.abs(og[i * block:(i + 1) * block, h, :] - ref)
        worst = max(worst, float(np.max(e / (FWD_MAX_ABS + BF16_ROUND_REL * np.abs(ref)))))
        tot += float(e.sum())
        cnt += e.size
    return worst, tot / cnt


def bf16_half_ulp(x):
    """Half a bf16 unit in the last place at |x| (8 significant bits): the most that
    rounding a value of that magnitude to bf16 can move it (2^(e-8) for |x| in
    [2^e, 2^(e+1)))."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.floor(np.log2(ax)) - 8).astype(np.int64))


def fwd_out_excess(o_gpu_rows, o_ref_rows):
    """bsa_fwd rows (bf16 values, as floats) against oracle rows: the largest ratio
    |o_gpu - o_ref| / (FWD_MAX_ABS + bf16_half_ulp(o_ref)) (<= 1 passes) and the mean
    abs error.  FWD_MAX_ABS bounds the fp32-accumulated arithmetic; the output buffer
    is bf16, and storing a value in it moves it by up to half a bf16 ulp -- 0.0078 at
    |o| in [2, 4), 0.0156 at [4, 8) -- which no kernel can avoid."""
    got = np.asarray(o_gpu_rows, np.float64)
    ref = np.asarray(o_ref_rows, np.float64)
    e = np.abs(got - ref)
    return float(np.max(e / (FWD_MAX_ABS + bf16_half_ulp(ref)))), float(e.mean())


def score_err_excess(gpu_I, ref_I, gpu_m, ref_m, R: float):
    """Largest violation ratio of the score tolerances (<= 1 passes):
      |dI_b| <= SCORE_REL * I_b + 1e-5 * m_b * R
      |dm_b| <= SCORE_REL * m_b + 1e-9
    where R = max_t ||v_t||.  The absolute terms cover exact cancellation (e.g. the
    single visible block of tile 0, where v_b = o and I_b = 0): r_b = P_b V_b - m_b o
    is formed in fp32 from P split into bf16 hi/lo (about 2^-17 relative per weight),
    leaving ~2^-17 m_b R absolute error; masses below ~1e-9 sit at the fp32
    flush-to-zero limit of the exponential."""
    gI, rI = np.asarray(gpu_I, np.float64), np.asarray(ref_I, np.float64)
    gm, rm = np.asarray(gpu_m, np.float64), np.asarray(ref_m, np.float64)
    tolI = SCORE_REL * rI + 1e-5 * rm * R + 1e-30
    tolm = SCORE_REL * rm + 1e-9
    return float(max(np.max(np.abs(gI - rI) / tolI), np.max(np.abs(gm - rm) / tolm)))


def masked_rows_threaded(prob, items):
    """Oracle masked-attention rows for a list of (h, token, blocks) items, computed
    concurrently on the host cores (each oracle call is one row, single-threaded,
    and releases the interpreter lock).  Returns an array [len(items), d]."""
    from concurrent.futures import ThreadPoolExecutor

    with ThreadPoolExecutor(max_workers=max(1, oracle.num_threads())) as ex:
        rows = list(ex.map(lambda it: prob.masked_row(it[0], it[1], it[2])[0], items))
    return np.stack(rows) if rows else np.zeros((0, prob.head_dim))


def max_value_norm(v: torch.Tensor) -> float:
    return float(v.float().norm(dim=-1).max())


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


# ---------------------------------------------------------------------------
# Practical (pooled-estimate) selector
# ---------------------------------------------------------------------------

# Pooled estimates m~, d~ are formed in fp32 from fp32 tile/block means:
#   |dm| <= POOL_REL * m + 1e-9,   |dd| <= POOL_REL * d + 1e-5 * max ||v~||
# (the absolute term covers d~ near 0, where fp32 cancellation leaves ~1e-6 |v~|).
POOL_REL = 1e-4


def pooled_err_excess(gpu_m, ref_m, gpu_d, ref_d, vbar_norm: float):
    gm, rm = np.asarray(gpu_m, np.float64), np.asarray(ref_m, np.float64)
    gd, rd = np.asarray(gpu_d, np.float64), np.asarray(ref_d, np.float64)
    tolm = POOL_REL * rm + 1e-9
    told = POOL_REL * rd + 1e-5 * vbar_norm + 1e-30
    return float(max(np.max(np.abs(gm - rm) / tolm), np.max(np.abs(gd - rd) / told)))


def _practical_keys(m, d, w):
    with np.errstate(divide="ignore"):
        lm = np.where(m > 0, np.log(np.where(m > 0, m, 1.0)), -np.inf)
        ld = np.where(d > 0, np.log(np.where(d > 0, d, 1.0)), -np.inf)
    if w == 0:
        return lm
    key = lm + w * np.where(np.isfinite(ld), ld, 0.0)
    return np.where((lm == -np.inf) | (ld == -np.inf), -np.inf, key)


def practical_row_ambiguous(i, m, d, w, gamma, rho, band_m, band_key, band_acc):
    """True when a perturbation of the row's estimates within the bands could change
    its kept set: a near-tie at the stage-1 shortlist boundary (relative band_m), a
    near-tie of the stage-2 keys across the cut (absolute band_key, log domain), or
    an accumulated mass within band_acc of gamma at the cut."""
    m = np.asarray(m, np.float64)
    d = np.asarray(d, np.float64)
    cand = np.arange(1, max(i - 1, 1), dtype=np.int64) if i >= 3 else np.zeros(0, np.int64)
    nc = cand.size
    o1 = cand[np.lexsort((cand, -m[cand]))] if nc else cand
    n1 = min(nc, max(0, int(np.ceil(rho * nc))))
    if 0 < n1 < nc and abs(m[o1[n1 - 1]] - m[o1[n1]]) <= band_m * max(m[o1[n1 - 1]], 1e-300):
        return True
    sl = o1[:n1]
    key = _practical_keys(m[sl], d[sl], w)
    o2 = sl[np.lexsort((sl, -key))]
    k2 = _practical_keys(m[o2], d[o2], w)
    acc = m[0]
    if i >= 2:
        acc += m[i - 1]
    if i >= 1:
        acc += m[i]
    accs = [acc]
    for b in o2:
        acc += m[b]
        accs.append(acc)
    kcut = next((k for k, a in enumerate(accs) if a >= gamma), n1)
    for k in (kcut - 1, kcut):
        if 0 <= k <= n1 and abs(accs[k] - gamma) <= band_acc:
            return True
    if 0 < kcut < n1 and np.isfinite(k2[kcut - 1]) and abs(k2[kcut - 1] - k2[kcut]) <= band_key:
        return True
    return False


def check_list_valid(rows, n_tiles):
    """Every row ascending, unique, within 0..i and holding the mandatory blocks."""
    for r, row in enumerate(rows):
        i = r % n_tiles
        assert row == sorted(set(row)), r
        assert all(0 <= b <= i for b in row), r
        mand = {0, i} | ({i - 1} if i >= 1 else set())
        assert mand <= set(row), r


def practical_lists_agree(gpu_rows, ref_rows, m_ref, d_ref, n_q_heads, n_tiles, w, gamma, rho, band_m, band_key,
                          band_acc, rows=None):
    """Rows must match exactly unless practical_row_ambiguous flags them on the
    reference estimates.  Returns (n_rows_differing, violations)."""
    bad, differ = [], 0
    rows = range(n_q_heads * n_tiles) if rows is None else rows
    for r in rows:
        if list(gpu_rows[r]) == list(ref_rows[r]):
            continue
        differ += 1
        h, i = divmod(r, n_tiles)
        off = oracle.tri_offset(n_tiles, h, i)
        if not practical_row_ambiguous(i, m_ref[off:off + i + 1], d_ref[off:off + i + 1], w, gamma, rho, band_m,
                                       band_key, band_acc):
            bad.append((h, i, sorted(set(gpu_rows[r]) - set(ref_rows[r])), sorted(set(ref_rows[r]) - set(gpu_rows[r]))))
    return differ, bad
