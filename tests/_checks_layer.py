"""Run by test_checks_gpu.py in a child process with POEM_LIBRARY_VARIANT=checks:
one small exact layer, a chunked call and the practical path through the debug
build of the library (device bounds checks on), each checked against the fp64
oracle; every poem_check must report POEM_OK (no bounds check fired)."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import block_sparse_attention_poem_b200 as poem  # noqa: E402
import oracle  # noqa: E402
import poem_synth  # noqa: E402
from _parity import (compare_fwd, csr_rows, lists_agree_at_cut, max_value_norm, problem_from,  # noqa: E402
                     score_err_excess)


def main():
    assert poem.LIB_PATH.endswith("libpoem_checks.so"), poem.LIB_PATH
    oracle.build()
    n, hq, hkv, d, B, tau = 2048, 4, 1, 128, 128, 0.2
    T = n // B
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=4)
    q, k, v = x["q"].cuda(), x["k"].cuda(), x["v"].cuda()
    layer = poem.prefill_layer(q, k, v, tau, block=B)
    for ws in (layer.ws_score, layer.ws_select, layer.ws_fwd):
        st = poem.poem_check_status(ws)
        assert st == 0, poem.STATUS[st]
    prob = problem_from(x, B)
    Ir, mr = prob.score_all()
    assert score_err_excess(layer.I_hat.cpu().numpy(), Ir, layer.m_hat.cpu().numpy(), mr, max_value_norm(x["v"])) <= 1
    rp = layer.row_ptr.cpu().numpy()
    ci = layer.col_idx[: int(rp[-1])].cpu().numpy()
    ref_rp, ref_ci, _ = oracle.select_all(hq, T, Ir, mr, tau)
    _, bad = lists_agree_at_cut(csr_rows(rp, ci), csr_rows(ref_rp, ref_ci), Ir, mr, hq, T, tau)
    assert not bad, bad
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, _ = prob.masked_units(units, rp, ci)
    mx, mean = compare_fwd(layer.o, O_ref, units, B)
    assert mx <= 1e-2 and mean <= 1e-3, (mx, mean)
    # a chunk: the last half of the queries against all keys
    ch = poem.prefill_layer(q[n // 2:].contiguous(), k, v, tau, block=B)
    for ws in (ch.ws_score, ch.ws_select, ch.ws_fwd):
        st = poem.poem_check_status(ws)
        assert st == 0, poem.STATUS[st]
    # the practical selector
    pl = poem.prefill_layer_practical(q, k, v, 1.0, 0.95, 0.5, block=B)
    for ws in (pl.ws_pooled, pl.ws_select, pl.ws_fwd):
        st = poem.poem_check_status(ws)
        assert st == 0, poem.STATUS[st]
    print("checks build ok")


if __name__ == "__main__":
    main()
