"""GPU parity of bsa_fwd_grouped (two query heads of a KV group sharing K/V tiles
over the union of their lists).  Each head runs the same MMAs and softmax as
bsa_fwd on its own list, so the outputs and lse must be bit-identical to bsa_fwd's;
one case also goes straight to the fp64 oracle.  Cases: POEM lists, random masks,
an odd group size, d = 64 / B = 64, one head, a query offset, lists with bad ids,
empty rows, and the full 128K layer."""
import numpy as np
import pytest
import torch

import oracle
import poem_synth
from _parity import FWD_MAX_ABS, FWD_MEAN_ABS, compare_fwd, problem_from, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def poem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_poem_b200 import build

    build.build()
    oracle.build()
    import block_sparse_attention_poem_b200 as m

    return m


def _both(poem, q, k, v, rp, ci, B):
    """bsa_fwd and bsa_fwd_grouped on the same lists: (o, lse, status) of each."""
    out = []
    for grouped in (False, True):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((q.shape[1], q.shape[0]), float("nan"), device="cuda")
        ws = poem.alloc_workspace(256)
        if grouped:
            poem.bsa_fwd_grouped(q, k, v, rp, ci, o, ws, lse=lse, block=B)
        else:
            poem.bsa_fwd(q, k, v, rp, ci, o, ws, lse=lse, block=B)
        out.append((o, lse, poem.poem_check_status(ws)))
    return out


def _assert_identical(a, b):
    (oa, la, sa), (ob, lb, sb) = a, b
    assert sa == sb
    assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
    assert torch.equal(la.view(torch.int32), lb.view(torch.int32))


def _dev_lists(rp, ci):
    rpd = torch.from_numpy(np.ascontiguousarray(rp, dtype=np.int32)).cuda()
    cid = torch.from_numpy(np.ascontiguousarray(ci, dtype=np.int32)).cuda()
    if cid.numel() == 0:
        cid = torch.zeros(4, dtype=torch.int32, device="cuda")
    return rpd, cid


CASES = [
    # (n_tokens, Hq, Hkv, d, block, density, seed)
    (2048, 8, 2, 128, 128, 0.5, 0),
    (1024, 10, 2, 128, 128, 0.4, 1),   # 5-way GQA: the last pair of each group has one head
    (1024, 1, 1, 64, 64, 0.5, 2),      # one head per group
    (1024, 4, 1, 128, 64, 0.3, 3),
    (768, 4, 2, 64, 128, 1.0, 4),
]


@pytest.mark.parametrize("n,hq,hkv,d,B,dens,seed", CASES)
def test_grouped_equals_bsa_fwd_random_lists(poem, n, hq, hkv, d, B, dens, seed):
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=seed)
    q, k, v = to_dev(x)
    rp, ci = poem_synth.random_block_lists(hq, n // B, dens, seed=seed)
    a, b = _both(poem, q, k, v, *_dev_lists(rp, ci), B)
    assert a[2] == 0
    _assert_identical(a, b)


def test_grouped_equals_bsa_fwd_on_poem_lists_and_matches_oracle(poem):
    n, hq, hkv, d, B, tau = 2048, 4, 1, 128, 128, 0.05
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=11)
    q, k, v = to_dev(x)
    layer = poem.prefill_layer(q, k, v, tau, block=B)
    poem.poem_check(layer.ws_fwd)
    a, b = _both(poem, q, k, v, layer.row_ptr, layer.col_idx, B)
    _assert_identical(a, b)
    T = n // B
    prob = problem_from(x, B)
    units = [(h, i) for h in range(hq) for i in range(T)]
    O_ref, _ = prob.masked_units(units, layer.row_ptr.cpu().numpy(), layer.col_idx.cpu().numpy())
    mx, mean = compare_fwd(b[0], O_ref, units, B)
    assert mx <= FWD_MAX_ABS and mean <= FWD_MEAN_ABS


def test_grouped_with_query_offset(poem):
    """Chunked prefill: the last half of the tokens as queries."""
    n, hq, hkv, d, B = 2048, 8, 2, 128, 128
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=21)
    q, k, v = to_dev(x)
    qc = q[n // 2:].contiguous()
    T, t0 = (n // 2) // B, (n // 2) // B
    rng = np.random.default_rng(3)
    rows = []
    for h in range(hq):
        for i in range(T):
            g = t0 + i
            rows.append(sorted(set([0, g]) | set(rng.choice(g + 1, size=(g + 1) // 3, replace=False).tolist())))
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])])
    ci = np.array([b for r in rows for b in r])
    a, b = _both(poem, qc, k, v, *_dev_lists(rp, ci), B)
    assert a[2] == 0
    _assert_identical(a, b)


def test_grouped_bad_ids_and_empty_rows(poem):
    """Ids outside 0..tile are skipped and reported, as bsa_fwd does; empty rows give
    zeros and lse = -inf; a head whose partner's list is empty still runs."""
    n, hq, hkv, d, B = 1024, 4, 1, 128, 128
    T = n // B
    x = poem_synth.iid_layer(n, hq, hkv, d, seed=22)
    q, k, v = to_dev(x)
    rows = []
    for h in range(hq):
        for i in range(T):
            if h == 1 or (h == 2 and i % 2):
                rows.append([])                      # head 1 empty: head 0 runs alone
            elif h == 3 and i == 5:
                rows.append([0, 2, i + 3, i])        # an id beyond the tile (and out of order after it)
            else:
                rows.append(list(range(0, i + 1, 2)) + ([i] if i % 2 else []))
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])])
    ci = np.array([b for r in rows for b in r])
    a, b = _both(poem, q, k, v, *_dev_lists(rp, ci), B)
    assert a[2] == b[2] == 7  # POEM_ERR_BAD_LIST
    _assert_identical(a, b)
    o = b[0].float()
    assert torch.all(o[:, 1] == 0)
    assert torch.all(torch.isinf(b[1][1])) and torch.all(b[1][1] < 0)


def test_grouped_full_size_llama_128k(poem):
    """The benchmark layer (131072 tokens, 32/8 heads, tau = 0.05 lists)."""
    n, hq, hkv, d, B = 131072, 32, 8, 128, 128
    x = poem_synth.heavy_block_layer(n, hq, hkv, d, block=B, seed=0)
    q, k, v = to_dev(x)
    layer = poem.prefill_layer(q, k, v, 0.05, block=B)
    poem.poem_check(layer.ws_fwd)
    o = torch.full_like(q, float("nan"))
    ws = poem.alloc_workspace(256)
    poem.bsa_fwd_grouped(q, k, v, layer.row_ptr, layer.col_idx, o, ws, block=B)
    poem.poem_check(ws)
    assert torch.equal(o.view(torch.int16), layer.o.view(torch.int16))
