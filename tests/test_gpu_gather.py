"""Token-gather forward (sparse_attn_fwd_gather) against the oracle and the block path.

The gather path enumerates each query's keys from the presence bitmap and gathers their
K/V rows, so it must give the oracle's O and LSE on every index-mode case: causal and not,
entries above the diagonal, repeated entries (set semantics), Sq != Sk, rows with no key,
group sizes 1 to 8 and the three supported head-dim pairs.  Unsupported shapes are
refused before any work.
"""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import _lib
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
IDX = W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"]
CASES = [
    I.scaled(IDX, Sq=520, Sk=520, HQ=8, HK=1, topk=128, name="g8_causal_d192_128"),
    I.scaled(IDX, Sq=300, Sk=700, HQ=8, HK=2, topk=150, span="all", causal=False, dup=0.3,
             name="g4_noncausal_dup_sq_lt_sk_d192_128"),
    I.scaled(IDX, Sq=600, Sk=333, HQ=4, HK=4, topk=64, span="all", causal=True,
             name="g1_above_diag_sq_gt_sk_d192_128"),
    I.scaled(IDX, Sq=450, Sk=450, HQ=6, HK=2, Dqk=128, Dv=128, topk=100, name="g3_d128"),
    I.scaled(IDX, Sq=257, Sk=257, HQ=4, HK=2, Dqk=64, Dv=64, topk=40, name="g2_d64"),
    I.scaled(IDX, B=2, Sq=200, Sk=200, HQ=8, HK=1, topk=300, name="b2_topk_gt_seq_d192_128"),
]


def _run(w, inp, empty_rows=()):
    import torch
    import index_sparse_attention_b200 as sa
    if empty_rows:
        inp.idx[:, list(empty_rows)] = -1
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    o, lse = sa.sparse_attn_fwd_gather(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    ob, lseb = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse, ob, lseb


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_gather_forward_matches_the_oracle(w):
    inp = I.make_inputs(w, with_grad=False)
    o, lse, ob, lseb = _run(w, inp)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)
    assert_close("O vs block path", bf16_to_f64(o), bf16_to_f64(ob))
    assert_lse(lse.cpu().numpy().astype(np.float64), lseb.cpu().numpy().astype(np.float64))


def test_gather_forward_rows_without_keys():
    w = I.scaled(IDX, Sq=300, Sk=300, HQ=8, HK=1, topk=64, name="empty_rows")
    inp = I.make_inputs(w, with_grad=False)
    rows = (0, 17, 128, 299)
    o, lse, _, _ = _run(w, inp, empty_rows=rows)
    lse_h = lse.cpu().numpy()
    o_h = bf16_to_f64(o)
    for r in rows:
        assert np.all(np.isneginf(lse_h[:, :, r]))
        assert np.all(o_h[:, r] == 0.0)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    assert_lse(lse_h.astype(np.float64), lse_ref)
    assert_close("O", o_h, O_ref)


def test_gather_forward_refuses_unsupported_shapes():
    import torch
    import index_sparse_attention_b200 as sa
    w = I.scaled(IDX, Sq=128, Sk=128, HQ=16, HK=1, topk=32, name="g16")
    inp = I.make_inputs(w, with_grad=False)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    with pytest.raises(_lib.SparseAttnError) as e:  # a group of 16 heads
        sa.sparse_attn_fwd_gather(g["q"], g["k"], g["v"], bsp, w.scale)
    assert e.value.code == _lib.SA_ERR_UNSUPPORTED
    wb = I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=256, Sk=256, HQ=4, HK=2,
                  name="block")
    inb = I.make_inputs(wb, with_grad=False)
    gb = to_gpu(inb)
    bspb = build_lists(inb, gb)
    with pytest.raises(_lib.SparseAttnError) as e:  # block mode has no bitmap
        sa.sparse_attn_fwd_gather(gb["q"], gb["k"], gb["v"], bspb, wb.scale)
    assert e.value.code == _lib.SA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
