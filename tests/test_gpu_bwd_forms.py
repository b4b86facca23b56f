"""The (192,128) backward's two key-tile forms, each against the oracle.

At head dims (192,128) the fp32 dK and dV of the whole head dim take 320 of a CTA's 512
TMEM columns.  "split" runs two CTAs per 128-key tile, each owning part of the head dim
of dK, dV and dQ and each recomputing S^T and dP^T in double-buffered tiles; "whole" runs
one CTA per key tile with single S^T / dP^T buffers, its dQ^T in two 128-row windows
(head dims 0-127 and 64-191), the second drained by elementwise warps.
sparse_attn_set_backward_form selects the form ("auto" picks by grid size, so the small
cases here would all take "split").  Every case runs under both: dQ, dK and dV against
the fp64 oracle (O and LSE from the library's forward) and the forms against each
other.  A second test shortens the pipeline wait limit under "whole", so that its abort
path (the helper warps' paired exits included) runs, and checks that the next call is
clean.
"""
import time

import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import _lib
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
IDX = W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"]
CASES = [
    I.scaled(IDX, Sq=520, Sk=520, HQ=8, HK=1, topk=128, name="index_g8_causal_ragged"),
    I.scaled(IDX, Sq=300, Sk=700, HQ=4, HK=2, topk=150, span="all", causal=False, dup=0.3,
             name="index_g2_noncausal_dup_sq_lt_sk"),
    I.scaled(IDX, Sq=600, Sk=333, HQ=4, HK=4, topk=64, span="all", causal=True,
             name="index_mha_above_diag_sq_gt_sk"),
    I.scaled(IDX, B=2, Sq=300, Sk=300, HQ=8, HK=2, topk=100, name="index_b2_g4"),
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=384, Sk=384, HQ=4, HK=2,
             Dqk=192, Dv=128, bs=64, density=0.5, name="block_bs64_g2_causal"),
]
FORMS = ("split", "whole")


def _run(w, g, bsp, form, status=None):
    import torch
    import index_sparse_attention_b200 as sa
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    sa.sparse_attn_set_backward_form(form)
    try:
        dq, dk, dv = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                        dev_status=status)
        torch.cuda.synchronize()
    finally:
        sa.sparse_attn_set_backward_form("auto")
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_both_backward_forms_match_the_oracle(w):
    import torch
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    outs = {}
    for form in FORMS:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        _, _, dq, dk, dv = _run(w, g, bsp, form, status)
        assert int(status.item()) == 0
        got = [bf16_to_f64(t) for t in (dq, dk, dv)]
        for name, x, ref in zip(("dQ", "dK", "dV"), got, (rQ, rK, rV)):
            assert_close(f"{name} ({form})", x, ref)
        outs[form] = got
    for name, a, b in zip(("dQ", "dK", "dV"), outs["whole"], outs["split"]):
        assert_close(f"{name} whole vs split", a, b)


def test_whole_form_timeout_then_recover():
    import torch
    import index_sparse_attention_b200 as sa
    L = _lib.load()
    w = CASES[0]
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sparse_attn_set_backward_form("whole")
    try:
        assert L.sparse_attn_set_wait_limit_ns(300) == _lib.SA_OK
        t0 = time.perf_counter()
        sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                           dev_status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        st = int(status.item())
    finally:
        L.sparse_attn_set_wait_limit_ns(0)
        sa.sparse_attn_set_backward_form("auto")
    assert st & _lib.STATUS_TIMEOUT, f"backward status {st}"
    assert elapsed < 30.0
    status.zero_()
    _, _, dq, dk, dv = _run(w, g, bsp, "whole", status)
    assert int(status.item()) == 0
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    for name, x, ref in zip(("dQ", "dK", "dV"), (dq, dk, dv), (rQ, rK, rV)):
        assert_close(name, bf16_to_f64(x), ref)
