"""The forward's two GQA forms, each against the oracle.

With an even GQA group size and Dv >= 128 the forward can run two query heads of one
group on a 2-CTA cluster whose MMAs span both CTAs (tcgen05 cta_group::2, M = 256) and
which split every K and V tile between them; sparse_attn_set_forward_pairs selects it
("on"), forbids it ("off") or leaves the choice to the library ("auto": head dims 256).
Every case runs under both "on" and "off": O and LSE against the fp64 oracle, and the
two forms against each other.  A third test shortens the pipeline wait limit under
"on", so that the pair's abort path (flag exchange, drains, the second cluster meeting)
runs, and checks that the next call is clean.
"""
import time

import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import _lib
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = [
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=2, Sq=520, Sk=520, HQ=4, HK=1,
             name="block_g4_ragged_d128"),
    I.scaled(W["dense_full_b2_h16_s4096_d128"], B=1, Sq=200, Sk=330, HQ=4, HK=2,
             name="full_sq_lt_sk_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=640, Sk=640, HQ=8, HK=1,
             topk=160, name="index_g8_d192_128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=300, Sk=520, HQ=4, HK=2,
             topk=100, span="all", causal=False, dup=0.2, name="index_noncausal_dup_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], B=2, Sq=384, Sk=384, HQ=4, HK=2,
             bs=64, density=0.5, name="bs64_b2_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], mode="index", Sq=450, Sk=450, HQ=4,
             HK=2, topk=120, name="index_ragged_d256"),
]


def _forward(w, g, bsp, policy):
    import torch
    import index_sparse_attention_b200 as sa
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sparse_attn_set_forward_pairs(policy)
    try:
        o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
        torch.cuda.synchronize()
    finally:
        sa.sparse_attn_set_forward_pairs("auto")
    assert int(status.item()) == 0
    return o, lse


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_pair_and_single_forms_match_the_oracle(w):
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    outs = {}
    for policy in ("on", "off"):
        o, lse = _forward(w, g, bsp, policy)
        assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
        assert_close(f"O ({policy})", bf16_to_f64(o), O_ref)
        outs[policy] = (bf16_to_f64(o), lse.cpu().numpy().astype(np.float64))
    assert_close("O on vs off", outs["on"][0], outs["off"][0])
    assert_lse(outs["on"][1], outs["off"][1])


@pytest.mark.parametrize("w", CASES[:3:2], ids=[w.name for w in CASES[:3:2]])
def test_pair_form_timeout_then_recovers(w):
    import torch
    import index_sparse_attention_b200 as sa
    L = _lib.load()
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sparse_attn_set_forward_pairs("on")
    try:
        assert L.sparse_attn_set_wait_limit_ns(300) == _lib.SA_OK
        t0 = time.perf_counter()
        sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        st = int(status.item())
    finally:
        L.sparse_attn_set_wait_limit_ns(0)
        sa.sparse_attn_set_forward_pairs("auto")
    assert st & _lib.STATUS_TIMEOUT, f"forward status {st}"
    assert elapsed < 30.0
    o, lse = _forward(w, g, bsp, "on")
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)
