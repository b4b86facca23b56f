"""The forward's head-to-CTA forms, each against the oracle.

The query heads of one GQA group walk the same tile list, so with an even group size the
forward can run two of them (same query tile) together: on a 2-CTA cluster whose MMAs
span both CTAs (tcgen05 cta_group::2, M = 256) and which split every K and V tile
("cta_pair", Dv >= 128), or in one CTA with both heads' S and O in tensor memory and a
softmax warpgroup per head ("two_heads", Dqk <= 192, Dv <= 128); "one_head" runs one CTA
per (query tile, head).  "two_tiles" (Dqk, Dv <= 128) holds two consecutive query tiles of
one head in one CTA the way "two_heads" holds two heads, and walks the union of the two
tiles' lists, masking out for each tile the key tiles its own list lacks: the MHA cases
below give it an odd number of query tiles (the last CTA has no second tile), random
block masks (many tiles in one list only), 64-blocks with Sq > Sk, and index lists with
duplicates.  sparse_attn_set_forward_form selects the form; a form that does not apply
falls back to one head per CTA.  Every case runs under all four: O and LSE against the
fp64 oracle, and the forms against each other.  Dense mode (no mask) runs the library's
choice, one head per CTA and two query tiles per CTA against the oracle's dense
attention.  A second test shortens the
pipeline wait limit under each two-head form, so that its abort path (drains; for the
pair the flag exchange and the second cluster meeting) runs, and checks that the next
call is clean.
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
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=300, Sk=300, HQ=4, HK=2, causal=True,
             name="bs64_causal_d64"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], B=2, Sq=384, Sk=384, HQ=4, HK=2,
             bs=64, density=0.5, name="bs64_b2_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], mode="index", Sq=450, Sk=450, HQ=4,
             HK=2, topk=120, name="index_ragged_d256"),
    # group of six (head pairs (0,1), (2,3), (4,5) inside the group) and of three (odd:
    # every form falls back to one head per CTA)
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=384, Sk=384, HQ=12, HK=2,
             name="block_g6_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=300, Sk=300, HQ=6, HK=2,
             topk=80, name="index_g3_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=256, Sk=256, HQ=6, HK=1,
             density=0.5, name="block_g6_d256"),
    # MHA (two query tiles per CTA)
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=1, Sq=520, Sk=520, HQ=2, HK=2,
             name="mha_causal_odd_tiles_d128"),
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=900, Sk=900, HQ=2, HK=2,
             name="mha_block_sparse_d128"),
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=600, Sk=333, HQ=2, HK=2, causal=True,
             name="mha_bs64_causal_sq_gt_sk_d64"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=400, Sk=520, HQ=2, HK=2,
             Dqk=128, Dv=128, topk=90, span="all", causal=False, dup=0.2,
             name="mha_index_noncausal_dup_d128"),
]
FORMS = ("one_head", "cta_pair", "two_heads", "two_tiles")


def _forward(w, g, bsp, form):
    import torch
    import index_sparse_attention_b200 as sa
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sparse_attn_set_forward_form(form)
    try:
        o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
        torch.cuda.synchronize()
    finally:
        sa.sparse_attn_set_forward_form("auto")
    assert int(status.item()) == 0
    return o, lse


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_every_form_matches_the_oracle(w):
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    outs = {}
    for form in FORMS:
        o, lse = _forward(w, g, bsp, form)
        assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
        assert_close(f"O ({form})", bf16_to_f64(o), O_ref)
        outs[form] = (bf16_to_f64(o), lse.cpu().numpy().astype(np.float64))
    for form in FORMS[1:]:
        assert_close(f"O {form} vs one_head", outs[form][0], outs["one_head"][0])
        assert_lse(outs[form][1], outs["one_head"][1])


@pytest.mark.parametrize("form", FORMS[1:])
@pytest.mark.parametrize("w", CASES[:3:2], ids=[w.name for w in CASES[:3:2]])
def test_two_unit_forms_timeout_then_recover(w, form):
    import torch
    import index_sparse_attention_b200 as sa
    L = _lib.load()
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sparse_attn_set_forward_form(form)
    try:
        assert L.sparse_attn_set_wait_limit_ns(300) == _lib.SA_OK
        t0 = time.perf_counter()
        sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        st = int(status.item())
    finally:
        L.sparse_attn_set_wait_limit_ns(0)
        sa.sparse_attn_set_forward_form("auto")
    assert st & _lib.STATUS_TIMEOUT, f"forward status {st}"
    assert elapsed < 30.0
    o, lse = _forward(w, g, bsp, form)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)


# dense mode (block_mask_to_block_sparse without a mask): the library's own choice, one
# head per CTA and two query tiles per CTA, against the oracle's dense attention
DENSE = [
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=1, Sq=520, Sk=520, HQ=2, HK=2,
             name="dense_mha_causal_odd_tiles_d128"),
    I.scaled(W["dense_full_b2_h16_s4096_d128"], B=2, Sq=300, Sk=700, HQ=3, HK=1, Dqk=64, Dv=64,
             name="dense_g3_sq_lt_sk_d64"),
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=1, Sq=640, Sk=333, HQ=2, HK=2,
             name="dense_mha_causal_sq_gt_sk_d128"),
]


@pytest.mark.parametrize("w", DENSE, ids=[w.name for w in DENSE])
def test_dense_mode_matches_the_oracle(w):
    import index_sparse_attention_b200 as sa
    inp = I.make_inputs(w, with_grad=False)
    g = to_gpu(inp)
    bsp = sa.block_mask_to_block_sparse(None, w.B, w.HK, w.Sq, w.Sk, causal=w.causal,
                                        device=g["q"].device)
    P = oracle.Problem(inp.f32("q"), inp.f32("k"), inp.f32("v"), scale=w.scale,
                       causal=w.causal, mode="dense")
    O_ref, lse_ref = oracle.forward(P)
    outs = {}
    for form in ("auto", "one_head", "two_tiles"):
        o, lse = _forward(w, g, bsp, form)
        assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
        assert_close(f"O ({form})", bf16_to_f64(o), O_ref)
        outs[form] = (bf16_to_f64(o), lse.cpu().numpy().astype(np.float64))
    assert_close("O two_tiles vs one_head", outs["two_tiles"][0], outs["one_head"][0])
    assert_lse(outs["two_tiles"][1], outs["one_head"][1])
