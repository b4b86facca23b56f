"""Degenerate case of the method: query rows with no allowed key.  Such a row gets O = 0,
LSE = -inf and zero gradients, and contributes nothing to dK / dV.  Built by emptying
index rows (all -1) and whole query-block rows of a block mask, for the three backward
kernels' head dims; forward and backward against the oracle."""
import dataclasses

import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I
from helpers import assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu
W = I.WORKLOADS

CASES = [
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=400, Sk=400, HQ=4, HK=2,
             topk=64, name="empty_index_d192_128"),
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=512, Sk=512, HQ=4, HK=2,
             causal=False, density=0.5, name="empty_block_d128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=384, Sk=384, HQ=2, HK=1,
             causal=False, density=0.5, name="empty_block_d256"),
]


def with_empty_rows(inp):
    """Empty some query rows: index rows 0..9 and 200..263 of KV head 0 set to -1; in block
    mode the mask rows of query blocks 1 and the last one of KV head 0 set to 0."""
    if inp.idx is not None:
        idx = inp.idx.copy()
        idx[:, 0:10, 0, :] = -1
        idx[:, 200:264, 0, :] = -1
        return dataclasses.replace(inp, idx=idx)
    mask = inp.mask.copy()
    mask[:, 0, 1, :] = 0
    mask[:, 0, -1, :] = 0
    return dataclasses.replace(inp, mask=mask)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_empty_rows(w):
    import torch
    import index_sparse_attention_b200 as sa
    inp = with_empty_rows(I.make_inputs(w))
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    dq, dk, dv = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                    dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    lse_got = lse.cpu().numpy()
    empty = ~np.isfinite(lse_ref)
    assert empty.any(), "the case has no empty row"
    assert np.all(lse_got[empty] == -np.inf)
    O_got, dq_got = bf16_to_f64(o), bf16_to_f64(dq)
    G = w.HQ // w.HK
    for b, h, i in zip(*np.nonzero(empty)):
        assert np.all(O_got[b, i, h] == 0) and np.all(dq_got[b, i, h] == 0)
    assert_close("O", O_got, O_ref)
    assert_lse(lse_got, lse_ref)
    assert_close("dQ", dq_got, rQ)
    assert_close("dK", bf16_to_f64(dk), rK)
    assert_close("dV", bf16_to_f64(dv), rV)
