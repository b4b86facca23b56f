"""Deterministic backward (sparse_attn_bwd_deterministic): dQ, dK and dV are bitwise
identical across calls, within the parity tolerance of the oracle, and close to the
default backward, for the three backward kernels (D=64/128 single CTA, the 192/128
head-dim split, the 256/256 pair)."""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I
from helpers import assert_close, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu
W = I.WORKLOADS

CASES = [
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=2, Sq=640, Sk=640, HQ=4, HK=2,
             density=0.6, name="det_gqa_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=520, Sk=520, HQ=4, HK=2,
             topk=200, name="det_index_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=1024, Sk=1024, HQ=2, HK=2,
             density=0.5, name="det_d256"),
    # the grid interleaves heads (and batches) in this mode: GQA, batch > 1, 64-wide
    # blocks and a ragged length on the pair kernel, index mode on it, and a ragged
    # (64, 64) case on the single-CTA kernel
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], B=2, Sq=450, Sk=450, HQ=4, HK=2,
             bs=64, density=0.5, name="det_bs64_gqa_b2_ragged_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], mode="index", Sq=520, Sk=520, HQ=4,
             HK=2, topk=150, name="det_index_gqa_d256"),
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=300, Sk=300, HQ=4, HK=2, causal=True,
             name="det_ragged_bs64_causal_gqa_d64"),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_bitwise_reproducible_and_correct(w):
    import torch
    import index_sparse_attention_b200 as sa
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    runs = []
    for _ in range(3):
        runs.append(sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                       dev_status=status, deterministic=True))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    dq, dk, dv = runs[0]
    assert_close("dQ", bf16_to_f64(dq), rQ)
    assert_close("dK", bf16_to_f64(dk), rK)
    assert_close("dV", bf16_to_f64(dv), rV)
    # the default backward agrees up to summation order (the deterministic mode walks
    # each key tile's query tiles in ascending order, the default full tiles first)
    dq2, dk2, dv2 = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                       dev_status=status)
    torch.cuda.synchronize()
    for name, x, y in (("dQ", dq2, dq), ("dK", dk2, dk), ("dV", dv2, dv)):
        assert_close(f"{name} (default vs deterministic)", bf16_to_f64(x), bf16_to_f64(y), tol=1e-2)
