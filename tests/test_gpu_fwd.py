"""GPU forward (O, LSE) vs the fp64 oracle on the same seeded bf16 inputs.

Small cases span several tiles and ragged tails and are compared element by element;
the benchmark workloads at full size are compared on sampled rows.
"""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I

from helpers import (assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem, to_gpu)

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
SMALL = [
    W["blocksparse_mha_s256_d64"],
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=300, Sk=300, HQ=4, HK=2, causal=True,
             name="ragged_bs64_causal_gqa_d64"),
    I.scaled(W["dense_full_b2_h16_s4096_d128"], B=1, Sq=640, Sk=640, HQ=2, HK=2, name="full_d128"),
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=2, Sq=600, Sk=600, HQ=2, HK=2,
             name="ragged_causal_d128"),
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=1024, Sk=1024, HQ=8, HK=2,
             name="gqa_blocksparse_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=1000, Sk=1000, HQ=8, HK=2,
             topk=256, name="index_gqa_d192_128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=200, Sk=200, HQ=2, HK=1,
             topk=400, name="index_topk_gt_seq"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=768, Sk=768, HQ=2, HK=2,
             density=0.3, name="causal_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=333, Sk=333, HQ=1, HK=1,
             density=0.5, name="ragged_d256"),
    # head dims 256/256 run on the 2-CTA backward: GQA, batch > 1, 64-wide blocks,
    # index mode, and a non-causal case with Sq != Sk
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], B=2, Sq=384, Sk=384, HQ=4, HK=2,
             bs=64, density=0.5, name="bs64_gqa_b2_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], mode="index", Sq=520, Sk=520, HQ=4,
             HK=2, topk=150, name="index_gqa_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=200, Sk=450, HQ=2, HK=1,
             causal=False, density=1.0, name="noncausal_sq_ne_sk_d256"),
]
FULL = [W[k] for k in ("dense_full_b2_h16_s4096_d128", "dense_causal_b2_h16_s4096_d128",
                       "gqa_blocksparse_b2_hq32_hk8_s8192_d128",
                       "indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048",
                       "long_causal_blocksparse_h16_s32768_d256")]


def run_fwd(inp):
    import torch
    import index_sparse_attention_b200 as sa
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, inp.w.scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    return bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_forward_small(w):
    inp = I.make_inputs(w, with_grad=False)
    o, lse = run_fwd(inp)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    assert_lse(lse, lse_ref)
    assert_close("O", o, O_ref)


def sample_rows(w, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.HQ, n), rng.integers(0, w.Sq, n)],
                    axis=1)
    rows[0] = (w.B - 1, w.HQ - 1, w.Sq - 1)
    rows[1] = (0, 0, 0)
    rows[2] = (0, 0, 127)
    rows[3] = (w.B - 1, 0, 128)
    return rows.astype(np.int64)


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_forward_full_size_sampled(w):
    inp = I.make_inputs(w, with_grad=False)
    o, lse = run_fwd(inp)
    rows = sample_rows(w)
    o_ref, lse_ref = oracle.forward_rows(oracle_problem(inp), rows)
    got_o = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    got_lse = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_lse(got_lse, lse_ref)
    assert_close("O", got_o, o_ref)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
