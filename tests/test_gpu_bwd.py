"""GPU backward (dQ, dK, dV) vs the fp64 oracle on the same seeded bf16 inputs.

Small cases (several tiles, ragged tails, GQA, every head-dim pair, index and block
modes) are compared element by element against the oracle's full backward.  The
benchmark workloads at full size are compared on sampled query rows (dQ) and sampled
keys (dK, dV), with the oracle's LSE and Delta evaluated for every row those samples
depend on.
"""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
SMALL = [
    W["blocksparse_mha_s256_d64"],
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=300, Sk=300, HQ=4, HK=2, causal=True,
             name="ragged_bs64_causal_gqa_d64"),
    I.scaled(W["dense_full_b2_h16_s4096_d128"], B=1, Sq=512, Sk=512, HQ=2, HK=2, name="full_d128"),
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=2, Sq=600, Sk=600, HQ=2, HK=2,
             name="ragged_causal_d128"),
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=768, Sk=768, HQ=8, HK=2,
             name="gqa_blocksparse_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=700, Sk=700, HQ=4, HK=2,
             topk=200, name="index_gqa_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=640, Sk=640, HQ=2, HK=2,
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
FULL = [W[k] for k in ("blocksparse_mha_s256_d64", "dense_full_b2_h16_s4096_d128",
                       "dense_causal_b2_h16_s4096_d128", "gqa_blocksparse_b2_hq32_hk8_s8192_d128",
                       "indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048",
                       "long_causal_blocksparse_h16_s32768_d256")]


def run_fwd_bwd(inp):
    import torch
    import index_sparse_attention_b200 as sa
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, inp.w.scale, dev_status=status)
    dq, dk, dv = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, inp.w.scale,
                                    dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    return [bf16_to_f64(t) for t in (dq, dk, dv)]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_backward_small(w):
    inp = I.make_inputs(w)
    dq, dk, dv = run_fwd_bwd(inp)
    P = oracle_problem(inp)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"))
    assert_close("dV", dv, rV)
    assert_close("dK", dk, rK)
    assert_close("dQ", dq, rQ)


def _rows_attending(w, inp, b, g, keys_j):
    """Query rows i (of batch b, KV head g) whose allowed set may hold one of the keys:
    a superset read off the block mask or the index tensor (the causal cut is left to
    the oracle)."""
    need = np.zeros(w.Sq, bool)
    for j in keys_j:
        if w.mode == "block":
            col = inp.mask[b, g, :, j // w.bs].astype(bool)          # per query block
            need |= np.repeat(col, w.bs)[:w.Sq]
        else:
            need |= (inp.idx[b, :, g, :] == j).any(axis=1)
    return np.nonzero(need)[0]


def _sampled_reference(w, inp, n_rows=24):
    """Oracle dQ at sampled rows and dK/dV at sampled keys of KV head 0 of batch B-1.

    The keys span the sequence: key tile 0 (under causal masking the longest transposed
    list, so the deepest dK/dV accumulation), a mid-sequence tile and the last keys.
    The oracle's LSE and Delta are evaluated at every row that can attend them."""
    P = oracle_problem(inp)
    rng = np.random.default_rng(7)
    G = w.HQ // w.HK
    b, g = w.B - 1, 0
    mid = (w.Sk // 256) * 128  # first key of a mid-sequence tile
    keys_j = np.unique(np.clip(np.array([0, 5, 127, mid + 3, mid + 100, w.Sk - 129, w.Sk - 1]),
                               0, w.Sk - 1)).astype(np.int64)
    keys = np.stack([np.full(len(keys_j), b), np.full(len(keys_j), g), keys_j], 1)
    ii = _rows_attending(w, inp, b, g, keys_j)
    hh, ii = np.meshgrid(np.arange(g * G, (g + 1) * G), ii, indexing="ij")
    rows_k = np.stack([np.full(hh.size, b), hh.ravel(), ii.ravel()], 1)
    rows_q = np.stack([rng.integers(0, w.B, n_rows), rng.integers(0, w.HQ, n_rows),
                       rng.integers(0, w.Sq, n_rows)], 1)
    rows_q[0] = (w.B - 1, w.HQ - 1, w.Sq - 1)
    rows_q[1] = (0, 0, 1)
    rows = np.unique(np.concatenate([rows_k, rows_q]), axis=0).astype(np.int64)
    o_r, lse_r = oracle.forward_rows(P, rows)
    do = inp.f32("do")
    dlt_r = np.einsum("nd,nd->n", do[rows[:, 0], rows[:, 2], rows[:, 1]].astype(np.float64), o_r)
    lse = np.full((w.B, w.HQ, w.Sq), np.nan)
    dlt = np.full((w.B, w.HQ, w.Sq), np.nan)
    lse[rows[:, 0], rows[:, 1], rows[:, 2]] = lse_r
    dlt[rows[:, 0], rows[:, 1], rows[:, 2]] = dlt_r
    dq = oracle.backward_rows(P, do, lse, dlt, rows_q)
    dk, dv = oracle.backward_keys(P, do, lse, dlt, keys)
    return rows_q, dq, keys, dk, dv


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_backward_full_size_sampled(w):
    inp = I.make_inputs(w)
    dq, dk, dv = run_fwd_bwd(inp)
    rows_q, rdq, keys, rdk, rdv = _sampled_reference(w, inp)
    assert np.isfinite(rdq).all() and np.isfinite(rdk).all() and np.isfinite(rdv).all()
    assert_close("dQ", dq[rows_q[:, 0], rows_q[:, 2], rows_q[:, 1]], rdq)
    assert_close("dK", dk[keys[:, 0], keys[:, 2], keys[:, 1]], rdk)
    assert_close("dV", dv[keys[:, 0], keys[:, 2], keys[:, 1]], rdv)
    for t in (dq, dk, dv):
        assert np.isfinite(t).all()
