"""Parity of the CUDA top-k selector (topk_select) with the numpy oracle: indices
bit-exact, values bit-exact (up to -0 / +0 and NaN payloads), on normal and concentrated
score distributions, packed causal ranges, rows with fewer valid columns than k, empty
and offset ranges, k = 1 and k = SA_TOPK_MAX_K, long rows, and special values.  Also the
device status of an invalid range, and top-k feeding index-sparse attention."""
import numpy as np
import pytest

import oracle
from oracle import topk as T
from index_sparse_attention_b200 import inputs as I

pytestmark = pytest.mark.gpu


def run(scores, k, starts=None, ends=None, ld_pad=0):
    import torch
    import index_sparse_attention_b200 as sa
    R, C = scores.shape
    host = np.zeros((R, C + ld_pad), np.float32)
    host[:, :C] = scores
    dev = torch.from_numpy(host).cuda()[:, :C]
    st = None if starts is None else torch.from_numpy(np.ascontiguousarray(starts, np.int32)).cuda()
    en = None if ends is None else torch.from_numpy(np.ascontiguousarray(ends, np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, val = sa.topk_select(dev, k, st, en, with_values=True, dev_status=status)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy(), int(status.item())


def check(scores, k, starts=None, ends=None, ld_pad=0, rows=None):
    idx, val, status = run(scores, k, starts, ends, ld_pad)
    assert status == 0
    ridx, rval = T.topk_select(scores, k, starts, ends, rows=rows)
    got_idx = idx if rows is None else idx[rows]
    got_val = val if rows is None else val[rows]
    bad = np.argwhere(got_idx != ridx)
    assert bad.size == 0, f"index mismatch at {bad[:5].tolist()}"
    assert np.array_equal(got_val, rval, equal_nan=True)


@pytest.mark.parametrize("dist", ["normal", "concentrated"])
@pytest.mark.parametrize("k", [1, 64, 256])
def test_packed_causal(dist, k):
    L = 1500
    x = I.topk_scores(L, L, seed=11 + k, dist=dist)
    s, e = I.packed_causal_ranges(L, segments=(700, 800))
    check(x, k, s, e)


def test_whole_rows_and_padded_leading_dimension():
    x = I.topk_scores(64, 3000, seed=5)
    check(x, 100, ld_pad=12)


def test_k_max_and_short_rows():
    from index_sparse_attention_b200 import _lib
    k = _lib.SA_TOPK_MAX_K
    x = I.topk_scores(8, 6000, seed=6, dist="concentrated")
    starts = np.array([0, 0, 100, 3000, 5999, 6000, 17, 0], np.int32)
    ends = np.array([6000, 4096, 4000, 6000, 6000, 6000, 4200, 1], np.int32)
    check(x, k, starts, ends)


def test_long_rows():
    L = 131072
    x = I.topk_scores(4, L, seed=9)
    starts = np.array([0, 1, 65536, 0], np.int32)
    ends = np.array([L, L, L, 70001], np.int32)
    check(x, 2048, starts, ends)


def test_special_values_and_ties():
    rng = np.random.default_rng(3)
    levels = np.array([-1.0, -0.0, 0.0, 0.5, 2.0, np.inf, -np.inf, np.nan], np.float32)
    x = levels[rng.integers(0, len(levels), (50, 1000))]
    starts = rng.integers(0, 1000, 50).astype(np.int32)
    ends = np.minimum(1000, starts + rng.integers(0, 1000, 50)).astype(np.int32)
    check(x, 37, starts, ends)


def test_invalid_range_sets_status_and_pads():
    x = I.topk_scores(3, 100, seed=1)
    starts = np.array([0, 60, 0], np.int32)
    ends = np.array([100, 50, 101], np.int32)
    idx, _, status = run(x, 5, starts, ends)
    assert status & 1
    assert (idx[1] == -1).all() and (idx[2] == -1).all()
    ridx, _ = T.topk_select(x, 5, rows=[0])
    assert idx[0].tolist() == ridx[0].tolist()


def test_feeds_index_sparse_attention():
    """Scores -> top-k -> tile lists -> forward equals the oracle on the same indices."""
    import torch
    import index_sparse_attention_b200 as sa
    from helpers import assert_close, assert_lse, bf16_to_f64
    w = I.scaled(I.WORKLOADS["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=384, Sk=384,
                 HQ=4, HK=2, topk=48, name="topk_fed")
    inp = I.make_inputs(w)
    s, e = I.packed_causal_ranges(w.Sq)
    scores = I.topk_scores(w.Sq * w.HK, w.Sk, seed=77)
    st, en = np.repeat(s, w.HK), np.repeat(e, w.HK)  # rows ordered (query, KV head)
    idx_host, _ = T.topk_select(scores, w.topk, st, en)
    idx_dev = sa.topk_select(torch.from_numpy(scores).cuda(), w.topk,
                             torch.from_numpy(st).cuda(), torch.from_numpy(en).cuda())
    assert np.array_equal(idx_dev.cpu().numpy(), idx_host)
    idx4 = idx_dev.view(1, w.Sq, w.HK, w.topk).contiguous()
    bsp = sa.index_to_block_sparse(idx4, w.Sk, causal=True)

    def bf(a):
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()

    o, lse = sa.sparse_attn_fwd(bf(inp.q), bf(inp.k), bf(inp.v), bsp, w.scale)
    torch.cuda.synchronize()
    P = oracle.Problem(inp.f32("q"), inp.f32("k"), inp.f32("v"), scale=w.scale, causal=True,
                       mode="index", idx=idx_host.reshape(1, w.Sq, w.HK, w.topk))
    O_ref, lse_ref = oracle.forward(P)
    assert_close("O", bf16_to_f64(o), O_ref)
    assert_lse(lse.cpu().numpy(), lse_ref)
