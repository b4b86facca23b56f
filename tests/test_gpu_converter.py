"""GPU tile-list conversion vs the oracle: bit-exact lists, counts and bitmaps."""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I

from helpers import build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
SMALL = [
    I.scaled(W["blocksparse_mha_s256_d64"]),
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=300, Sk=300, causal=True, name="ragged_bs64"),
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], Sq=1000, Sk=1000, HQ=4, HK=2,
             name="ragged_gqa_bs128"),
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], Sq=520, Sk=520, HQ=2, HK=2, name="dense_causal"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=333, Sk=333, HQ=4, HK=2,
             topk=50, name="ragged_index"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=600, Sk=600, HQ=2, HK=1,
             topk=700, name="index_topk_gt_seq"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=256, Sk=256, HQ=2, HK=2,
             topk=64, causal=False, span="all", dup=0.2, name="index_noncausal"),
]
FULL = [W[k] for k in ("blocksparse_mha_s256_d64", "dense_full_b2_h16_s4096_d128",
                       "dense_causal_b2_h16_s4096_d128", "gqa_blocksparse_b2_hq32_hk8_s8192_d128",
                       "indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048")]
FULL.append(I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=8192, Sk=8192,
                     name="long_causal_s8192"))


def check_lists(w):
    import torch
    inp = I.make_inputs(w, with_grad=False)
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.block_lists(oracle_problem(inp), tile=128)
    for key in ("cnt", "idx", "tcnt", "tidx"):
        got = getattr(bsp, key).cpu().numpy()
        np.testing.assert_array_equal(got, ref[key], err_msg=f"{w.name}: {key}")
    if w.mode == "index":
        got = bsp.bitmap.cpu().numpy().view(np.uint32)
        np.testing.assert_array_equal(got, ref["bitmap"], err_msg=f"{w.name}: bitmap")


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_lists_small(w):
    check_lists(w)


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_lists_full_size(w):
    check_lists(w)


def test_out_of_range_index_sets_status():
    import torch
    import index_sparse_attention_b200 as sa
    idx = torch.full((1, 256, 1, 4), -1, dtype=torch.int32, device="cuda")
    idx[0, 10, 0, 0] = 256  # Sk = 256
    idx[0, 11, 0, 1] = -7
    idx[0, 12, 0, 2] = 5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = sa.index_to_block_sparse(idx, 256, causal=False, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 1
    bm = bsp.bitmap.cpu().numpy().view(np.uint32)
    assert bm[0, 0, 12, 0] == 1 << 5 and bm[0, 0, 10].sum() == 0 and bm[0, 0, 11].sum() == 0
