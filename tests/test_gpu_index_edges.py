"""Index-mode edge cases on the GPU against the fp64 oracle: index entries ABOVE the
diagonal (drawn from every key, span "all"), which a causal call must mask and a
non-causal call must attend (key tiles above the diagonal then appear in the lists),
rows with repeated indices (set semantics: the presence matrix of MagiAttention
PR #334, section 2), Sq != Sk both ways, and a pattern whose rows hold every key (FULL
tiles in index mode).  Every head-dim pair runs: (64,64), (128,128), (192,128) and
(256,256), each over several tiles with a ragged tail.  The converter is compared bit
for bit, O / LSE and dQ / dK / dV element by element.
"""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I

from helpers import (assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem,
                     to_gpu)

pytestmark = pytest.mark.gpu

BASE = I.WORKLOADS["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"]


def case(name, Dqk, Dv, causal, Sq=450, Sk=450, HQ=4, HK=2, topk=120, dup=0.25, B=1):
    return I.scaled(BASE, name=name, B=B, Sq=Sq, Sk=Sk, HQ=HQ, HK=HK, Dqk=Dqk, Dv=Dv,
                    causal=causal, topk=topk, span="all", dup=dup)


CASES = [
    case("above_diag_causal_d128", 128, 128, True),
    case("above_diag_noncausal_d128", 128, 128, False),
    case("above_diag_causal_d192_128", 192, 128, True),
    case("above_diag_noncausal_sq_lt_sk_d192_128", 192, 128, False, Sq=300, Sk=520),
    case("above_diag_causal_sq_gt_sk_d192_128", 192, 128, True, Sq=520, Sk=300),
    case("above_diag_causal_d256", 256, 256, True, Sq=400, Sk=400, topk=100),
    case("above_diag_noncausal_d256", 256, 256, False, Sq=400, Sk=400, topk=100),
    case("above_diag_noncausal_d64_b2", 64, 64, False, B=2, Sq=330, Sk=330, topk=64),
    # every row holds every key: FULL tiles in index mode (the last key tile crosses Sk)
    case("all_keys_full_tiles_d128", 128, 128, False, Sq=384, Sk=300, topk=512, dup=0.0),
]
IDS = [w.name for w in CASES]


def _run(w, backward):
    import torch
    import index_sparse_attention_b200 as sa
    inp = I.make_inputs(w, with_grad=backward)
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    grads = None
    if backward:
        grads = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                   dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    return inp, bsp, o, lse, grads


def test_generator_reaches_the_edges():
    """Each case really holds what it is named for (checked on the inputs, no GPU work)."""
    for w in CASES:
        idx = I.topk_indices(w)
        i = np.arange(w.Sq)[None, :, None, None]
        assert (idx > i).any(), w.name  # entries above the diagonal
        if w.dup > 0:
            r = idx[0, w.Sq // 2, 0]
            assert len(set(r[r >= 0].tolist())) < int((r >= 0).sum()), w.name


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_lists_bit_exact(w):
    inp, bsp, *_ = _run(w, backward=False)
    ref = oracle.block_lists(oracle_problem(inp), tile=128)
    for key in ("cnt", "idx", "tcnt", "tidx"):
        np.testing.assert_array_equal(getattr(bsp, key).cpu().numpy(), ref[key],
                                      err_msg=f"{w.name}: {key}")
    np.testing.assert_array_equal(bsp.bitmap.cpu().numpy().view(np.uint32), ref["bitmap"],
                                  err_msg=f"{w.name}: bitmap")
    if not w.causal:  # key tiles above the diagonal are listed
        tm, tn = np.nonzero(ref["idx"][0, 0] >= 0)
        assert (ref["idx"][0, 0][tm, tn] > tm).any()


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_forward(w):
    inp, _, o, lse, _ = _run(w, backward=False)
    O_ref, lse_ref = oracle.forward(oracle_problem(inp))
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_backward(w):
    inp, _, _, _, (dq, dk, dv) = _run(w, backward=True)
    rQ, rK, rV = oracle.backward(oracle_problem(inp), inp.f32("do"))
    assert_close("dV", bf16_to_f64(dv), rV)
    assert_close("dK", bf16_to_f64(dk), rK)
    assert_close("dQ", bf16_to_f64(dq), rQ)
