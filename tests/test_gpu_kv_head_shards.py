"""Head sharding, the multi-GPU split of this path: a GQA problem cut into KV-head shards.

Each (batch, KV head) group and its query heads form an independent problem (no exchange:
dK and dV sum only over the group's own query heads), so N GPUs can each take whole KV
heads.  These tests run one problem as two shards, each through its own calls on
per-shard tensors (KV heads [0, HK/2) with their query heads, then the rest), reassemble
O, LSE, dQ, dK and dV, and compare them with the fp64 oracle on the unsharded problem,
and with the unsharded GPU call.  Block mode (D=128) and index mode ((192,128) and
(256,256)) are covered.
"""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = [
    I.scaled(W["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=2, Sq=640, Sk=640, HQ=8, HK=4,
             name="gqa_block_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=520, Sk=520, HQ=8, HK=2,
             topk=128, name="gqa_index_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], mode="index", Sq=400, Sk=400, HQ=4,
             HK=2, topk=96, name="gqa_index_d256"),
]


def _run(sa, g, w, lists):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], lists, w.scale, dev_status=status)
    dq, dk, dv = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], lists, w.scale,
                                    dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_two_kv_head_shards_reassemble_the_whole(w):
    import torch
    import index_sparse_attention_b200 as sa
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    G = w.HQ // w.HK
    half = w.HK // 2
    parts = []
    for k0, k1 in ((0, half), (half, w.HK)):
        gs = {
            "q": g["q"][:, :, k0 * G:k1 * G].contiguous(),
            "k": g["k"][:, :, k0:k1].contiguous(),
            "v": g["v"][:, :, k0:k1].contiguous(),
            "do": g["do"][:, :, k0 * G:k1 * G].contiguous(),
        }
        ws = I.scaled(w, HQ=(k1 - k0) * G, HK=k1 - k0)
        if w.mode == "block":
            gs["mask"] = g["mask"][:, k0:k1].contiguous()
            lists = sa.block_mask_to_block_sparse(gs["mask"], ws.B, ws.HK, ws.Sq, ws.Sk,
                                                  bs=ws.bs, causal=ws.causal)
        else:
            gs["idx"] = g["idx"][:, :, k0:k1].contiguous()
            lists = sa.index_to_block_sparse(gs["idx"], ws.Sk, causal=ws.causal)
        parts.append(_run(sa, gs, ws, lists))
    o = torch.cat([p[0] for p in parts], dim=2)
    lse = torch.cat([p[1] for p in parts], dim=1)
    dq = torch.cat([p[2] for p in parts], dim=2)
    dk = torch.cat([p[3] for p in parts], dim=2)
    dv = torch.cat([p[4] for p in parts], dim=2)

    whole = _run(sa, g, w, build_lists(inp, g))
    # the same kernels on the same per-group data: O, LSE, dK and dV are bitwise equal
    # (dK and dV sum in TMEM in a fixed order); dQ is added by several CTAs in an order
    # the hardware picks, so it matches within the parity tolerance
    for name, got, ref in (("O", o, whole[0]), ("LSE", lse, whole[1]), ("dK", dk, whole[3]),
                           ("dV", dv, whole[4])):
        assert torch.equal(got, ref), f"{name}: shards differ from the whole"
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)
    assert_close("dQ", bf16_to_f64(dq), rQ)
    assert_close("dK", bf16_to_f64(dk), rK)
    assert_close("dV", bf16_to_f64(dv), rV)
    assert_close("dQ vs whole", bf16_to_f64(dq), bf16_to_f64(whole[2]))
