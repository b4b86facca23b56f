"""Output canaries: every output the kernels write (O, LSE, dQ, dK, dV) is placed inside a
larger buffer whose guard regions before and after it hold a NaN bit pattern.  After the
forward and the backward the guards must be bit-identical, so a TMA store, a bulk
reduce or a plain store whose box spills past Sq or Sk (or before the tensor) is caught
even when it lands outside the elements the parity checks read.  The outputs are also
compared with the oracle.  Batch 1, ragged Sq / Sk, every head-dim pair and both modes.
"""
import numpy as np
import pytest

import oracle
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, assert_lse, bf16_to_f64, build_lists, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = [
    I.scaled(W["blocksparse_mha_s256_d64"], Sq=300, Sk=300, HQ=4, HK=2, causal=True,
             name="ragged_bs64_d64"),
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=1, Sq=600, Sk=600, HQ=2, HK=2,
             name="ragged_causal_d128"),
    I.scaled(W["dense_full_b2_h16_s4096_d128"], B=1, Sq=200, Sk=330, HQ=2, HK=1,
             name="full_sq_lt_sk_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=700, Sk=700, HQ=4, HK=2,
             topk=200, name="index_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=333, Sk=333, HQ=2, HK=1,
             density=0.5, name="ragged_d256"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], mode="index", Sq=390, Sk=390, HQ=2,
             HK=1, topk=100, span="all", causal=False, name="index_noncausal_d256"),
]
FRONT = 4096  # guard elements before each output (16-byte aligned start)
BF16_NAN = np.int16(0x7FC1)
F32_NAN = np.int32(0x7FC00001)


def guarded(shape, dtype, back):
    """(buffer, view): `view` has `shape` and lies in `buffer` after FRONT guard elements
    and before `back` more; the guards hold a NaN pattern."""
    import torch
    n = int(np.prod(shape))
    buf = torch.empty(FRONT + n + back, dtype=dtype, device="cuda")
    if dtype == torch.bfloat16:
        buf.view(torch.int16).fill_(int(BF16_NAN))
    else:
        buf.view(torch.int32).fill_(int(F32_NAN))
    return buf, buf[FRONT:FRONT + n].view(shape)


def assert_guards(name, buf, n):
    import torch
    iv = buf.view(torch.int16 if buf.dtype == torch.bfloat16 else torch.int32).cpu().numpy()
    pat = BF16_NAN if buf.dtype == torch.bfloat16 else F32_NAN
    front, back = iv[:FRONT], iv[FRONT + n:]
    assert (front == pat).all(), f"{name}: {int((front != pat).sum())} guard words before it changed"
    assert (back == pat).all(), f"{name}: {int((back != pat).sum())} guard words after it changed"


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_outputs_stay_inside_their_tensors(w):
    import torch
    import index_sparse_attention_b200 as sa
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g, dev_status=status)
    # two whole 128-row tiles of guard after every row-major output
    bq, o = guarded((1, w.Sq, w.HQ, w.Dv), torch.bfloat16, 256 * w.HQ * w.Dv)
    bl, lse = guarded((1, w.HQ, w.Sq), torch.float32, 4096)
    bdq, dq = guarded((1, w.Sq, w.HQ, w.Dqk), torch.bfloat16, 256 * w.HQ * w.Dqk)
    bdk, dk = guarded((1, w.Sk, w.HK, w.Dqk), torch.bfloat16, 256 * w.HK * w.Dqk)
    bdv, dv = guarded((1, w.Sk, w.HK, w.Dv), torch.bfloat16, 256 * w.HK * w.Dv)
    sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, o=o, lse=lse, dev_status=status)
    sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale, dq=dq, dk=dk,
                       dv=dv, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for name, buf, t in (("O", bq, o), ("LSE", bl, lse), ("dQ", bdq, dq), ("dK", bdk, dk),
                         ("dV", bdv, dv)):
        assert_guards(name, buf, t.numel())
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)
    assert_close("dQ", bf16_to_f64(dq), rQ)
    assert_close("dK", bf16_to_f64(dk), rK)
    assert_close("dV", bf16_to_f64(dv), rV)
