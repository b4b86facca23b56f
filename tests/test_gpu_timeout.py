"""Bounded pipeline waits: a wait that runs out reports itself and the kernel still ends.

Every mbarrier wait of the attention kernels gives up after a limit (2 s by default),
sets the timeout flag (value 2) in the device status word, and its CTA drains the copies and tensor-core
operations it has in flight before it releases its resources and leaves.  These tests
set a limit below 1 us through the C ABI (sparse_attn_set_wait_limit_ns), which makes a
wait give up at its first test when its phase has not completed, so that ordinary
waits (a TMA load just issued, the first MMA) run out.  For each kernel family
(forward, backward at D=128 and at (192,128), the 2-CTA backward at (256,256), and the
deterministic backward) they check that the call returns, that the status word carries the timeout bit, and that the next call at
the default limit matches the oracle: the CUDA context is still usable.  No GPU fault,
trap or endless wait is involved: the waits end by themselves.
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
    I.scaled(W["dense_causal_b2_h16_s4096_d128"], B=1, Sq=512, Sk=512, HQ=2, HK=2,
             name="causal_d128"),
    I.scaled(W["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], Sq=400, Sk=400, HQ=4, HK=2,
             topk=96, name="index_d192_128"),
    I.scaled(W["long_causal_blocksparse_h16_s32768_d256"], Sq=512, Sk=512, HQ=2, HK=2,
             density=0.5, name="causal_d256_pair"),
]
SHORT_NS = 300


def _problem(w):
    import torch
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    bsp = build_lists(inp, g)
    torch.cuda.synchronize()
    return inp, g, bsp


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
@pytest.mark.parametrize("deterministic", [False, True], ids=["default", "deterministic"])
def test_short_wait_limit_reports_timeout_then_recovers(w, deterministic):
    import torch
    import index_sparse_attention_b200 as sa
    L = _lib.load()
    inp, g, bsp = _problem(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        assert L.sparse_attn_set_wait_limit_ns(SHORT_NS) == _lib.SA_OK
        t0 = time.perf_counter()
        o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
        torch.cuda.synchronize()
        fwd_status = int(status.item())
        status.zero_()
        sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                           dev_status=status, deterministic=deterministic)
        torch.cuda.synchronize()
        bwd_status = int(status.item())
        elapsed = time.perf_counter() - t0
    finally:
        L.sparse_attn_set_wait_limit_ns(0)
    assert fwd_status & _lib.STATUS_TIMEOUT, f"forward status {fwd_status}"
    assert bwd_status & _lib.STATUS_TIMEOUT, f"backward status {bwd_status}"
    assert elapsed < 30.0  # the drains are bounded too

    # default limit again: a clean run that matches the oracle
    status.zero_()
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, dev_status=status)
    dq, dk, dv = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                    dev_status=status, deterministic=deterministic)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    P = oracle_problem(inp)
    O_ref, lse_ref = oracle.forward(P)
    rQ, rK, rV = oracle.backward(P, inp.f32("do"), O_ref, lse_ref)
    assert_lse(lse.cpu().numpy().astype(np.float64), lse_ref)
    assert_close("O", bf16_to_f64(o), O_ref)
    assert_close("dQ", bf16_to_f64(dq), rQ)
    assert_close("dK", bf16_to_f64(dk), rK)
    assert_close("dV", bf16_to_f64(dv), rV)
