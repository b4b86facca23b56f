"""sparse_attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or pass a workspace (a host framework that owns
all device allocations, or a latency-critical loop that cannot afford cudaMalloc's
implicit synchronisation).  For them the library runs the same backward kernels with
their scratch in a fixed device array.  This file checks, through the C ABI, that the
entry point gives the same gradients as sparse_attn_bwd and as the fp64 oracle (within
the parity tolerance) on two calls in a row, and that a problem larger than the fixed
array is refused before anything is enqueued.  It is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

from index_sparse_attention_b200 import _lib
from index_sparse_attention_b200 import inputs as I

from helpers import assert_close, bf16_to_f64, build_lists, to_gpu


def test_noalloc_rejects_problems_above_its_scratch_size():
    from index_sparse_attention_b200.build import build
    build()
    L = _lib.load()
    s = _lib.BlockSparseStruct(_lib.SA_MODE_DENSE, 0, 1, 8, 65536, 65536, 128, 0, 0, None, None,
                               0x1000, 0x1000, 0x1000, 0x1000)
    p = _lib.ParamsStruct(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000,
                          0x1000, 1, 8, 8, 128, 128, 65536, 65536, 0.1, ctypes.pointer(s), None)
    assert L.sparse_attn_bwd_workspace_size(ctypes.byref(p)) > _lib.SA_NOALLOC_SCRATCH_BYTES
    # refused on the host, before any CUDA call (this runs without a GPU)
    assert L.sparse_attn_bwd_noalloc(ctypes.byref(p), None) == _lib.SA_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.error_string(_lib.SA_ERR_SCRATCH_LIMIT)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    """Two calls in a row: the first through the Python wrapper, the second straight
    through the C symbol.  Each is compared with sparse_attn_bwd (the workspace entry
    point) and with the fp64 oracle, at the parity tolerance."""
    import torch
    import index_sparse_attention_b200 as sa
    import oracle
    from helpers import oracle_problem

    w = I.scaled(I.WORKLOADS["gqa_blocksparse_b2_hq32_hk8_s8192_d128"], B=1, Sq=640, Sk=640,
                 HQ=4, HK=2, density=0.5, name="noalloc")
    inp = I.make_inputs(w)
    g = to_gpu(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsp = build_lists(inp, g)
    o, lse = sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale)
    ref = sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale)
    torch.cuda.synchronize()
    ref = [bf16_to_f64(t) for t in ref]
    exact = oracle.backward(oracle_problem(inp), inp.f32("do"))

    L = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        dq, dk, dv = (torch.full_like(g["q"], float("nan")), torch.full_like(g["k"], float("nan")),
                      torch.full_like(g["v"], float("nan")))
        if call == 0:
            sa.sparse_attn_bwd_noalloc(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale,
                                       dq=dq, dk=dk, dv=dv, dev_status=status)
        else:
            p = sa._params(g["q"], g["k"], g["v"], o, lse, bsp, w.scale, g["do"], dq, dk, dv,
                           status)
            rc = L.sparse_attn_bwd_noalloc(ctypes.byref(p), stream)
            assert rc == _lib.SA_OK, _lib.error_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for name, got, r, x in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref, exact):
            assert_close(f"{name} (call {call}) vs sparse_attn_bwd", bf16_to_f64(got), r)
            assert_close(f"{name} (call {call}) vs the oracle", bf16_to_f64(got), x)
