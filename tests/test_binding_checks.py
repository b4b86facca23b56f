"""Argument checks of the Python binding, which run before any device work: the C ABI
sees pointers and sizes only, so a tensor of the wrong shape, type or device would be
read or written out of bounds.  CPU tensors stand in where a check must fire first."""
import pytest
import torch

import index_sparse_attention_b200 as sa
from index_sparse_attention_b200 import _lib
from index_sparse_attention_b200.build import build


@pytest.fixture(scope="module", autouse=True)
def lib():
    build()
    return _lib.load()


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_cpu_tensors_are_rejected():
    q, k, v = bf16(1, 128, 2, 64), bf16(1, 128, 2, 64), bf16(1, 128, 2, 64)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        sa.sparse_attn_bwd_workspace_size(q, k, v, None)
    with pytest.raises(ValueError, match="idx must be a CUDA tensor"):
        sa.index_to_block_sparse(torch.zeros((1, 128, 2, 4), dtype=torch.int32), 128)
    with pytest.raises(ValueError, match="mask must be a CUDA tensor"):
        sa.block_mask_to_block_sparse(torch.zeros((1, 2, 1, 1), dtype=torch.uint8), 1, 2, 128, 128)
    with pytest.raises(ValueError, match="scores must be a CUDA tensor"):
        sa.topk_select(torch.zeros((4, 8), dtype=torch.float32), 2)


def test_wrong_dtypes_are_type_errors():
    q = torch.zeros((1, 128, 2, 64), dtype=torch.float16)
    with pytest.raises(TypeError, match="q must be torch.bfloat16"):
        sa.sparse_attn_bwd_workspace_size(q, q, q, None)
    with pytest.raises(TypeError, match="idx must be torch.int32"):
        sa.index_to_block_sparse(torch.zeros((1, 128, 2, 4), dtype=torch.int64), 128)
    with pytest.raises(TypeError, match="mask must be torch.uint8"):
        sa.block_mask_to_block_sparse(torch.zeros((1, 2, 1, 1), dtype=torch.bool), 1, 2, 128, 128)
    with pytest.raises(TypeError, match="scores must be torch.float32"):
        sa.topk_select(torch.zeros((4, 8), dtype=torch.float64), 2)
    with pytest.raises(TypeError, match="must be a torch.Tensor"):
        sa.topk_select([[1.0, 2.0]], 1)


def test_wrong_ranks_and_shapes_are_rejected():
    with pytest.raises(ValueError, match="idx must have 4 dimensions"):
        sa.index_to_block_sparse(torch.zeros((128, 2, 4), dtype=torch.int32), 128)
    with pytest.raises(ValueError, match="q must have 4 dimensions"):
        sa.sparse_attn_bwd_workspace_size(bf16(128, 2, 64), bf16(1, 128, 2, 64),
                                          bf16(1, 128, 2, 64), None)
    with pytest.raises(ValueError, match="scores must have 2 dimensions"):
        sa.topk_select(torch.zeros((2, 4, 8), dtype=torch.float32), 2)


@pytest.fixture
def cuda_check_off(monkeypatch):
    """The shape logic of the checks, on CPU tensors: only the CUDA-residency check is
    skipped (nothing here reaches a kernel)."""
    strict = sa._require

    def lenient(cond, msg, exc=ValueError):
        if "CUDA tensor" not in msg:
            strict(cond, msg, exc)

    monkeypatch.setattr(sa, "_require", lenient)


def _problem(w):
    from index_sparse_attention_b200 import inputs as I
    w = I.scaled(w, B=min(w.B, 2), Sq=min(w.Sq, 256), Sk=min(w.Sk, 256))
    q, k, v = bf16(w.B, w.Sq, w.HQ, w.Dqk), bf16(w.B, w.Sk, w.HK, w.Dqk), bf16(w.B, w.Sk, w.HK, w.Dv)
    o, do = bf16(w.B, w.Sq, w.HQ, w.Dv), bf16(w.B, w.Sq, w.HQ, w.Dv)
    lse = torch.zeros((w.B, w.HQ, w.Sq), dtype=torch.float32)
    bsp = sa.BlockSparse(_lib.SA_MODE_DENSE, w.B, w.HK, w.Sq, w.Sk, w.causal, "cpu")
    return w, q, k, v, o, do, lse, bsp


def test_valid_shapes_of_every_workload_pass(cuda_check_off):
    from index_sparse_attention_b200 import inputs as I
    for w in I.WORKLOADS.values():
        w, q, k, v, o, do, lse, bsp = _problem(w)
        status = torch.zeros(1, dtype=torch.int32)
        p = sa._params(q, k, v, o, lse, bsp, w.scale, do, torch.empty_like(q),
                       torch.empty_like(k), torch.empty_like(v), status)
        assert (p.B, p.HQ, p.HK, p.Dqk, p.Dv, p.Sq, p.Sk) == (
            w.B, w.HQ, w.HK, w.Dqk, w.Dv, w.Sq, w.Sk)
        assert sa.sparse_attn_bwd_workspace_size(q, k, v, bsp) > 0


def test_mismatched_shapes_are_rejected(cuda_check_off):
    from index_sparse_attention_b200 import inputs as I
    w, q, k, v, o, do, lse, bsp = _problem(I.WORKLOADS["gqa_blocksparse_b2_hq32_hk8_s8192_d128"])
    with pytest.raises(ValueError, match="o must have shape"):
        sa._params(q, k, v, o[:, :-1].contiguous(), lse, bsp, 0.1)
    with pytest.raises(ValueError, match="lse must have shape"):
        sa._params(q, k, v, o, lse.transpose(1, 2).contiguous(), bsp, 0.1)
    with pytest.raises(ValueError, match="dq must have shape"):
        sa._params(q, k, v, o, lse, bsp, 0.1, do, torch.empty_like(k), torch.empty_like(k),
                   torch.empty_like(v))
    with pytest.raises(ValueError, match="v must be"):
        sa._params(q, k, v[:, :-1].contiguous(), o, lse, bsp, 0.1)
    with pytest.raises(ValueError, match="k must be"):
        sa._params(q, k[:, :, :, :-8].contiguous(), v, o, lse, bsp, 0.1)
    strided = bf16(*do.shape[:3], 2 * do.shape[3])[..., ::2]  # right shape, not contiguous
    with pytest.raises(ValueError, match="dout must be contiguous"):
        sa._params(q, k, v, o, lse, bsp, 0.1, strided)
    with pytest.raises(TypeError, match="sparse must be a BlockSparse"):
        sa._params(q, k, v, o, lse, None, 0.1)
    with pytest.raises(TypeError, match="dev_status must be torch.int32"):
        sa._params(q, k, v, o, lse, bsp, 0.1, dev_status=torch.zeros(1))


ENTRY_POINTS = ("block_mask_to_block_sparse", "index_to_block_sparse", "sparse_attn_fwd",
                "sparse_attn_bwd_workspace_size", "sparse_attn_bwd", "sparse_attn_bwd_noalloc",
                "topk_select")


def test_every_entry_point_runs_on_its_tensors_device():
    """The C ABI launches on the current device, so each binding entry point makes the
    device of its tensor argument current for the call."""
    for name in ENTRY_POINTS:
        fn = getattr(sa, name)
        assert getattr(fn, "device_arg", None), f"{name} has no device guard"


def test_device_guard_enters_the_tensor_device(monkeypatch):
    entered = []

    class Recorder:
        def __init__(self, dev):
            self.dev = dev

        def __enter__(self):
            entered.append(self.dev)

        def __exit__(self, *exc):
            return False

    class FakeCuda(torch.Tensor):
        @property
        def is_cuda(self):
            return True

        @property
        def device(self):
            return torch.device("cuda", 3)

    monkeypatch.setattr(torch.cuda, "device", Recorder)
    t = torch.zeros(2).as_subclass(FakeCuda)
    guarded = sa._on_device("x")(lambda a, x=None: (a, x))
    assert guarded(1, x=t)[0] == 1 and entered == [torch.device("cuda", 3)]
    assert guarded(1, t)[0] == 1 and len(entered) == 2
    guarded(1, x=torch.zeros(2))  # a CPU tensor: no device switch
    assert len(entered) == 2
