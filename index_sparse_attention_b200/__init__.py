"""Block-sparse and index-sparse softmax attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libsparse_attn.so`` (include/sparse_attn.h).
PyTorch supplies device memory and the current CUDA stream; every step of the
computation (tile-list conversion, forward, backward) runs in the library's CUDA
kernels.  The functions carry the names of the C entry points.
"""
import ctypes
import math

import torch

from . import _lib
from ._lib import SA_MODE_BLOCK, SA_MODE_DENSE, SA_MODE_INDEX, SA_TILE, SparseAttnError

__all__ = ["BlockSparse", "block_mask_to_block_sparse", "index_to_block_sparse",
           "sparse_attn_fwd", "sparse_attn_bwd", "sparse_attn_bwd_workspace_size",
           "sparse_attn_bwd_noalloc", "topk_select",
           "SparseAttnError", "SA_TILE"]


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class BlockSparse:
    """Tile lists (and the partial-tile mask data) of one sparsity pattern.

    Holds the device tensors the C struct ``sa_block_sparse`` points to:
    cnt [B,HK,Tm,2], idx [B,HK,Tm,Tn], tcnt [B,HK,Tn,2], tidx [B,HK,Tn,Tm] (int32),
    and ``bitmap`` [B,HK,Sq,ceil(Sk/32)] (uint32 as int32) in index mode or ``mask``
    [B,HK,Mb,Nb] (uint8) in block mode.
    """

    def __init__(self, mode, B, HK, Sq, Sk, causal, device, bs=SA_TILE, mask=None, bitmap=None):
        Tm, Tn = -(-Sq // SA_TILE), -(-Sk // SA_TILE)
        i32 = dict(dtype=torch.int32, device=device)
        self.mode, self.B, self.HK, self.Sq, self.Sk = mode, B, HK, Sq, Sk
        self.causal, self.bs, self.Tm, self.Tn = bool(causal), bs, Tm, Tn
        self.cnt = torch.empty((B, HK, Tm, 2), **i32)
        self.idx = torch.empty((B, HK, Tm, Tn), **i32)
        self.tcnt = torch.empty((B, HK, Tn, 2), **i32)
        self.tidx = torch.empty((B, HK, Tn, Tm), **i32)
        self.mask = mask
        self.bitmap = bitmap
        Mb = Nb = 0
        if mask is not None:
            Mb, Nb = mask.shape[2], mask.shape[3]
        self.c = _lib.BlockSparseStruct(
            mode, int(bool(causal)), B, HK, Sq, Sk, bs, Mb, Nb,
            None if mask is None else mask.data_ptr(),
            None if bitmap is None else bitmap.data_ptr(),
            self.cnt.data_ptr(), self.idx.data_ptr(), self.tcnt.data_ptr(), self.tidx.data_ptr())

    def active_tiles(self):
        """Active (query tile, key tile) pairs per (b, KV head), summed: full + partial."""
        return int(self.cnt.sum().item())


def block_mask_to_block_sparse(mask, B, HK, Sq, Sk, bs=SA_TILE, causal=False, device=None):
    """Tile lists from a block mask uint8 [B,HK,Mb,Nb] at granularity bs (64 or 128).

    ``mask=None`` means every block (dense attention, optionally causal).
    """
    L = _lib.load()
    if mask is not None:
        device = mask.device
        assert mask.dtype == torch.uint8 and mask.is_contiguous()
        mode = SA_MODE_BLOCK
    else:
        mode = SA_MODE_DENSE
    bsp = BlockSparse(mode, B, HK, Sq, Sk, causal, device, bs=bs, mask=mask)
    _lib.check("block_mask_to_block_sparse",
               L.block_mask_to_block_sparse(ctypes.byref(bsp.c), _stream(device)))
    return bsp


def index_to_block_sparse(idx, Sk, causal=False, dev_status=None):
    """Tile lists and presence bitmap from top-k indices int32 [B,Sq,HK,topk] (-1 = pad)."""
    L = _lib.load()
    assert idx.dtype == torch.int32 and idx.is_contiguous() and idx.dim() == 4
    B, Sq, HK, topk = idx.shape
    W = -(-Sk // 32)
    bitmap = torch.empty((B, HK, Sq, W), dtype=torch.int32, device=idx.device)
    bsp = BlockSparse(SA_MODE_INDEX, B, HK, Sq, Sk, causal, idx.device, bitmap=bitmap)
    _lib.check("index_to_block_sparse",
               L.index_to_block_sparse(_ptr(idx), topk, ctypes.byref(bsp.c), _ptr(dev_status),
                                       _stream(idx.device)))
    return bsp


def _params(q, k, v, o, lse, sparse, scale, dout=None, dq=None, dk=None, dv=None,
            dev_status=None):
    B, Sq, HQ, Dqk = q.shape
    _, Sk, HK, _ = k.shape
    Dv = v.shape[3]
    for t in (q, k, v, o, dout, dq, dk, dv):
        if t is not None:
            assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.is_cuda
    return _lib.ParamsStruct(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
        None if dout is None else dout.data_ptr(), None if dq is None else dq.data_ptr(),
        None if dk is None else dk.data_ptr(), None if dv is None else dv.data_ptr(),
        B, HQ, HK, Dqk, Dv, Sq, Sk, float(scale), ctypes.pointer(sparse.c),
        None if dev_status is None else dev_status.data_ptr())


def sparse_attn_fwd(q, k, v, sparse, softmax_scale=None, o=None, lse=None, dev_status=None):
    """O [B,Sq,HQ,Dv] (bf16) and LSE [B,HQ,Sq] (fp32) of sparse attention."""
    L = _lib.load()
    B, Sq, HQ, Dqk = q.shape
    Dv = v.shape[3]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(Dqk)
    if o is None:
        o = torch.empty((B, Sq, HQ, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, HQ, Sq), dtype=torch.float32, device=q.device)
    p = _params(q, k, v, o, lse, sparse, softmax_scale, dev_status=dev_status)
    _lib.check("sparse_attn_fwd", L.sparse_attn_fwd(ctypes.byref(p), _stream(q.device)))
    return o, lse


def sparse_attn_bwd_workspace_size(q, k, v, sparse):
    L = _lib.load()
    o = q.new_empty((1,))
    p = _params(q, k, v, o, o, sparse, 1.0)
    p.Dv = v.shape[3]
    return int(L.sparse_attn_bwd_workspace_size(ctypes.byref(p)))


def sparse_attn_bwd(q, k, v, o, lse, dout, sparse, softmax_scale=None, dq=None, dk=None,
                    dv=None, workspace=None, dev_status=None, deterministic=False):
    """dQ, dK, dV (bf16, layouts of q, k, v) of sparse attention; with
    ``deterministic`` dQ is accumulated in a fixed order (bitwise reproducible)."""
    L = _lib.load()
    Dqk = q.shape[3]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(Dqk)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    p = _params(q, k, v, o, lse, sparse, softmax_scale, dout, dq, dk, dv, dev_status)
    need = int(L.sparse_attn_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    fn = L.sparse_attn_bwd_deterministic if deterministic else L.sparse_attn_bwd
    _lib.check("sparse_attn_bwd",
               fn(ctypes.byref(p), _ptr(workspace), workspace.numel(), _stream(q.device)))
    return dq, dk, dv


def sparse_attn_bwd_noalloc(q, k, v, o, lse, dout, sparse, softmax_scale=None, dq=None, dk=None,
                            dv=None, dev_status=None):
    """dQ, dK, dV like sparse_attn_bwd, with the scratch taken from the library's fixed
    device array instead of a workspace (for callers that cannot allocate device memory;
    see include/sparse_attn.h).  Calls on one device share that array: do not overlap
    them on the GPU."""
    L = _lib.load()
    Dqk = q.shape[3]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(Dqk)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    p = _params(q, k, v, o, lse, sparse, softmax_scale, dout, dq, dk, dv, dev_status)
    _lib.check("sparse_attn_bwd_noalloc", L.sparse_attn_bwd_noalloc(ctypes.byref(p),
                                                                    _stream(q.device)))
    return dq, dk, dv


def topk_select(scores, k, starts=None, ends=None, with_values=False, out_idx=None, out_val=None,
                dev_status=None):
    """Column indices (int32 [rows, k]) of the k largest fp32 scores of each row's range
    [starts[r], ends[r]), largest first, ties to the smaller column, -1 past the number
    of valid columns; with ``with_values`` also the selected scores (fp32 [rows, k])."""
    L = _lib.load()
    assert scores.dtype == torch.float32 and scores.dim() == 2 and scores.is_cuda
    assert scores.stride(1) == 1
    rows, cols = scores.shape
    for t in (starts, ends):
        if t is not None:
            assert t.dtype == torch.int32 and t.is_contiguous() and t.numel() == rows
    if out_idx is None:
        out_idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    if with_values and out_val is None:
        out_val = torch.empty((rows, k), dtype=torch.float32, device=scores.device)
    _lib.check("topk_select",
               L.topk_select(_ptr(scores), rows, cols, scores.stride(0), _ptr(starts), _ptr(ends),
                             k, _ptr(out_idx), _ptr(out_val), _ptr(dev_status),
                             _stream(scores.device)))
    return (out_idx, out_val) if with_values else out_idx

