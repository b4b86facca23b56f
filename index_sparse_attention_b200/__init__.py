"""Block-sparse and index-sparse softmax attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libsparse_attn.so`` (include/sparse_attn.h).
PyTorch supplies device memory and the current CUDA stream; every step of the
computation (tile-list conversion, forward, backward) runs in the library's CUDA
kernels.  The functions carry the names of the C entry points.
"""
import ctypes
import functools
import math

import torch

from . import _lib
from ._lib import SA_MODE_BLOCK, SA_MODE_DENSE, SA_MODE_INDEX, SA_TILE, SparseAttnError

__all__ = ["BlockSparse", "block_mask_to_block_sparse", "index_to_block_sparse",
           "sparse_attn_fwd", "sparse_attn_fwd_gather", "sparse_attn_bwd",
           "sparse_attn_bwd_workspace_size", "sparse_attn_bwd_noalloc", "topk_select",
           "sparse_attn_set_wait_limit_ns", "sparse_attn_set_forward_form",
           "sparse_attn_set_backward_form", "SparseAttnError", "SA_TILE"]


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _on_device(arg):
    """Runs the wrapped entry point with the device of its tensor argument `arg` (name)
    made current: the C ABI launches on the current device and refuses a stream of
    another device, so a tensor on cuda:1 must not be handed over while cuda:0 is
    current."""
    def deco(fn):
        import inspect
        pos = list(inspect.signature(fn).parameters).index(arg)

        @functools.wraps(fn)
        def wrapper(*args, **kw):
            t = kw.get(arg) if arg in kw else (args[pos] if pos < len(args) else None)
            if isinstance(t, torch.Tensor) and t.is_cuda:
                with torch.cuda.device(t.device):
                    return fn(*args, **kw)
            return fn(*args, **kw)

        wrapper.device_arg = arg
        return wrapper
    return deco


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(cond, msg, exc=ValueError):
    if not cond:
        raise exc(msg)


def _check(name, t, dtype, shape=None, ndim=None, device=None, contiguous=True):
    """Argument checks done here because the C ABI sees pointers and sizes only: a
    tensor of the wrong shape would be read or written out of bounds by the kernels."""
    _require(isinstance(t, torch.Tensor), f"{name} must be a torch.Tensor", TypeError)
    _require(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}", TypeError)
    if ndim is not None:
        _require(t.dim() == ndim, f"{name} must have {ndim} dimensions, got {t.dim()}")
    if shape is not None:
        _require(tuple(t.shape) == tuple(shape),
                 f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    _require(t.is_cuda, f"{name} must be a CUDA tensor")
    if contiguous:
        _require(t.is_contiguous(), f"{name} must be contiguous")
    if device is not None:
        _require(t.device == device, f"{name} is on {t.device}, expected {device}")


def _check_status(dev_status, device):
    if dev_status is not None:
        _check("dev_status", dev_status, torch.int32, device=device)
        _require(dev_status.numel() >= 1, "dev_status must hold at least one int32")


def _check_qkv(q, k, v):
    _check("q", q, torch.bfloat16, ndim=4)
    B, Sq, HQ, Dqk = q.shape
    _check("k", k, torch.bfloat16, ndim=4, device=q.device)
    _require(k.shape[0] == B and k.shape[3] == Dqk,
             f"k must be [B={B}, Sk, HK, Dqk={Dqk}], got {tuple(k.shape)}")
    _check("v", v, torch.bfloat16, ndim=4, device=q.device)
    _require(tuple(v.shape[:3]) == tuple(k.shape[:3]),
             f"v must be [B, Sk, HK, Dv] with k's first three sizes {tuple(k.shape[:3])}, "
             f"got {tuple(v.shape)}")


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


@_on_device("mask")
def block_mask_to_block_sparse(mask, B, HK, Sq, Sk, bs=SA_TILE, causal=False, device=None):
    """Tile lists from a block mask uint8 [B,HK,Mb,Nb] at granularity bs (64 or 128).

    ``mask=None`` means every block (dense attention, optionally causal).
    """
    L = _lib.load()
    if mask is not None:
        _check("mask", mask, torch.uint8, ndim=4)
        _require(tuple(mask.shape[:2]) == (B, HK),
                 f"mask must be [B={B}, HK={HK}, Mb, Nb], got {tuple(mask.shape)}")
        device = mask.device
        mode = SA_MODE_BLOCK
    else:
        mode = SA_MODE_DENSE
        device = torch.device("cuda") if device is None else torch.device(device)
        _require(device.type == "cuda", "device must be a CUDA device")
    with torch.cuda.device(device):
        bsp = BlockSparse(mode, B, HK, Sq, Sk, causal, device, bs=bs, mask=mask)
        _lib.check("block_mask_to_block_sparse",
                   L.block_mask_to_block_sparse(ctypes.byref(bsp.c), _stream(device)))
    return bsp


@_on_device("idx")
def index_to_block_sparse(idx, Sk, causal=False, dev_status=None):
    """Tile lists and presence bitmap from top-k indices int32 [B,Sq,HK,topk] (-1 = pad)."""
    L = _lib.load()
    _check("idx", idx, torch.int32, ndim=4)
    _check_status(dev_status, idx.device)
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
    _check_qkv(q, k, v)
    B, Sq, HQ, Dqk = q.shape
    _, Sk, HK, _ = k.shape
    Dv = v.shape[3]
    _require(isinstance(sparse, BlockSparse), "sparse must be a BlockSparse", TypeError)
    dev = q.device
    _check("o", o, torch.bfloat16, shape=(B, Sq, HQ, Dv), device=dev)
    _check("lse", lse, torch.float32, shape=(B, HQ, Sq), device=dev)
    for name, t, like in (("dout", dout, o), ("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t is not None:
            _check(name, t, torch.bfloat16, shape=like.shape, device=dev)
    _check_status(dev_status, dev)
    return _params_struct(q, k, v, o, lse, sparse, scale, dout, dq, dk, dv, dev_status)


def _params_struct(q, k, v, o, lse, sparse, scale, dout=None, dq=None, dk=None, dv=None,
                   dev_status=None):
    B, Sq, HQ, Dqk = q.shape
    _, Sk, HK, _ = k.shape
    Dv = v.shape[3]
    return _lib.ParamsStruct(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
        None if dout is None else dout.data_ptr(), None if dq is None else dq.data_ptr(),
        None if dk is None else dk.data_ptr(), None if dv is None else dv.data_ptr(),
        B, HQ, HK, Dqk, Dv, Sq, Sk, float(scale), ctypes.pointer(sparse.c),
        None if dev_status is None else dev_status.data_ptr())


@_on_device("q")
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


@_on_device("q")
def sparse_attn_fwd_gather(q, k, v, sparse, softmax_scale=None, o=None, lse=None,
                           dev_status=None):
    """The forward of sparse_attn_fwd by per-query gathers of the selected K/V rows
    (index mode only; HQ / HK <= 8; Dv <= 128): a comparison path, same O and LSE."""
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
    _lib.check("sparse_attn_fwd_gather", L.sparse_attn_fwd_gather(ctypes.byref(p), _stream(q.device)))
    return o, lse


@_on_device("q")
def sparse_attn_bwd_workspace_size(q, k, v, sparse):
    """Bytes of device workspace sparse_attn_bwd needs for these shapes."""
    L = _lib.load()
    _check_qkv(q, k, v)
    o = q.new_empty((1,))
    p = _params_struct(q, k, v, o, o, sparse, 1.0)
    return int(L.sparse_attn_bwd_workspace_size(ctypes.byref(p)))


@_on_device("q")
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
    _require(dout is not None, "dout is required")
    p = _params(q, k, v, o, lse, sparse, softmax_scale, dout, dq, dk, dv, dev_status)
    need = int(L.sparse_attn_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check("workspace", workspace, torch.uint8, device=q.device)
    fn = L.sparse_attn_bwd_deterministic if deterministic else L.sparse_attn_bwd
    _lib.check("sparse_attn_bwd",
               fn(ctypes.byref(p), _ptr(workspace), workspace.numel(), _stream(q.device)))
    return dq, dk, dv


@_on_device("q")
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
    _require(dout is not None, "dout is required")
    p = _params(q, k, v, o, lse, sparse, softmax_scale, dout, dq, dk, dv, dev_status)
    _lib.check("sparse_attn_bwd_noalloc", L.sparse_attn_bwd_noalloc(ctypes.byref(p),
                                                                    _stream(q.device)))
    return dq, dk, dv


@_on_device("scores")
def topk_select(scores, k, starts=None, ends=None, with_values=False, out_idx=None, out_val=None,
                dev_status=None):
    """Column indices (int32 [rows, k]) of the k largest fp32 scores of each row's range
    [starts[r], ends[r]), largest first, ties to the smaller column, -1 past the number
    of valid columns; with ``with_values`` also the selected scores (fp32 [rows, k])."""
    L = _lib.load()
    _check("scores", scores, torch.float32, ndim=2, contiguous=False)
    _require(scores.stride(1) == 1, "scores rows must be contiguous (stride(1) == 1)")
    rows, cols = scores.shape
    dev = scores.device
    for name, t in (("starts", starts), ("ends", ends)):
        if t is not None:
            _check(name, t, torch.int32, shape=(rows,), device=dev)
    _check_status(dev_status, dev)
    if out_idx is None:
        out_idx = torch.empty((rows, k), dtype=torch.int32, device=dev)
    _check("out_idx", out_idx, torch.int32, shape=(rows, k), device=dev)
    if with_values and out_val is None:
        out_val = torch.empty((rows, k), dtype=torch.float32, device=dev)
    if out_val is not None:
        _check("out_val", out_val, torch.float32, shape=(rows, k), device=dev)
    _lib.check("topk_select",
               L.topk_select(_ptr(scores), rows, cols, scores.stride(0), _ptr(starts), _ptr(ends),
                             k, _ptr(out_idx), _ptr(out_val), _ptr(dev_status),
                             _stream(scores.device)))
    return (out_idx, out_val) if with_values else out_idx


def sparse_attn_set_wait_limit_ns(ns):
    """Test instrumentation: the limit (ns) of every pipeline wait of the attention
    kernels enqueued after this call (0 restores the default of 2 s).  A wait that runs
    out sets the timeout flag (SA_STATUS_TIMEOUT, value 2) in the device status word and
    its CTA leaves; see include/sparse_attn.h."""
    _lib.check("sparse_attn_set_wait_limit_ns", _lib.load().sparse_attn_set_wait_limit_ns(int(ns)))


_FWD_FORMS = {"auto": _lib.SA_FWD_FORM_AUTO, "one_head": _lib.SA_FWD_FORM_ONE_HEAD,
              "cta_pair": _lib.SA_FWD_FORM_CTA_PAIR, "two_heads": _lib.SA_FWD_FORM_TWO_HEADS,
              "two_tiles": _lib.SA_FWD_FORM_TWO_TILES}


def sparse_attn_set_forward_form(form):
    """How the forward maps query heads and tiles to CTAs: "auto" (the library's
    choice), "one_head" (one CTA per query tile and head), "cta_pair" (two heads of a GQA
    group on a 2-CTA cluster with cta_group::2 MMAs sharing each K/V tile), "two_heads"
    (two heads of a group in one CTA, one softmax warpgroup each) or "two_tiles" (two
    consecutive query tiles of one head in one CTA, walking the union of their lists).  A
    form that does not apply to a call falls back to one head per CTA.  Applies to the forward calls made after it,
    process-wide; see include/sparse_attn.h."""
    code = _FWD_FORMS.get(form, form) if isinstance(form, str) else int(form)
    if isinstance(code, str):
        raise ValueError(f"form must be one of {sorted(_FWD_FORMS)}, got {form!r}")
    _lib.check("sparse_attn_set_forward_form", _lib.load().sparse_attn_set_forward_form(code))


_BWD_FORMS = {"auto": _lib.SA_BWD_FORM_AUTO, "split": _lib.SA_BWD_FORM_SPLIT,
              "whole": _lib.SA_BWD_FORM_WHOLE}


def sparse_attn_set_backward_form(form):
    """How the backward covers a key tile at head dims (192,128): "auto" (the library's
    choice by grid size), "split" (two CTAs per key tile, each with part of the head dim,
    both recomputing S^T and dP^T) or "whole" (one CTA per key tile, single-buffered).
    The deterministic backward always splits.  Applies to the backward calls made after
    it, process-wide; see include/sparse_attn.h."""
    code = _BWD_FORMS.get(form, form) if isinstance(form, str) else int(form)
    if isinstance(code, str):
        raise ValueError(f"form must be one of {sorted(_BWD_FORMS)}, got {form!r}")
    _lib.check("sparse_attn_set_backward_form", _lib.load().sparse_attn_set_backward_form(code))
