"""fp64 CPU oracle for block-sparse / index-sparse softmax attention.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product path never does.
It shares no code with the CUDA library.  The arithmetic lives in ``oracle.c``
(plain loops, fp64); this module only marshals numpy arrays through ctypes.

Inputs are fp64 arrays (bf16 values widen to them exactly), in the layouts
q [B,Sq,HQ,Dqk], k [B,Sk,HK,Dqk], v [B,Sk,HK,Dv], dO [B,Sq,HQ,Dv].
"""
import ctypes
import os

import numpy as np

from .build import build as _build

DENSE, BLOCK, INDEX = 0, 1, 2
_MODES = {"dense": DENSE, "block": BLOCK, "index": INDEX}


class _Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("Sq", ctypes.c_int64), ("Sk", ctypes.c_int64),
        ("HQ", ctypes.c_int64), ("HK", ctypes.c_int64), ("Dqk", ctypes.c_int64),
        ("Dv", ctypes.c_int64), ("scale", ctypes.c_double), ("causal", ctypes.c_int64),
        ("mode", ctypes.c_int64), ("mask", ctypes.c_void_p), ("bs", ctypes.c_int64),
        ("Mb", ctypes.c_int64), ("Nb", ctypes.c_int64), ("idx", ctypes.c_void_p),
        ("topk", ctypes.c_int64),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(_Problem)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        L.oracle_fwd_rows.argtypes = [P, vp, vp, vp, i64, vp, vp, vp]
        L.oracle_delta_rows.argtypes = [P, vp, i64, vp, vp, vp]
        L.oracle_bwd_rows.argtypes = [P, vp, vp, vp, vp, vp, vp, i64, vp, vp]
        L.oracle_bwd_keys.argtypes = [P, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp]
        L.oracle_presence_bitmap.argtypes = [P, vp]
        L.oracle_block_lists.argtypes = [P, i64, vp, vp, vp, vp, vp]
        L.oracle_is_allowed.argtypes = [P, i64, i64, i64, i64]
        for f in ("oracle_fwd_rows", "oracle_delta_rows", "oracle_bwd_rows", "oracle_bwd_keys",
                  "oracle_presence_bitmap", "oracle_block_lists", "oracle_is_allowed"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


class Problem:
    """Shapes, scale and allowed-set specification of one attention problem.

    mode: "dense" | "block" | "index".  Block mode takes ``mask`` uint8
    [B,HK,Mb,Nb] at granularity ``bs``; index mode takes ``idx`` int32
    [B,Sq,HK,topk] with -1 padding.
    """

    def __init__(self, q, k, v, *, scale, causal=False, mode="dense", mask=None, bs=0,
                 idx=None):
        self.q = np.ascontiguousarray(q, dtype=np.float64)
        self.k = np.ascontiguousarray(k, dtype=np.float64)
        self.v = np.ascontiguousarray(v, dtype=np.float64)
        B, Sq, HQ, Dqk = self.q.shape
        _, Sk, HK, _ = self.k.shape
        Dv = self.v.shape[3]
        self.mask = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
        self.idx = None if idx is None else np.ascontiguousarray(idx, dtype=np.int32)
        Mb = Nb = 0
        if self.mask is not None:
            Mb, Nb = self.mask.shape[2], self.mask.shape[3]
        topk = 0 if self.idx is None else self.idx.shape[3]
        self.c = _Problem(B, Sq, Sk, HQ, HK, Dqk, Dv, float(scale), int(bool(causal)),
                          _MODES[mode], _ptr(self.mask), int(bs), Mb, Nb, _ptr(self.idx), topk)
        self.B, self.Sq, self.Sk, self.HQ, self.HK, self.Dqk, self.Dv = B, Sq, Sk, HQ, HK, Dqk, Dv

    def all_rows(self):
        b, h, i = np.meshgrid(np.arange(self.B), np.arange(self.HQ), np.arange(self.Sq),
                              indexing="ij")
        return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int64)

    def all_keys(self):
        b, g, j = np.meshgrid(np.arange(self.B), np.arange(self.HK), np.arange(self.Sk),
                              indexing="ij")
        return np.stack([b.ravel(), g.ravel(), j.ravel()], axis=1).astype(np.int64)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def forward_rows(P, rows):
    """O (n, Dv) and LSE (n,) in fp64 for rows given as (b, h, i) triplets."""
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    o = np.zeros((len(rows), P.Dv), np.float64)
    lse = np.zeros(len(rows), np.float64)
    _check(lib().oracle_fwd_rows(ctypes.byref(P.c), _ptr(P.q), _ptr(P.k), _ptr(P.v), len(rows),
                                 _ptr(rows), _ptr(o), _ptr(lse)), "forward")
    return o, lse


def forward(P):
    """Full O [B,Sq,HQ,Dv] and LSE [B,HQ,Sq] in fp64."""
    rows = P.all_rows()
    o, lse = forward_rows(P, rows)
    O = o.reshape(P.B, P.HQ, P.Sq, P.Dv).transpose(0, 2, 1, 3).copy()
    return O, lse.reshape(P.B, P.HQ, P.Sq)


def delta(P, dout, O):
    """Delta [B,HQ,Sq] = <dO_i, O_i> from the oracle's own fp64 O [B,Sq,HQ,Dv]."""
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    rows = P.all_rows()
    o_rows = np.ascontiguousarray(O.transpose(0, 2, 1, 3).reshape(-1, P.Dv), dtype=np.float64)
    d = np.zeros(len(rows), np.float64)
    _check(lib().oracle_delta_rows(ctypes.byref(P.c), _ptr(dout), len(rows), _ptr(rows),
                                   _ptr(o_rows), _ptr(d)), "delta")
    return d.reshape(P.B, P.HQ, P.Sq)


def backward_rows(P, dout, lse, dlt, rows):
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    dlt = np.ascontiguousarray(dlt, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    dq = np.zeros((len(rows), P.Dqk), np.float64)
    _check(lib().oracle_bwd_rows(ctypes.byref(P.c), _ptr(P.q), _ptr(P.k), _ptr(P.v), _ptr(dout),
                                 _ptr(lse), _ptr(dlt), len(rows), _ptr(rows), _ptr(dq)), "bwd rows")
    return dq


def backward_keys(P, dout, lse, dlt, keys):
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    dlt = np.ascontiguousarray(dlt, dtype=np.float64)
    keys = np.ascontiguousarray(keys, dtype=np.int64).reshape(-1, 3)
    dk = np.zeros((len(keys), P.Dqk), np.float64)
    dv = np.zeros((len(keys), P.Dv), np.float64)
    _check(lib().oracle_bwd_keys(ctypes.byref(P.c), _ptr(P.q), _ptr(P.k), _ptr(P.v), _ptr(dout),
                                 _ptr(lse), _ptr(dlt), len(keys), _ptr(keys), _ptr(dk), _ptr(dv)),
           "bwd keys")
    return dk, dv


def backward(P, dout, O=None, lse=None):
    """Full fp64 gradients: dQ [B,Sq,HQ,Dqk], dK [B,Sk,HK,Dqk], dV [B,Sk,HK,Dv]."""
    if O is None or lse is None:
        O, lse = forward(P)
    dlt = delta(P, dout, O)
    dq = backward_rows(P, dout, lse, dlt, P.all_rows())
    dk, dv = backward_keys(P, dout, lse, dlt, P.all_keys())
    dQ = dq.reshape(P.B, P.HQ, P.Sq, P.Dqk).transpose(0, 2, 1, 3).copy()
    dK = dk.reshape(P.B, P.HK, P.Sk, P.Dqk).transpose(0, 2, 1, 3).copy()
    dV = dv.reshape(P.B, P.HK, P.Sk, P.Dv).transpose(0, 2, 1, 3).copy()
    return dQ, dK, dV


def presence_bitmap(P):
    W = (P.Sk + 31) // 32
    bm = np.zeros((P.B, P.HK, P.Sq, W), np.uint32)
    _check(lib().oracle_presence_bitmap(ctypes.byref(P.c), _ptr(bm)), "bitmap")
    return bm


def block_lists(P, tile=128):
    """Tile lists of the oracle: dict with cnt, idx, tcnt, tidx (and bitmap in index mode)."""
    Tm, Tn = -(-P.Sq // tile), -(-P.Sk // tile)
    out = dict(
        cnt=np.zeros((P.B, P.HK, Tm, 2), np.int32), idx=np.zeros((P.B, P.HK, Tm, Tn), np.int32),
        tcnt=np.zeros((P.B, P.HK, Tn, 2), np.int32), tidx=np.zeros((P.B, P.HK, Tn, Tm), np.int32))
    bm = None
    if P.c.mode == INDEX:
        bm = np.zeros((P.B, P.HK, P.Sq, (P.Sk + 31) // 32), np.uint32)
        out["bitmap"] = bm
    _check(lib().oracle_block_lists(ctypes.byref(P.c), tile, _ptr(bm), _ptr(out["cnt"]),
                                    _ptr(out["idx"]), _ptr(out["tcnt"]), _ptr(out["tidx"])),
           "block lists")
    return out


def is_allowed(P, b, g, i, j):
    return bool(lib().oracle_is_allowed(ctypes.byref(P.c), b, g, i, j))
