"""Shared helpers for the parity tests: seeded inputs on the GPU, oracle runs, checks.

The tolerances are the acceptance bar for this library: O, dQ, dK and dV within
max-abs error <= 2e-2 * max|reference|, LSE within max-abs error <= 1e-3 (natural
log), tile lists and bitmaps bit-exact.
"""
import numpy as np

import oracle
from index_sparse_attention_b200 import inputs as I

O_TOL = 2e-2  # relative to max |reference|
LSE_TOL = 1e-3  # absolute


def oracle_problem(inp: I.Inputs):
    w = inp.w
    kw = dict(scale=w.scale, causal=w.causal)
    if w.mode == "block":
        kw.update(mode="block", mask=inp.mask, bs=w.bs)
    elif w.mode == "index":
        kw.update(mode="index", idx=inp.idx)
    return oracle.Problem(inp.f32("q"), inp.f32("k"), inp.f32("v"), **kw)


def to_gpu(inp: I.Inputs, device="cuda"):
    import torch

    def bf(a):
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)

    out = dict(q=bf(inp.q), k=bf(inp.k), v=bf(inp.v))
    if inp.do is not None:
        out["do"] = bf(inp.do)
    if inp.mask is not None:
        out["mask"] = torch.from_numpy(inp.mask).to(device)
    if inp.idx is not None:
        out["idx"] = torch.from_numpy(inp.idx).to(device)
    return out


def build_lists(inp: I.Inputs, g, dev_status=None):
    import index_sparse_attention_b200 as sa
    w = inp.w
    if w.mode == "block":
        return sa.block_mask_to_block_sparse(g["mask"], w.B, w.HK, w.Sq, w.Sk, bs=w.bs,
                                             causal=w.causal)
    return sa.index_to_block_sparse(g["idx"], w.Sk, causal=w.causal, dev_status=dev_status)


def bf16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def max_rel_err(got, ref):
    scale = max(np.abs(ref).max(), 1e-30)
    return np.abs(got - ref).max() / scale


def assert_close(name, got, ref, tol=O_TOL):
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    err = max_rel_err(got, ref)
    assert err <= tol, f"{name}: max-abs error {err:.3e} x max|ref| exceeds {tol}"
    return err


def assert_lse(got, ref, tol=LSE_TOL):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "LSE: -inf pattern differs"
    if fin.any():
        err = np.abs(got[fin] - ref[fin]).max()
        assert err <= tol, f"LSE: max-abs error {err:.3e} exceeds {tol}"
        return err
    return 0.0
