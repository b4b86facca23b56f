"""Pins of the fp64 CPU oracle against things other than itself.

Every check here runs on the CPU and compares the oracle (oracle/oracle.c) with
  * a library routine: torch's scaled_dot_product_attention in fp64 (dense and
    element-masked attention) and its autograd gradients,
  * closed forms: zero queries give LSE = log|A_i| and O = mean of the allowed values;
    all-ones values give O = 1 (softmax rows sum to one); one allowed key gives
    O = v_j and LSE = s_ij; an empty allowed set gives O = 0 and LSE = -inf,
  * central finite differences of L = sum(dO * O) at S=32, D=16,
  * explicit gathering of the top-k keys (index mode),
  * an independent dense-matrix classification and hand-counted golden lists for the
    tile lists and the presence bitmap.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, shape):
    return np.random.default_rng(seed).standard_normal(shape)


def allowed_dense(B, HK, Sq, Sk, causal, mode, mask=None, bs=None, idx=None):
    """Independent numpy construction of the allowed matrix [B, HK, Sq, Sk]."""
    if mode == "dense":
        A = np.ones((B, HK, Sq, Sk), bool)
    elif mode == "block":
        A = np.kron(mask.astype(bool), np.ones((bs, bs), bool))[:, :, :Sq, :Sk]
    else:
        A = np.zeros((B, HK, Sq, Sk), bool)
        bb, ii, gg, tt = np.nonzero(idx >= 0)
        A[bb, gg, ii, idx[bb, ii, gg, tt]] = True
    if causal:
        A &= np.tril(np.ones((Sq, Sk), bool))[None, None]
    return A


def sdpa_ref(q, k, v, A, scale):
    """O [B,Sq,HQ,Dv] and LSE [B,HQ,Sq] from torch SDPA (fp64, CPU) with a boolean mask.

    LSE comes from a second SDPA call with one extra "sink" key of score 0 whose value
    is a unit vector in an extra column: that column of the output is 1 / (Z + 1) with
    Z = sum_j exp(s_ij), so LSE = log(1 / o - 1).
    """
    B, Sq, HQ, _ = q.shape
    HK = k.shape[2]
    G = HQ // HK
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    tA = torch.from_numpy(A).repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=tA, scale=scale)
    Dv = v.shape[3]
    tk2 = torch.cat([tk, torch.zeros_like(tk[:, :, :1])], dim=2)
    tv2 = torch.cat([torch.cat([tv, torch.zeros_like(tv[..., :1])], dim=3),
                     torch.zeros_like(tv[:, :, :1, :1]).expand(B, HQ, 1, Dv + 1).clone()], dim=2)
    tv2[:, :, -1, -1] = 1.0
    tA2 = torch.cat([tA, torch.ones_like(tA[..., :1])], dim=3)
    o2 = F.scaled_dot_product_attention(tq, tk2, tv2, attn_mask=tA2, scale=scale)
    lse = torch.log(1.0 / o2[..., -1] - 1.0)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


def sdpa_grads(q, k, v, dout, A, scale):
    B, Sq, HQ, _ = q.shape
    G = HQ // k.shape[2]
    tq = torch.from_numpy(q).permute(0, 2, 1, 3).requires_grad_(True)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).requires_grad_(True)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).requires_grad_(True)
    tA = torch.from_numpy(A).repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(tq, tk.repeat_interleave(G, dim=1),
                                       tv.repeat_interleave(G, dim=1), attn_mask=tA, scale=scale)
    (o * torch.from_numpy(dout).permute(0, 2, 1, 3)).sum().backward()
    return tuple(t.grad.permute(0, 2, 1, 3).numpy() for t in (tq, tk, tv))


CASES = [
    # B, Sq, Sk, HQ, HK, Dqk, Dv, causal, mode, bs
    (1, 40, 40, 2, 2, 16, 16, False, "dense", 0),
    (2, 37, 45, 4, 2, 16, 8, True, "dense", 0),
    (1, 64, 64, 4, 1, 32, 32, False, "block", 8),
    (2, 48, 52, 4, 2, 16, 24, True, "block", 16),
    (1, 50, 50, 4, 2, 16, 16, True, "index", 0),
    (1, 33, 41, 2, 2, 8, 16, False, "index", 0),
]


def make_case(c, seed=0, topk=12):
    B, Sq, Sk, HQ, HK, Dqk, Dv, causal, mode, bs = c
    q, k, v = rnd(seed, (B, Sq, HQ, Dqk)), rnd(seed + 1, (B, Sk, HK, Dqk)), rnd(seed + 2, (B, Sk, HK, Dv))
    dout = rnd(seed + 3, (B, Sq, HQ, Dv))
    mask = idx = None
    rng = np.random.default_rng(seed + 4)
    if mode == "block":
        Mb, Nb = -(-Sq // bs), -(-Sk // bs)
        mask = (rng.random((B, HK, Mb, Nb)) < 0.5).astype(np.uint8)
        for m in range(min(Mb, Nb)):
            mask[:, :, m, m] = 1  # keep a key for every row
    elif mode == "index":
        idx = np.full((B, Sq, HK, topk), -1, np.int32)
        for b in range(B):
            for i in range(Sq):
                hi = min(i, Sk - 1) if causal else Sk - 1
                for g in range(HK):
                    n = rng.integers(1, topk + 1)
                    sel = rng.integers(0, hi + 1, size=n)  # duplicates allowed on purpose
                    sel[0] = min(i, Sk - 1)  # never empty
                    idx[b, i, g, :n] = sel
    P = oracle.Problem(q, k, v, scale=1.0 / np.sqrt(Dqk), causal=causal, mode=mode, mask=mask,
                       bs=bs, idx=idx)
    A = allowed_dense(B, HK, Sq, Sk, causal, mode, mask, bs, idx)
    return P, A, dout


@pytest.mark.parametrize("case", CASES, ids=[f"{c[8]}-{'causal' if c[7] else 'full'}-{c[1]}x{c[2]}" for c in CASES])
def test_forward_matches_sdpa(case):
    """All-ones (dense), block-masked and index-sparse forward == SDPA with -inf masking."""
    P, A, _ = make_case(case)
    O, lse = oracle.forward(P)
    O_ref, lse_ref = sdpa_ref(P.q, P.k, P.v, A, P.c.scale)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-10)


@pytest.mark.parametrize("Sq,Sk", [(37, 45), (45, 37), (40, 40)])
def test_causal_alignment_matches_sdpa_is_causal(Sq, Sk):
    """The causal reading (top-left: key j allowed for query i iff j <= i, also when
    Sq != Sk) equals torch SDPA's own is_causal mask, with no mask built here."""
    q, k, v = rnd(10, (1, Sq, 2, 16)), rnd(11, (1, Sk, 2, 16)), rnd(12, (1, Sk, 2, 16))
    dout = rnd(13, (1, Sq, 2, 16))
    P = oracle.Problem(q, k, v, scale=0.25, causal=True, mode="dense")
    O, lse = oracle.forward(P)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).requires_grad_(True) for x in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.25)
    np.testing.assert_allclose(O, o.detach().permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    (o * torch.from_numpy(dout).permute(0, 2, 1, 3)).sum().backward()
    dq, dk, dv = oracle.backward(P, dout, O, lse)
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, t.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("case", CASES, ids=[f"{c[8]}-{'causal' if c[7] else 'full'}-{c[1]}x{c[2]}" for c in CASES])
def test_backward_matches_autograd(case):
    P, A, dout = make_case(case, seed=10)
    dQ, dK, dV = oracle.backward(P, dout)
    rQ, rK, rV = sdpa_grads(P.q, P.k, P.v, dout, A, P.c.scale)
    for got, ref in ((dQ, rQ), (dK, rK), (dV, rV)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11 * max(1.0, np.abs(ref).max()))


def test_index_equals_explicit_gather():
    """Index mode == dense attention over the gathered (deduplicated) top-k key rows."""
    P, A, _ = make_case(CASES[4], seed=20)
    O, lse = oracle.forward(P)
    G = P.HQ // P.HK
    for b in range(P.B):
        for h in range(P.HQ):
            g = h // G
            for i in range(P.Sq):
                sel = np.unique(P.idx[b, i, g][P.idx[b, i, g] >= 0])
                sel = sel[sel <= i] if P.c.causal else sel
                kk = torch.from_numpy(P.k[b, sel, g])[None, None]
                vv = torch.from_numpy(P.v[b, sel, g])[None, None]
                qq = torch.from_numpy(P.q[b, i, h])[None, None, None]
                o = F.scaled_dot_product_attention(qq, kk, vv, scale=P.c.scale)[0, 0, 0].numpy()
                np.testing.assert_allclose(O[b, i, h], o, rtol=0, atol=1e-12)


def test_zero_queries_closed_form():
    """q = 0: every score is 0, so LSE_i = log|A_i| and O_i = mean of v_j over A_i."""
    for c in CASES:
        P, A, _ = make_case(c, seed=30)
        P = oracle.Problem(np.zeros_like(P.q), P.k, P.v, scale=P.c.scale, causal=bool(P.c.causal),
                           mode=["dense", "block", "index"][P.c.mode], mask=P.mask, bs=P.c.bs,
                           idx=P.idx)
        O, lse = oracle.forward(P)
        G = P.HQ // P.HK
        for h in range(P.HQ):
            Ah = A[:, h // G]  # [B, Sq, Sk]
            n = Ah.sum(-1)
            np.testing.assert_allclose(lse[:, h], np.log(n), rtol=0, atol=1e-13)
            mean = np.einsum("bij,bjd->bid", Ah.astype(np.float64), P.v[:, :, h // G]) / n[..., None]
            np.testing.assert_allclose(O[:, :, h], mean, rtol=0, atol=1e-13)


def test_softmax_rows_sum_to_one():
    """v = 1 everywhere: O_i = sum_j P_ij = 1 for every non-empty row."""
    for c in CASES:
        P, _, _ = make_case(c, seed=40)
        P1 = oracle.Problem(P.q * 3.0, P.k, np.ones_like(P.v), scale=P.c.scale,
                            causal=bool(P.c.causal), mode=["dense", "block", "index"][P.c.mode],
                            mask=P.mask, bs=P.c.bs, idx=P.idx)
        O, _ = oracle.forward(P1)
        np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-12)


def test_single_key_and_empty_rows():
    """One allowed key: O = v_j, LSE = scale q.k.  No allowed key: O = 0, LSE = -inf, dq = 0."""
    B, S, H, D = 1, 6, 1, 8
    q, k, v, dout = rnd(50, (B, S, H, D)), rnd(51, (B, S, H, D)), rnd(52, (B, S, H, D)), rnd(53, (B, S, H, D))
    idx = np.full((B, S, H, 2), -1, np.int32)
    pick = [3, 0, 5, -1, 1, 4]
    for i, j in enumerate(pick):
        idx[0, i, 0, 0] = j
    P = oracle.Problem(q, k, v, scale=0.3, causal=False, mode="index", idx=idx)
    O, lse = oracle.forward(P)
    for i, j in enumerate(pick):
        if j < 0:
            assert np.all(O[0, i, 0] == 0.0) and lse[0, 0, i] == -np.inf
        else:
            np.testing.assert_allclose(O[0, i, 0], v[0, j, 0], rtol=0, atol=1e-14)
            np.testing.assert_allclose(lse[0, 0, i], 0.3 * np.dot(q[0, i, 0], k[0, j, 0]), rtol=0,
                                       atol=1e-14)
    dQ, dK, dV = oracle.backward(P, dout)
    assert np.all(dQ[0, 3] == 0.0)
    # a single allowed key has P = 1 and dS = dP - Delta = 0, so every gradient of q is 0
    np.testing.assert_allclose(dQ, 0.0, atol=1e-13)


def _loss(P, dout):
    O, _ = oracle.forward(P)
    return float((O * dout).sum())


@pytest.mark.parametrize("mode,causal,HQ,HK", [("block", False, 2, 2), ("block", True, 4, 2),
                                               ("dense", True, 4, 2), ("index", True, 2, 1)])
def test_gradients_central_differences(mode, causal, HQ, HK):
    """dQ, dK, dV == central finite differences of L = sum(dO * O) (S=32, D=16, h=1e-6)."""
    B, S, D = 1, 32, 16
    q, k, v, dout = rnd(60, (B, S, HQ, D)), rnd(61, (B, S, HK, D)), rnd(62, (B, S, HK, D)), rnd(63, (B, S, HQ, D))
    rng = np.random.default_rng(64)
    mask = idx = None
    bs = 8
    if mode == "block":
        mask = (rng.random((B, HK, 4, 4)) < 0.5).astype(np.uint8)
        for m in range(4):
            mask[:, :, m, m] = 1
    if mode == "index":
        idx = np.full((B, S, HK, 6), -1, np.int32)
        for i in range(S):
            for g in range(HK):
                idx[0, i, g, :] = rng.integers(0, i + 1, size=6)
                idx[0, i, g, 0] = i
    kw = dict(scale=0.25, causal=causal, mode=mode, mask=mask, bs=bs, idx=idx)
    P = oracle.Problem(q, k, v, **kw)
    dQ, dK, dV = oracle.backward(P, dout)
    h = 1e-6
    for name, arr, grad in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
        flat = np.random.default_rng(65).choice(arr.size, size=48, replace=False)
        fd = np.empty(len(flat))
        for t, e in enumerate(flat):
            ap, am = arr.copy(), arr.copy()
            ap.flat[e] += h
            am.flat[e] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = ap
            lp = _loss(oracle.Problem(args["q"], args["k"], args["v"], **kw), dout)
            args[name] = am
            lm = _loss(oracle.Problem(args["q"], args["k"], args["v"], **kw), dout)
            fd[t] = (lp - lm) / (2 * h)
        an = grad.flat[flat]
        rel = np.abs(fd - an).max() / max(np.abs(an).max(), 1e-30)
        assert rel <= 1e-6, (name, rel)


# ---------------------------------------------------------------------------------
# Tile lists and presence bitmap
# ---------------------------------------------------------------------------------

def numpy_lists(A, T, Sk):
    """Independent classification from the dense allowed matrix A [B,HK,Sq,Sk]."""
    B, HK, Sq, _ = A.shape
    Tm, Tn = -(-Sq // T), -(-Sk // T)
    pad = np.zeros((B, HK, Tm * T, Tn * T), bool)
    valid = np.zeros_like(pad)
    pad[:, :, :Sq, :Sk] = A
    valid[:, :, :Sq, :Sk] = True
    t = pad.reshape(B, HK, Tm, T, Tn, T)
    vt = valid.reshape(B, HK, Tm, T, Tn, T)
    anyt = t.any(axis=(3, 5))
    allt = (t | ~vt).all(axis=(3, 5))
    allt[..., (np.arange(Tn) + 1) * T > Sk] = False
    cls = np.where(anyt, np.where(allt, 2, 1), 0)
    out = {"cnt": np.zeros((B, HK, Tm, 2), np.int32), "idx": np.full((B, HK, Tm, Tn), -1, np.int32),
           "tcnt": np.zeros((B, HK, Tn, 2), np.int32), "tidx": np.full((B, HK, Tn, Tm), -1, np.int32)}
    for b in range(B):
        for g in range(HK):
            for m in range(Tm):
                f = np.nonzero(cls[b, g, m] == 2)[0]
                p = np.nonzero(cls[b, g, m] == 1)[0]
                out["cnt"][b, g, m] = (len(f), len(p))
                out["idx"][b, g, m, :len(f) + len(p)] = np.concatenate([f, p])
            for n in range(Tn):
                f = np.nonzero(cls[b, g, :, n] == 2)[0]
                p = np.nonzero(cls[b, g, :, n] == 1)[0]
                out["tcnt"][b, g, n] = (len(f), len(p))
                out["tidx"][b, g, n, :len(f) + len(p)] = np.concatenate([f, p])
    return out


def numpy_bitmap(idx, Sk):
    B, Sq, HK, _ = idx.shape
    W = -(-Sk // 32)
    bits = np.zeros((B, HK, Sq, W * 32), np.uint64)
    bb, ii, gg, tt = np.nonzero(idx >= 0)
    bits[bb, gg, ii, idx[bb, ii, gg, tt]] = 1
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (bits.reshape(B, HK, Sq, W, 32) * weights).sum(-1).astype(np.uint32)


@pytest.mark.parametrize("case", CASES, ids=[f"{c[8]}-{'causal' if c[7] else 'full'}-{c[1]}x{c[2]}" for c in CASES])
@pytest.mark.parametrize("T", [4, 16])
def test_block_lists_match_dense_classification(case, T):
    P, A, _ = make_case(case, seed=70)
    got = oracle.block_lists(P, tile=T)
    ref = numpy_lists(A, T, P.Sk)
    for key in ("cnt", "idx", "tcnt", "tidx"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=key)
    if P.idx is not None:
        np.testing.assert_array_equal(got["bitmap"], numpy_bitmap(P.idx, P.Sk))


def test_block_lists_golden():
    cases = json.load(open(os.path.join(GOLDEN, "converter_tiny.json")))["cases"]
    for c in cases:
        B, HK, Sq, Sk, T = c["B"], c["HK"], c["Sq"], c["Sk"], c["T"]
        q = np.zeros((B, Sq, HK, 4))
        k = np.zeros((B, Sk, HK, 4))
        if c["mode"] == "index":
            idx = np.array(c["idx"], np.int32).reshape(B, Sq, HK, -1)
            P = oracle.Problem(q, k, k, scale=1.0, causal=bool(c["causal"]), mode="index", idx=idx)
        else:
            mask = np.array(c["mask"], np.uint8).reshape(B, HK, *np.array(c["mask"]).shape)
            P = oracle.Problem(q, k, k, scale=1.0, causal=bool(c["causal"]), mode="block",
                               mask=mask, bs=c["bs"])
        got = oracle.block_lists(P, tile=T)
        np.testing.assert_array_equal(got["cnt"][0, 0], c["cnt"], err_msg=c["name"])
        np.testing.assert_array_equal(got["idx"][0, 0], c["idx_lists"], err_msg=c["name"])
        np.testing.assert_array_equal(got["tcnt"][0, 0], c["tcnt"], err_msg=c["name"])
        np.testing.assert_array_equal(got["tidx"][0, 0], c["tidx_lists"], err_msg=c["name"])
        if "bitmap" in c:
            np.testing.assert_array_equal(got["bitmap"][0, 0, :, 0], c["bitmap"], err_msg=c["name"])


def test_out_of_range_index_is_rejected():
    q = np.zeros((1, 4, 1, 4))
    idx = np.zeros((1, 4, 1, 2), np.int32)
    idx[0, 2, 0, 1] = 4  # Sk = 4: out of range
    P = oracle.Problem(q, q, q, scale=1.0, mode="index", idx=idx)
    with pytest.raises(RuntimeError):
        oracle.block_lists(P, tile=4)
    idx[0, 2, 0, 1] = -2
    P = oracle.Problem(q, q, q, scale=1.0, mode="index", idx=idx)
    with pytest.raises(RuntimeError):
        oracle.forward(P)
