"""Pins of the top-k oracle (CPU): the hand-worked fixture, torch.topk on unique
scores, and an independent rank-counting definition on tie-heavy rows.  Also the
library's host-side argument checks of topk_select (no GPU needed)."""
import ctypes
import json
import os

import numpy as np
import pytest

from oracle import topk as T
from index_sparse_attention_b200 import inputs as I

HERE = os.path.dirname(os.path.abspath(__file__))


def test_golden_fixture():
    g = json.load(open(os.path.join(HERE, "golden", "topk_tiny.json")))
    scores = np.array([[float(x) for x in r] for r in g["scores"]], dtype=np.float32)
    idx, val = T.topk_select(scores, g["k"], np.array(g["starts"]), np.array(g["ends"]))
    assert idx.tolist() == g["expected"]
    for r in range(len(idx)):
        for j, c in enumerate(idx[r]):
            if c >= 0:
                assert np.array_equal(val[r, j], scores[r, c], equal_nan=True)
            else:
                assert val[r, j] == -np.inf


@pytest.mark.parametrize("k", [1, 7, 64])
def test_matches_torch_topk_on_unique_scores(k):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(k)
    R, C = 40, 300
    scores = rng.permutation(R * C).astype(np.float32).reshape(R, C) / 17.0 - 200.0
    starts = rng.integers(0, C, R).astype(np.int32)
    ends = np.minimum(C, starts + rng.integers(0, 2 * k + 5, R)).astype(np.int32)
    idx, val = T.topk_select(scores, k, starts, ends)
    for r in range(R):
        s, e = starts[r], ends[r]
        n = min(k, e - s)
        if n:
            tv, ti = torch.topk(torch.from_numpy(scores[r, s:e].copy()), n, sorted=True)
            assert idx[r, :n].tolist() == (ti.numpy() + s).tolist()
            assert np.array_equal(val[r, :n], tv.numpy())
        assert (idx[r, n:] == -1).all()


def _rank_select(row, s, e, k):
    """Independent definition: column j's rank is the number of columns of the range
    that beat it (NaN beats every number; a larger score; an equal score at a smaller
    column); the output slot of j is its rank when the rank is below k."""
    out = [-1] * k
    vals = [float(row[j]) for j in range(s, e)]
    for a, va in enumerate(vals):
        rank = 0
        for b, vb in enumerate(vals):
            if a == b:
                continue
            na, nb = np.isnan(va), np.isnan(vb)
            if nb and not na:
                rank += 1
            elif na and nb:
                rank += b < a
            elif not na and not nb:
                rank += (vb > va) or (vb == va and b < a)
        if rank < k:
            out[rank] = s + a
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_rank_counting_on_tie_heavy_rows(seed):
    rng = np.random.default_rng(100 + seed)
    R, C, k = 30, 24, 6
    levels = np.array([-1.0, -0.0, 0.0, 0.5, 2.0, np.inf, -np.inf, np.nan], dtype=np.float32)
    scores = levels[rng.integers(0, len(levels), (R, C))]
    starts = rng.integers(0, C, R).astype(np.int32)
    ends = np.minimum(C, starts + rng.integers(0, C, R)).astype(np.int32)
    idx, _ = T.topk_select(scores, k, starts, ends)
    for r in range(R):
        assert idx[r].tolist() == _rank_select(scores[r], starts[r], ends[r], k)


def test_selected_dominate_the_rest():
    x = I.topk_scores(64, 512, seed=7, dist="concentrated")
    starts, ends = I.packed_causal_ranges(64, segments=(20, 44))
    starts = np.minimum(starts, 511)
    k = 9
    idx, val = T.topk_select(x, k, starts, ends)
    for r in range(64):
        sel = [c for c in idx[r] if c >= 0]
        assert len(sel) == min(k, ends[r] - starts[r])
        rest = sorted(set(range(starts[r], ends[r])) - set(sel))
        if sel and rest:
            assert x[r, sel].min() >= x[r, rest].max()
        assert list(val[r, :len(sel)]) == sorted(val[r, :len(sel)], reverse=True)


def test_packed_ranges_are_causal_per_segment():
    s, e = I.packed_causal_ranges(10, segments=(4, 6))
    assert s.tolist() == [0, 0, 0, 0, 4, 4, 4, 4, 4, 4]
    assert e.tolist() == [1, 2, 3, 4, 5, 6, 7, 8, 9, 10]


def test_library_rejects_bad_arguments_on_host():
    from index_sparse_attention_b200 import _lib
    from index_sparse_attention_b200.build import build
    build()
    L = _lib.load()
    fake = ctypes.c_void_p(0x1000)
    assert L.topk_select(fake, 4, 8, 8, None, None, 0, fake, None, None, None) == _lib.SA_ERR_INVALID
    assert L.topk_select(fake, 4, 8, 8, None, None, _lib.SA_TOPK_MAX_K + 1, fake, None, None,
                         None) == _lib.SA_ERR_INVALID
    assert L.topk_select(fake, 4, 8, 7, None, None, 3, fake, None, None, None) == _lib.SA_ERR_INVALID
    assert L.topk_select(None, 4, 8, 8, None, None, 3, fake, None, None, None) == _lib.SA_ERR_INVALID
    assert L.topk_select(None, 0, 8, 8, None, None, 3, None, None, None, None) == _lib.SA_OK
