"""Top-k selection oracle (plain numpy, one row at a time).

TEST INFRASTRUCTURE ONLY: the test suite and the benchmark's CPU-baseline leg may
import this module; the product path never does.  It shares no code with the CUDA
library.

Operation (xtuner PR #2096, "[Feature] Add optional TileLang Top-K selector", Main
Changes 1): for each row, among the columns of its valid range [start, end), take the
k largest scores ordered largest first (the order torch.topk gives with sorted=True)
and return their column indices as int32, -1 in the slots past the number of valid
columns.  Where the page leaves the order open: ties go to the smaller column (the page
avoids ties by testing unique values; torch leaves their order unspecified), -0 equals
+0, and every NaN ranks above +inf.
"""
import numpy as np


def topk_row(scores, start, end, k):
    """(indices int32 [k], values float32 [k]) of one row: a sort of the valid range by
    (NaN first, then score descending, then column ascending)."""
    v = np.asarray(scores[start:end], dtype=np.float64)
    cols = np.arange(start, end, dtype=np.int64)
    nan = np.isnan(v)
    vv = np.where(nan, 0.0, v)
    # np.lexsort sorts by the last key first: NaN before numbers, then -score, then column
    order = np.lexsort((cols, -vv, ~nan))
    take = order[:k]
    idx = np.full(k, -1, dtype=np.int32)
    val = np.full(k, -np.inf, dtype=np.float32)
    idx[:len(take)] = cols[take]
    val[:len(take)] = scores[start:end][take]
    return idx, val


def topk_select(scores, k, starts=None, ends=None, rows=None):
    """Top-k of every row (or of the listed rows) of a 2-D float32 score array."""
    scores = np.asarray(scores, dtype=np.float32)
    R, C = scores.shape
    rows = np.arange(R) if rows is None else np.asarray(rows)
    idx = np.empty((len(rows), k), dtype=np.int32)
    val = np.empty((len(rows), k), dtype=np.float32)
    for n, r in enumerate(rows):
        s = 0 if starts is None else int(starts[r])
        e = C if ends is None else int(ends[r])
        if not (0 <= s <= e <= C):
            raise ValueError(f"row {r}: invalid range [{s}, {e}) for {C} columns")
        idx[n], val[n] = topk_row(scores[r], s, e, k)
    return idx, val
