"""Seeded synthetic workloads for block-sparse / index-sparse attention.

This module holds the workload definitions and random draws only; it contains none
of the attention arithmetic and is shared by the tests, the benchmark and the CPU
oracle's callers so that both sides see the same bytes.

Draws: for workload seed base ``s``, q, k, v and dO come from
``numpy.random.default_rng(s + 0..3).standard_normal(float32)`` rounded to bf16
(round to nearest even), and the block mask or the top-k indices come from
``default_rng(s + 4)``.

Structures (the workloads the pages and the benchmark are about):
  * block mask [B, HK, Mb, Nb] (uint8) at block size ``bs``: each eligible block is
    kept with probability ``density``; diagonal blocks are always kept; with
    ``causal`` only the lower triangle is eligible.
  * index mode: per (query, KV head), ``topk`` distinct int32 key positions drawn
    uniformly from the causal range [0, q] (``span="causal"``) or from every key
    [0, Sk) (``span="all"``: entries above the diagonal, which a causal call must mask
    and a non-causal call must attend), stored in random order, with -1 padding at the
    tail when fewer than ``topk`` are valid.  With ``dup`` > 0 each filled slot is,
    with that probability, overwritten by a copy of a random slot of its own row, so
    rows hold repeated keys (the attended set is still the row's set of keys).  This is the int32 / -1 output
    format of the Top-K selector in xtuner PR #2096 ("Add optional TileLang Top-K
    selector", Main Changes 1) that feeds IndexSparse attention (MagiAttention
    PR #334, section 2).
"""
from dataclasses import dataclass, field, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Sq: int
    Sk: int
    HQ: int
    HK: int
    Dqk: int
    Dv: int
    mode: str  # "block" | "index"
    causal: bool
    bs: int = 128  # block-mask granularity (block mode)
    density: float = 1.0  # keep probability of an eligible off-diagonal block
    topk: int = 0  # index mode
    span: str = "causal"  # index mode: keys drawn from [0, q] ("causal") or [0, Sk) ("all")
    dup: float = 0.0  # index mode: probability that a slot repeats another key of its row
    seed: int = 0
    tags: tuple = field(default_factory=tuple)

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.Dqk))


# The five benchmark workloads.  Seed base = 1000 * workload number.
WORKLOADS = {
    "blocksparse_mha_s256_d64": Workload(
        "blocksparse_mha_s256_d64", B=1, Sq=256, Sk=256, HQ=2, HK=2, Dqk=64, Dv=64,
        mode="block", causal=False, bs=64, density=0.5, seed=1000),
    "dense_full_b2_h16_s4096_d128": Workload(
        "dense_full_b2_h16_s4096_d128", B=2, Sq=4096, Sk=4096, HQ=16, HK=16, Dqk=128, Dv=128,
        mode="block", causal=False, bs=128, density=1.0, seed=2000),
    "dense_causal_b2_h16_s4096_d128": Workload(
        "dense_causal_b2_h16_s4096_d128", B=2, Sq=4096, Sk=4096, HQ=16, HK=16, Dqk=128,
        Dv=128, mode="block", causal=True, bs=128, density=1.0, seed=2000),
    "gqa_blocksparse_b2_hq32_hk8_s8192_d128": Workload(
        "gqa_blocksparse_b2_hq32_hk8_s8192_d128", B=2, Sq=8192, Sk=8192, HQ=32, HK=8,
        Dqk=128, Dv=128, mode="block", causal=True, bs=128, density=0.25, seed=3000),
    "indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048": Workload(
        "indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048", B=1, Sq=16384, Sk=16384, HQ=32,
        HK=4, Dqk=192, Dv=128, mode="index", causal=True, topk=2048, seed=4000),
    "long_causal_blocksparse_h16_s32768_d256": Workload(
        "long_causal_blocksparse_h16_s32768_d256", B=1, Sq=32768, Sk=32768, HQ=16, HK=16,
        Dqk=256, Dv=256, mode="block", causal=True, bs=128, density=0.1, seed=5000),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (smaller shapes for parity tests)."""
    return replace(w, **kw)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) and return the raw uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, shape) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def block_mask(w: Workload) -> np.ndarray:
    """uint8 [B, HK, Mb, Nb] at granularity w.bs."""
    Mb, Nb = -(-w.Sq // w.bs), -(-w.Sk // w.bs)
    rng = np.random.default_rng(w.seed + 4)
    u = rng.random((w.B, w.HK, Mb, Nb))
    keep = u < w.density
    mi = np.arange(Mb)[:, None]
    ni = np.arange(Nb)[None, :]
    if w.causal:
        keep &= (ni < mi)[None, None]
    keep |= (ni == mi)[None, None]
    return keep.astype(np.uint8)


def topk_indices(w: Workload, rows_per_chunk: int = 4096) -> np.ndarray:
    """int32 [B, Sq, HK, topk]: distinct keys drawn uniformly from [0, q] (or [0, Sk)
    with span "all"), -1 padded, optionally with repeated entries (``dup``).

    Each (query, KV head) row with n = min(q, Sk-1) + 1 candidates (n = Sk with span
    "all") draws
    k = min(n, topk) of them by R. W. Floyd's sampling algorithm (step s: draw t
    uniformly from [0, n-k+s]; take t unless already taken, else take n-k+s), which
    yields every k-subset with equal probability; the k entries are then put in a
    uniformly random order and -1 fills the rest of the row.  The rows of a chunk
    advance together, one Floyd step per iteration.
    """
    rng = np.random.default_rng(w.seed + 4)
    out = np.full((w.B, w.Sq, w.HK, w.topk), -1, dtype=np.int32)
    if w.span == "causal":
        n_all = np.repeat(np.minimum(np.arange(w.Sq), w.Sk - 1) + 1, w.HK).astype(np.int64)
    elif w.span == "all":
        n_all = np.full(w.Sq * w.HK, w.Sk, dtype=np.int64)
    else:
        raise ValueError(f"span must be 'causal' or 'all', got {w.span!r}")
    for b in range(w.B):
        sel_b = out[b].reshape(-1, w.topk)
        for r0 in range(0, len(n_all), rows_per_chunk):
            n = n_all[r0:r0 + rows_per_chunk]
            k = np.minimum(n, w.topk)
            rows = len(n)
            taken = np.zeros((rows, (w.Sk + 7) // 8), dtype=np.uint8)  # packed membership bits
            sel = np.full((rows, w.topk), -1, dtype=np.int32)
            ar = np.arange(rows)
            for s in range(int(k.max())):
                act = ar[s < k] if s >= int(k.min()) else ar
                j = n[act] - k[act] + s
                t = rng.integers(0, j + 1)
                present = (taken[act, t >> 3] >> (t & 7).astype(np.uint8)) & 1
                c = np.where(present == 1, j, t)
                taken[act, c >> 3] |= (np.uint8(1) << (c & 7).astype(np.uint8))
                sel[act, s] = c
            full = k == w.topk
            sel[full] = rng.permuted(sel[full], axis=1)
            for r in np.nonzero(~full)[0]:
                sel[r, :k[r]] = rng.permutation(sel[r, :k[r]])
            sel_b[r0:r0 + rows] = sel
    if w.dup > 0:
        flat = out.reshape(-1, w.topk)
        filled = np.count_nonzero(flat >= 0, axis=1)
        slot = np.arange(w.topk)[None, :]
        over = (rng.random(flat.shape) < w.dup) & (slot < filled[:, None])
        src = np.minimum((rng.random(flat.shape) * filled[:, None]).astype(np.int64),
                         np.maximum(filled[:, None] - 1, 0))
        flat[over] = np.take_along_axis(flat, src, axis=1)[over]
    return out


@dataclass
class Inputs:
    w: Workload
    q: np.ndarray  # uint16 bf16 bits [B, Sq, HQ, Dqk]
    k: np.ndarray  # [B, Sk, HK, Dqk]
    v: np.ndarray  # [B, Sk, HK, Dv]
    do: np.ndarray  # [B, Sq, HQ, Dv]
    mask: np.ndarray = None  # block mode
    idx: np.ndarray = None  # index mode

    def f32(self, name: str) -> np.ndarray:
        return bf16_bits_to_f32(getattr(self, name))


def make_inputs(w: Workload, with_grad: bool = True) -> Inputs:
    q = normal_bf16(w.seed + 0, (w.B, w.Sq, w.HQ, w.Dqk))
    k = normal_bf16(w.seed + 1, (w.B, w.Sk, w.HK, w.Dqk))
    v = normal_bf16(w.seed + 2, (w.B, w.Sk, w.HK, w.Dv))
    do = normal_bf16(w.seed + 3, (w.B, w.Sq, w.HQ, w.Dv)) if with_grad else None
    mask = block_mask(w) if w.mode == "block" else None
    idx = topk_indices(w) if w.mode == "index" else None
    return Inputs(w, q, k, v, do, mask, idx)


# ---------------------------------------------------------------------------------
# Top-k selector inputs: fp32 indexer scores of one packed sequence
# ---------------------------------------------------------------------------------
def packed_causal_ranges(L, segments=None):
    """Per-row valid key ranges [start, end) of a packed causal sequence of length L
    made of the given segment lengths (one segment by default): row i of a segment
    [s, e) may attend to [s, i + 1)."""
    segments = (L,) if segments is None else tuple(segments)
    assert sum(segments) == L
    starts = np.empty(L, np.int32)
    ends = np.empty(L, np.int32)
    s0 = 0
    for n in segments:
        starts[s0:s0 + n] = s0
        ends[s0:s0 + n] = np.arange(s0 + 1, s0 + n + 1, dtype=np.int32)
        s0 += n
    return starts, ends


def topk_scores(rows, cols, seed, dist="normal"):
    """fp32 scores [rows, cols]: ``normal`` -- standard normal draws; ``concentrated``
    -- 5 + 1e-3 * standard normal, all in one narrow band that shares its leading radix
    digits, with many exact ties after rounding to fp32."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, cols), dtype=np.float32)
    if dist == "concentrated":
        x = (np.float32(5.0) + np.float32(1e-3) * x).astype(np.float32)
    elif dist != "normal":
        raise ValueError(dist)
    return x

