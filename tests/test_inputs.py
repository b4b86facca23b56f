"""The seeded input generators follow the stated recipe: bf16 round-to-nearest-even
(against torch's own conversion), block masks (diagonal kept, causal lower triangle,
keep probability), top-k index sets (distinct keys of [0, q], min(q + 1, topk) of them,
uniform over keys, random order, -1 tail) and packed causal ranges."""
import numpy as np
import torch

from index_sparse_attention_b200 import inputs as I


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1.0e-40, 1.00390625,
                                  1.01171875], np.float32)])  # the last two are bf16 ties
    ours = I.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(I.bf16_bits_to_f32(ours),
                                  torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_block_mask_recipe():
    w = I.scaled(I.WORKLOADS["long_causal_blocksparse_h16_s32768_d256"], HQ=2, HK=2,
                 Sq=128 * 200, Sk=128 * 200, density=0.1)
    m = I.block_mask(w).astype(bool)
    Mb = m.shape[2]
    assert m.shape == (1, 2, Mb, Mb)
    assert m[:, :, np.arange(Mb), np.arange(Mb)].all()          # diagonal kept
    assert not m[:, :, np.triu_indices(Mb, 1)[0], np.triu_indices(Mb, 1)[1]].any()  # causal
    lower = m[:, :, np.tril_indices(Mb, -1)[0], np.tril_indices(Mb, -1)[1]]
    assert abs(lower.mean() - 0.1) < 0.01                      # keep probability
    w2 = I.scaled(w, causal=False, density=0.5)
    m2 = I.block_mask(w2).astype(bool)
    off = ~np.eye(Mb, dtype=bool)
    assert m2[:, :, np.arange(Mb), np.arange(Mb)].all()
    assert abs(m2[:, :, off].mean() - 0.5) < 0.02               # upper blocks eligible too


def test_topk_index_recipe():
    w = I.scaled(I.WORKLOADS["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], B=2, Sq=300,
                 Sk=300, HQ=4, HK=2, topk=16)
    idx = I.topk_indices(w)
    assert idx.shape == (2, 300, 2, 16) and idx.dtype == np.int32
    counts = np.zeros(300)
    expect = np.zeros(300)
    sorted_rows = 0
    for b in range(2):
        for i in range(300):
            for g in range(2):
                row = idx[b, i, g]
                n = min(i + 1, 16)
                valid = row[:n]
                assert (row[n:] == -1).all()                    # -1 only at the tail
                assert len(set(valid.tolist())) == n            # distinct
                assert valid.min() >= 0 and valid.max() <= i    # keys of [0, q]
                counts[valid] += 1
                expect[:i + 1] += n / (i + 1)                   # uniform over [0, q]
                sorted_rows += n > 4 and bool((np.diff(valid) > 0).all())
    # uniform: each key's count close to its expectation (rows i >= 200 alone give every
    # key about 2*2*100*16/250 expected hits)
    assert np.abs(counts - expect).max() / expect.max() < 0.15
    assert sorted_rows < 5                                      # random order, not sorted


def test_packed_causal_ranges():
    s, e = I.packed_causal_ranges(10, segments=(4, 6))
    np.testing.assert_array_equal(s, [0, 0, 0, 0, 4, 4, 4, 4, 4, 4])
    np.testing.assert_array_equal(e, [1, 2, 3, 4, 5, 6, 7, 8, 9, 10])
    s, e = I.packed_causal_ranges(5)
    np.testing.assert_array_equal(s, np.zeros(5))
    np.testing.assert_array_equal(e, np.arange(1, 6))


def test_topk_score_distributions():
    x = I.topk_scores(64, 512, seed=1, dist="concentrated")
    assert x.dtype == np.float32 and x.shape == (64, 512)
    assert np.abs(x - 5.0).max() < 0.01
    assert all(len(np.unique(r)) < r.size for r in x)           # exact ties in every row
    assert len(np.unique(x)) < x.size // 3
    y = I.topk_scores(64, 512, seed=1)
    assert abs(float(y.mean())) < 0.05 and abs(float(y.std()) - 1.0) < 0.05


def test_topk_index_span_all_and_duplicates():
    """span "all": distinct keys of every position [0, Sk), above the diagonal too;
    dup > 0: repeated keys inside a row, drawn from that row's own set, -1 tail kept."""
    base = I.scaled(I.WORKLOADS["indexsparse_gqa_q16384_hq32_hk4_d192_128_top2048"], B=1,
                    Sq=300, Sk=260, HQ=2, HK=1, topk=40, span="all")
    idx = I.topk_indices(base)
    above = 0
    counts = np.zeros(260)
    for i in range(300):
        row = idx[0, i, 0]
        assert (row >= 0).all() and row.max() < 260            # k = min(Sk, topk) = 40
        assert len(set(row.tolist())) == 40                     # distinct
        above += int((row > i).sum())
        counts[row] += 1
    assert above > 40 * 40                                      # entries above the diagonal
    expect = 300 * 40 / 260                                     # per key; sd about 6.2
    assert np.abs(counts - expect).max() < 5 * np.sqrt(expect * (1 - 40 / 260))  # uniform
    dup = I.topk_indices(I.scaled(base, dup=0.3))
    assert dup.shape == idx.shape
    n_dup_rows = 0
    for i in range(300):
        row, ref = dup[0, i, 0], idx[0, i, 0]
        assert set(row.tolist()) <= set(ref.tolist())           # copies of the row's own keys
        n_dup_rows += len(set(row.tolist())) < 40
    assert n_dup_rows > 290                                     # almost every row repeats keys
    # the -1 tail survives duplication (topk > Sk: 260 keys then 40 pads)
    big = I.topk_indices(I.scaled(base, topk=300, dup=0.3))
    assert (big[0, :, 0, 260:] == -1).all() and (big[0, :, 0, :260] >= 0).all()
    # the default span and dup leave the causal recipe untouched
    causal = I.topk_indices(I.scaled(base, span="causal"))
    assert all(causal[0, i, 0][causal[0, i, 0] >= 0].max() <= i for i in range(300))
