"""dsa_topk (radix select + ordered compaction) against the oracle's sort-based selection, bit-exact."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


def _check(dsa, scores: np.ndarray, k: int, row_len=None, pos0=0):
    rows, ld = scores.shape
    st = torch.from_numpy(scores.astype(np.float32)).cuda()
    rl = None if row_len is None else torch.tensor(row_len, dtype=torch.int32, device="cuda")
    got = dsa.dsa_topk(st, k, row_len=rl, pos0=pos0).cpu().numpy()
    assert dsa.dsa_get_device_status() == 0
    s32 = scores.astype(np.float32).astype(np.float64)
    for r in range(rows):
        n = row_len[r] if row_len is not None else min(ld, pos0 + r + 1)
        ref = O.topk_row(s32[r, :n], k)
        assert np.array_equal(got[r], ref), f"row {r} (n={n})"


def test_integer_scores_heavy_ties(dsa):
    rng = np.random.default_rng(0)
    sc = rng.integers(-2, 3, size=(40, 5000)).astype(np.float32)
    _check(dsa, sc, 128, row_len=[int(x) for x in rng.integers(1, 5001, size=40)])
    _check(dsa, sc, 2048, row_len=[int(x) for x in rng.integers(1, 5001, size=40)])


def test_all_equal_and_signed_zero(dsa):
    sc = np.zeros((6, 3000), dtype=np.float32)
    sc[1, ::2] = -0.0
    sc[2] = -0.0
    sc[3, 100:] = 1.0
    sc[4, :] = -np.inf
    sc[5, 7] = np.nan
    _check(dsa, sc, 128, row_len=[3000] * 6)
    _check(dsa, sc, 2048, row_len=[3000] * 6)


def test_causal_rows_and_short_rows(dsa):
    rng = np.random.default_rng(1)
    sc = rng.normal(size=(300, 2600)).astype(np.float32)
    _check(dsa, sc, 2048, pos0=2300)          # rows of length 2301 .. 2600
    _check(dsa, sc[:50], 128, pos0=0)          # rows of length 1 .. 50 (<= k) and beyond
    _check(dsa, sc[:5], 64, row_len=[0, 1, 63, 64, 65])


def test_long_gaussian_rows(dsa):
    rng = np.random.default_rng(2)
    sc = rng.normal(size=(4, 131072)).astype(np.float32)
    _check(dsa, sc, 2048, row_len=[131072, 131071, 100000, 2049])


def test_integer_index_scores(dsa):
    rng = np.random.default_rng(3)
    H_I, d_I, n = 64, 128, 20000
    qi = rng.integers(-7, 8, size=(4, H_I, d_I)).astype(np.float64)
    ki = rng.integers(-7, 8, size=(n, d_I)).astype(np.float64)
    w = rng.integers(-3, 4, size=(4, H_I)).astype(np.float64)
    sc = np.stack([O.indexer_scores_row(qi[r], w[r], ki) for r in range(4)])
    _check(dsa, sc, 2048, row_len=[n, n - 1, 5000, 2048])


def test_rows_sorted_by_score_take_the_fallback_path(dsa):
    """Ascending scores put every candidate in the last warps' segments, overflowing their shared-memory
    regions, so the kernel switches to the multi-pass select; results must not change."""
    n = 20000
    asc = np.arange(n, dtype=np.float32)
    desc = asc[::-1].copy()
    blocks = np.repeat(np.arange(n // 100, dtype=np.float32), 100)    # 100-long runs of equal scores
    _check(dsa, np.stack([asc, desc, blocks, -asc]), 2048, row_len=[n, n, n, n])


def test_long_rows_where_the_sample_misleads(dsa):
    """Rows of 16384+ keys first estimate a threshold from one eighth of the row (128-key blocks every 1024
    keys); rows whose sampled blocks are unrepresentative must still select exactly (the kernel falls back)."""
    rng = np.random.default_rng(4)
    n = 40000
    sampled = np.zeros(n, dtype=bool)
    for b in range(n // 1024):
        sampled[1024 * b: 1024 * b + 128] = True
    base = rng.normal(size=(5, n)).astype(np.float32)
    rows = base.copy()
    rows[0, sampled] += 10.0          # the sample sees only large scores
    rows[1, ~sampled] += 10.0         # the sample sees only small scores
    rows[2, rng.choice(np.flatnonzero(~sampled), 3000, replace=False)] = 50.0   # outliers outside the sample
    rows[3] = np.round(rows[3])       # heavy ties
    _check(dsa, rows, 2048, row_len=[n, n, n, n, n - 7])
    # the same rows, 150 of them: at least as many rows as SMs take the one-CTA-per-row kernel and its sampled path
    many = np.tile(rows, (30, 1))
    _check(dsa, many, 2048, row_len=[n, n, n, n, n - 7] * 30)
