"""dsa_sparse_mla_attn (2-CTA tcgen05 sparse MLA) against the fp64 oracle, fed the same selections."""
import numpy as np
import pytest
import torch

import dsa_inputs as G
import oracle as O
from gpu_util import MAX_ABS, REL_L2, f64, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


def _random_selection(rng, T, S, k, pos0):
    """Ascending causal selections: all of 0..t when t + 1 <= k, else k distinct positions <= t."""
    idx = np.full((T, k), -1, dtype=np.int32)
    for r in range(T):
        t = min(pos0 + r, S - 1)
        if t + 1 <= k:
            idx[r, :t + 1] = np.arange(t + 1)
        else:
            idx[r] = np.sort(rng.choice(t + 1, size=k, replace=False))
    return idx


def _compare(dsa, q, c, idx, scale, rows=None):
    out, lse = dsa.dsa_sparse_mla_attn(q, c, torch.from_numpy(idx).cuda(), scale)
    assert dsa.dsa_get_device_status() == 0
    out, lse = f64(out), lse.cpu().numpy()
    qf = O.bf16_to_f64(q.view(torch.int16).cpu().numpy().view(np.uint16))
    cf = O.bf16_to_f64(c.view(torch.int16).cpu().numpy().view(np.uint16))
    rows = range(q.shape[0]) if rows is None else rows
    refs, gots = [], []
    for r in rows:
        sel = idx[r][idx[r] >= 0]
        u, l = O.attention_row(qf[r], cf[sel], scale, 512)
        refs.append(u)
        gots.append(out[r])
        assert np.allclose(lse[r], l, rtol=1e-4, atol=1e-3), f"lse row {r}"
    refs, gots = np.stack(refs), np.stack(gots)
    assert np.abs(gots - refs).max() <= MAX_ABS
    assert rel_l2(gots, refs) <= REL_L2
    return out


def test_tiny_heads_and_short_rows(dsa):
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    x = G.prefill_inputs(cfg, 21, device="cuda")
    idx = _random_selection(np.random.default_rng(21), cfg.L, cfg.L, cfg.k, 0)
    _compare(dsa, x["q"], x["c"], idx, cfg.scale)


def test_128_heads_k2048(dsa):
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    keys = G.prefill_keys(cfg, 22, device="cuda")
    rows = list(range(2040, 2040 + 12)) + [5000, 8191]
    qs = G.prefill_queries(cfg, 22, rows=rows, device="cuda")
    rng = np.random.default_rng(22)
    idx = np.concatenate([_random_selection(rng, 1, cfg.L, cfg.k, t) for t in rows])
    _compare(dsa, qs["q"], keys["c"], idx, cfg.scale)


def test_selection_order_and_padding_do_not_matter(dsa):
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    keys = G.prefill_keys(cfg, 23, device="cuda")
    qs = G.prefill_queries(cfg, 23, rows=[3000, 3001, 3002], device="cuda")
    rng = np.random.default_rng(23)
    idx = np.concatenate([_random_selection(rng, 1, cfg.L, cfg.k, 3000 + i) for i in range(3)])
    perm = idx.copy()
    for r in range(3):
        perm[r] = rng.permutation(perm[r])
    perm[2, :100] = -1          # fewer entries, -1 anywhere
    a = _compare(dsa, qs["q"], keys["c"], idx, cfg.scale)
    b = _compare(dsa, qs["q"], keys["c"], perm, cfg.scale)
    assert np.abs(a[:2] - b[:2]).max() <= 2 * MAX_ABS


@pytest.mark.parametrize("k", [192, 320, 640])
def test_k_ending_in_half_a_tile(dsa, k):
    # k a multiple of 64 but not of 128: a token's last 128-key tile holds 64 selection slots and 64 masked ones.
    # The rows straddle k, so tokens below it carry -1 padding as well; 160 tokens put two or three on every
    # cluster (token transitions in the score CTA's Q-chunk schedule).
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    keys = G.prefill_keys(cfg, 25, device="cuda")
    rows = list(range(k - 80, k + 80))
    qs = G.prefill_queries(cfg, 25, rows=rows, device="cuda")
    rng = np.random.default_rng(25 + k)
    idx = np.concatenate([_random_selection(rng, 1, cfg.L, k, t) for t in rows])
    _compare(dsa, qs["q"], keys["c"], idx, cfg.scale)


def test_rows_with_nothing_selected(dsa):
    # rows whose k entries are all padding attend to nothing: output 0 and lse -inf (the oracle's empty selection),
    # next to ordinary rows in the same launch; one row selects a single entry
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    x = G.prefill_inputs(cfg, 26, device="cuda")
    idx = _random_selection(np.random.default_rng(26), 6, cfg.L, cfg.k, 700)
    idx[1] = -1
    idx[4] = -1
    idx[5, 1:] = -1
    out = _compare(dsa, x["q"][700:706].contiguous(), x["c"], idx, cfg.scale)
    assert not np.abs(out[1]).any() and not np.abs(out[4]).any()


def test_bad_index_is_reported_and_skipped(dsa):
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    x = G.prefill_inputs(cfg, 24, device="cuda")
    idx = _random_selection(np.random.default_rng(24), 4, cfg.L, cfg.k, 500)
    bad = idx.copy()
    bad[0, 5] = cfg.L + 7       # out of range -> treated as -1
    bad[1, 9] = -5
    out, _ = dsa.dsa_sparse_mla_attn(x["q"][500:504].contiguous(), x["c"], torch.from_numpy(bad).cuda(), cfg.scale)
    assert dsa.dsa_get_device_status() == 6
    ok = idx.copy()
    ok[0, 5] = -1
    ok[1, 9] = -1
    ref, _ = dsa.dsa_sparse_mla_attn(x["q"][500:504].contiguous(), x["c"], torch.from_numpy(ok).cuda(), cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    assert torch.equal(out, ref)
