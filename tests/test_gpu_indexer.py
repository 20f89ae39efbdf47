"""dsa_indexer_scores (tcgen05 FP8 lightning indexer) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import dsa_inputs as G
import oracle as O
from gpu_util import oracle_prefill, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


def _run(dsa, cfg, seed, pos0=0, T=None, S=None):
    keys = G.prefill_keys(cfg, seed, device="cuda")
    qs = G.prefill_queries(cfg, seed, None, device="cuda", with_q=False)
    T = cfg.L if T is None else T
    S = cfg.L if S is None else S
    k_idx = keys["k_idx"][:S].contiguous()
    k_scale = None if keys["k_scale"] is None else keys["k_scale"][:S].contiguous()
    q_idx = qs["q_idx"][pos0:pos0 + T].contiguous()
    q_scale = None if qs["q_scale"] is None else qs["q_scale"][pos0:pos0 + T].contiguous()
    w = qs["w"][pos0:pos0 + T].contiguous()
    sc = dsa.dsa_indexer_scores(q_idx, q_scale, k_idx, k_scale, w, pos0=pos0)
    assert dsa.dsa_get_device_status() == 0
    return sc.cpu().numpy()


def _check_exact(sc, ref_rows, rows, pos0, S):
    for r, t in enumerate(rows):
        ref = ref_rows[r]
        got = sc[t - pos0]
        n = min(t + 1, S)
        assert np.array_equal(got[:n].astype(np.float64), ref[:n]), f"row {t}"
        assert np.isneginf(got[n:]).all(), f"row {t}: causal mask"


def test_tiny_all_rows_bit_exact(dsa):
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    sc = _run(dsa, cfg, 11)
    rows = list(range(cfg.L))
    ref = oracle_prefill(cfg, 11, rows, want_attention=False, want_scores=True)["scores"]
    _check_exact(sc, ref, rows, 0, cfg.L)


def test_8k_sampled_rows_bit_exact(dsa):
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    sc = _run(dsa, cfg, 12)
    rows = sample_rows(cfg.L, cfg.k, 24, 12)
    ref = oracle_prefill(cfg, 12, rows, want_attention=False, want_scores=True)["scores"]
    _check_exact(sc, ref, rows, 0, cfg.L)
    assert np.abs(sc[np.isfinite(sc)]).max() < 2 ** 24


@pytest.mark.parametrize("pos0,T,S", [(1000, 37, 1100), (129, 5, 300), (0, 1, 1), (4000, 300, 4250)])
def test_ragged_row_and_key_ranges(dsa, pos0, T, S):
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    sc = _run(dsa, cfg, 13, pos0=pos0, T=T, S=S)
    assert sc.shape == (T, S)
    keys = G.prefill_keys(cfg, 13)
    rows = list(range(pos0, pos0 + T))
    qs = G.prefill_queries(cfg, 13, rows=rows, with_q=False)
    kI = O.e4m3_to_f64(keys["k_idx"].view(torch.uint8).numpy()[:S])
    qI = O.e4m3_to_f64(qs["q_idx"].view(torch.uint8).numpy())
    w = qs["w"].numpy().astype(np.float64)
    for r, t in enumerate(rows):
        n = min(t + 1, S)
        ref = O.indexer_scores_row(qI[r], w[r], kI[:n])
        assert np.array_equal(sc[r, :n].astype(np.float64), ref)
        assert np.isneginf(sc[r, n:]).all()


def test_tiny_gaussian_mode_close(dsa):
    cfg = G.PrefillConfig("tiny_gauss", L=1024, H_I=4, d_I=64, k=128, H=8, mode="gauss")
    sc = _run(dsa, cfg, 14)
    rows = list(range(0, cfg.L, 7))
    ref = oracle_prefill(cfg, 14, rows, want_attention=False, want_scores=True)["scores"]
    for r, t in enumerate(rows):
        got = sc[t, :t + 1].astype(np.float64)
        scale = max(np.abs(ref[r]).max(), 1e-30)
        assert np.abs(got - ref[r]).max() <= 1e-5 * scale


def test_gaussian_mode_64_heads_close(dsa):
    cfg = G.PREFILL_CONFIGS["prefill_32k"]
    T, S, pos0 = 64, 3000, 2900
    sc = _run(dsa, cfg, 15, pos0=pos0, T=T, S=S)
    rows = list(range(pos0, pos0 + T))
    keys = G.prefill_keys(cfg, 15)
    keys = {"k_idx": keys["k_idx"][:S], "k_scale": keys["k_scale"][:S], "c": keys["c"][:S]}
    qs = G.prefill_queries(cfg, 15, rows=rows, with_q=False)
    ref = O.prefill_rows(keys, qs, rows, cfg.k, cfg.scale, want_scores=True, want_attention=False)["scores"]
    for r, t in enumerate(rows):
        n = min(t + 1, S)
        scale = max(np.abs(ref[r]).max(), 1e-30)
        assert np.abs(sc[r, :n].astype(np.float64) - ref[r][:n]).max() <= 1e-5 * scale
