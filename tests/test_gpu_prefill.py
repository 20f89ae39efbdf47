"""dsa_forward_prefill (indexer -> top-k -> sparse MLA) end to end against the fp64 oracle."""
import os

import numpy as np
import pytest
import torch

import dsa_inputs as G
from gpu_util import MAX_ABS, RECALL, REL_L2, f64, oracle_prefill, prefill_device, recall, rel_l2, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


def _forward(dsa, cfg, seed):
    x = prefill_device(cfg, seed)
    idx, out, lse = dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                            x["c"], cfg.k, cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    del x
    return idx.cpu().numpy(), out, lse


def _check_rows(cfg, seed, rows, idx, out, exact_idx):
    ref = oracle_prefill(cfg, seed, rows)
    got_out = f64(out[torch.as_tensor(rows, device=out.device)])
    recalls = []
    for r, t in enumerate(rows):
        if exact_idx or t + 1 <= cfg.k:
            assert np.array_equal(idx[t], ref["idx"][r]), f"row {t}"
        else:
            recalls.append(recall(idx[t], ref["idx"][r]))
    if recalls:
        assert np.mean(recalls) >= RECALL, f"mean recall {np.mean(recalls)}"
    assert np.abs(got_out - ref["out"]).max() <= MAX_ABS
    assert rel_l2(got_out, ref["out"]) <= REL_L2


def test_tiny_all_rows(dsa):
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    idx, out, lse = _forward(dsa, cfg, 31)
    rows = list(range(cfg.L))
    _check_rows(cfg, 31, rows, idx, out, exact_idx=True)


def test_8k_integer_mode(dsa):
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    idx, out, _ = _forward(dsa, cfg, 32)
    # every row: a valid, ascending, causal selection of the right size
    L, k = cfg.L, cfg.k
    for t in range(0, L, 97):
        v = idx[t][idx[t] >= 0]
        assert len(v) == min(k, t + 1) and (np.diff(v) > 0).all() and v.max() <= t
    _check_rows(cfg, 32, sample_rows(L, k, 24, 32), idx, out, exact_idx=True)


def test_32k_gaussian_mode(dsa):
    cfg = G.PREFILL_CONFIGS["prefill_32k"]
    idx, out, _ = _forward(dsa, cfg, 33)
    _check_rows(cfg, 33, sample_rows(cfg.L, cfg.k, 32, 33), idx, out, exact_idx=False)


@pytest.mark.parametrize("name", ["prefill_128k", "prefill_128k_gauss"])
def test_128k_sampled_rows(dsa, name):
    cfg = G.PREFILL_CONFIGS[name]
    idx, out, _ = _forward(dsa, cfg, 34)
    n = int(os.environ.get("DSA_ORACLE_ROWS_128K", "64"))
    rows = sample_rows(cfg.L, cfg.k, n, 34)
    _check_rows(cfg, 34, rows, idx, out, exact_idx=(cfg.mode == "int"))
