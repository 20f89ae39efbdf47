"""The DSA_CHECKS build (libdsa_checks.so): on correct inputs it computes what libdsa.so computes, bit for bit,
with no check firing; each planted violation is caught."""
import dataclasses

import numpy as np
import pytest
import torch

import dsa_inputs as G
from gpu_util import prefill_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    assert not m.dsa_checks_enabled()
    yield m
    m.use_library(m.LIB_PATH)


def _both(dsa, fn):
    """fn() through libdsa.so, then through libdsa_checks.so (device status 0 after each)."""
    dsa.use_library(dsa.LIB_PATH)
    a = fn()
    assert dsa.dsa_get_device_status() == 0
    dsa.use_library(dsa.CHECKS_LIB_PATH)
    assert dsa.dsa_checks_enabled()
    b = fn()
    status = dsa.dsa_get_device_status()
    dsa.use_library(dsa.LIB_PATH)
    assert status == 0, f"a check fired: status {status}"
    return a, b


def _equal(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name,L", [("tiny_1k", 1024), ("prefill_8k", 3000), ("prefill_32k", 2600)])
def test_prefill_identical_and_clean(dsa, name, L):
    # integer mode with 4 and 64 indexer heads (a ragged last block), and Gaussian mode with per-token scales
    cfg = dataclasses.replace(G.PREFILL_CONFIGS[name], L=L)
    x = prefill_device(cfg, 61)
    a, b = _both(dsa, lambda: dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"],
                                                      x["q"], x["c"], cfg.k, cfg.scale))
    _equal(a, b)


def test_prefill_kl_identical_and_clean(dsa):
    # the attention's KL mode (every CTA on tokens of its own) and the selected scores of the top-k
    cfg = dataclasses.replace(G.PREFILL_CONFIGS["prefill_8k"], L=2300)
    x = prefill_device(cfg, 67)
    a, b = _both(dsa, lambda: dsa.dsa_forward_prefill_kl(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"],
                                                         x["w"], x["q"], x["c"], cfg.k, cfg.scale))
    _equal(a, b)


def test_varlen_identical_and_clean(dsa):
    base = G.PREFILL_CONFIGS["prefill_8k"]
    lens, seeds = [700, 0, 2500, 2100], [62, 0, 63, 64]
    cfgs = [dataclasses.replace(base, L=max(n, 1)) for n in lens]
    parts = [prefill_device(cfg, sd) for cfg, sd, n in zip(cfgs, seeds, lens) if n]
    cat = {key: torch.cat([p[key] for p in parts]) for key in ("q_idx", "k_idx", "w", "q", "c")}
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    a, b = _both(dsa, lambda: dsa.dsa_forward_prefill_varlen(cu, cat["q_idx"], None, cat["k_idx"], None, cat["w"],
                                                             cat["q"], cat["c"], base.k, base.scale))
    _equal(a, b)


def test_decode_identical_and_clean(dsa):
    # three steps of a small batch (contexts 100..20000): the cluster top-k, the decode indexer's flat work list
    # and the attention's per-token key counts, the caches appended every step
    cfg = G.DecodeConfig("checks", B=6, len_lo=100, len_hi=20000, steps=3)
    runs = []
    for lib in ("LIB_PATH", "CHECKS_LIB_PATH"):
        dsa.use_library(getattr(dsa, lib))
        cache = G.decode_fill_cache(cfg, 65, device="cuda")
        cache_off = torch.tensor(cache["offs"], dtype=torch.int64, device="cuda")
        ctx = torch.tensor(cache["lens"], dtype=torch.int32, device="cuda")
        outs = []
        for step in range(cfg.steps):
            st = G.decode_step_inputs(cfg, 65, step, device="cuda")
            outs.append(dsa.dsa_forward_decode(cache_off, ctx, st["q_idx"], st["q_scale"], st["w"], st["q"],
                                               st["k_new"], st["k_scale_new"], st["c_new"], cache["k_cache"],
                                               cache["k_scale_cache"], cache["c_cache"], cfg.k, cfg.scale))
            ctx += 1
        assert dsa.dsa_get_device_status() == 0, lib
        runs.append(outs)
    dsa.use_library(dsa.LIB_PATH)
    for a, b in zip(*runs):
        _equal(a, b)


def test_topk_rows_identical_and_clean(dsa):
    # the one-CTA-per-row kernel on heavy ties and short rows (row_len), and the cluster kernel (fewer rows than SMs)
    g = torch.Generator(device="cuda").manual_seed(66)
    for rows, n in ((300, 40000), (20, 100000)):
        s = torch.randint(-50, 50, (rows, n), generator=g, device="cuda").float()
        ln = torch.randint(1, n + 1, (rows,), generator=g, device="cuda").int()
        a, b = _both(dsa, lambda: (dsa.dsa_topk(s, 2048, row_len=ln),))
        _equal(a, b)


def test_planted_violations_are_caught(dsa):
    dsa.use_library(dsa.CHECKS_LIB_PATH)
    try:
        assert dsa.dsa_checks_selftest(0) == 8       # DSA_ERR_CHECK: a top-k row out of order
        assert dsa.dsa_checks_selftest(1) == 6       # DSA_ERR_BAD_INDEX: a selected entry beyond its token's keys
        assert dsa.dsa_get_device_status() == 0      # read and cleared
    finally:
        dsa.use_library(dsa.LIB_PATH)
    with pytest.raises(dsa.DsaError):                # the normal build has no checks to plant into
        dsa.dsa_checks_selftest(0)
