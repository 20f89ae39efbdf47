"""The indexer's training objective on the GPU (dsa_forward_prefill_kl, dsa_indexer_kl) against the oracle's
indexer_kl_row: kl[t] = KL(p_t || Softmax(I_t)) over each row's selected entries, p_t the heads' attention
probabilities summed and L1-normalised (velog.io page, Stage 1 Dense Warm-up).

Tolerance.  The GPU forms p from fp32 logits of bf16 inputs and the attention's fp32 lse (about 1e-6 relative per
probability), and sums a log a, a I and the log-sum-exp of I in fp32.  The error of the sum of a I scales with the
size of the index scores, so the bound is 2e-3 + 1e-5 (|kl| + max |I|) nats."""
import dataclasses

import numpy as np
import pytest
import torch

import dsa_inputs as G
import oracle as O
from gpu_util import prefill_device, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


def _tol(kl, imax):
    return 2e-3 + 1e-5 * (abs(kl) + imax)


def _oracle_kl(cfg, seed, rows, idx):
    """The oracle's objective of each row over the given selected entries (index scores recomputed in fp64)."""
    keys = G.prefill_keys(cfg, seed)
    qs = G.prefill_queries(cfg, seed, rows=rows)
    kI = O.e4m3_to_f64(keys["k_idx"].view(torch.uint8).numpy())
    if keys["k_scale"] is not None:
        kI = kI * keys["k_scale"].numpy().astype(np.float64)[:, None]
    qI = O.e4m3_to_f64(qs["q_idx"].view(torch.uint8).numpy())
    if qs["q_scale"] is not None:
        qI = qI * qs["q_scale"].numpy().astype(np.float64)[:, None, None]
    w = qs["w"].numpy().astype(np.float64)
    c = O.bf16_to_f64(keys["c"].view(torch.int16).numpy().view(np.uint16))
    q = O.bf16_to_f64(qs["q"].view(torch.int16).numpy().view(np.uint16))
    out = []
    for r, t in enumerate(rows):
        sel = idx[r][idx[r] >= 0]
        I = O.indexer_scores_row(qI[r], w[r], kI[sel])
        out.append((O.indexer_kl_row(I, q[r], c[sel], cfg.scale), float(np.abs(I).max()) if len(I) else 0.0))
    return out


@pytest.mark.parametrize("name,L,k,seed", [("tiny_1k", 1024, None, 71), ("prefill_8k", 3000, None, 72),
                                            ("prefill_8k", 1500, 320, 73), ("prefill_8k", 1800, None, 74)])
def test_prefill_kl_integer_mode(dsa, name, L, k, seed):
    # k = 320 ends in half a 128-key tile: the objective's masks skip the padded half.  L = 1800 <= k: every row
    # selects all of 0..t, and the objective still needs the index scores of those keys.
    cfg = dataclasses.replace(G.PREFILL_CONFIGS[name], L=L)
    if k is not None:
        cfg = dataclasses.replace(cfg, k=k)
    x = prefill_device(cfg, seed)
    idx, out, lse, kl = dsa.dsa_forward_prefill_kl(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                                   x["c"], cfg.k, cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    # the forward part equals dsa_forward_prefill's
    i2, o2, l2 = dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"], x["c"],
                                         cfg.k, cfg.scale)
    assert torch.equal(idx, i2) and torch.equal(out, o2) and torch.equal(lse, l2)
    rows = sample_rows(L, cfg.k, 40, seed)
    idx_h, kl_h = idx.cpu().numpy(), kl.cpu().numpy()
    for (ref, imax), t in zip(_oracle_kl(cfg, seed, rows, idx_h[rows]), rows):
        assert abs(kl_h[t] - ref) <= _tol(ref, imax), f"row {t}: {kl_h[t]} vs {ref}"
    assert kl_h[0] == pytest.approx(0.0, abs=1e-6)        # one key: both distributions are that key


def test_prefill_kl_gaussian_mode(dsa):
    cfg = dataclasses.replace(G.PREFILL_CONFIGS["prefill_32k"], L=6000)
    seed = 73
    x = prefill_device(cfg, seed)
    idx, _, _, kl = dsa.dsa_forward_prefill_kl(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                               x["c"], cfg.k, cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    rows = sample_rows(cfg.L, cfg.k, 30, seed)
    idx_h, kl_h = idx.cpu().numpy(), kl.cpu().numpy()
    assert (kl_h >= -1e-3).all()
    for (ref, imax), t in zip(_oracle_kl(cfg, seed, rows, idx_h[rows]), rows):
        assert abs(kl_h[t] - ref) <= _tol(ref, imax), f"row {t}: {kl_h[t]} vs {ref}"


def test_indexer_kl_on_given_selections(dsa):
    # random selections (unsorted, with padding) and arbitrary index scores through dsa_indexer_kl
    cfg = G.PREFILL_CONFIGS["prefill_8k"]
    keys = G.prefill_keys(cfg, 74, device="cuda")
    T = 40
    qs = G.prefill_queries(cfg, 74, rows=range(cfg.L - T, cfg.L), device="cuda")
    rng = np.random.default_rng(74)
    idx = np.full((T, cfg.k), -1, dtype=np.int32)
    for r in range(T):
        m = int(rng.integers(1, cfg.k + 1))
        idx[r, :m] = rng.permutation(rng.choice(cfg.L, size=m, replace=False))
    sel = rng.standard_normal((T, cfg.k)).astype(np.float32) * 4
    idx_d = torch.from_numpy(idx).cuda()
    _, lse = dsa.dsa_sparse_mla_attn(qs["q"], keys["c"], idx_d, cfg.scale)
    kl = dsa.dsa_indexer_kl(qs["q"], keys["c"], idx_d, torch.from_numpy(sel).cuda(), lse, cfg.scale).cpu().numpy()
    assert dsa.dsa_get_device_status() == 0
    c = O.bf16_to_f64(keys["c"].cpu().view(torch.int16).numpy().view(np.uint16))
    q = O.bf16_to_f64(qs["q"].cpu().view(torch.int16).numpy().view(np.uint16))
    for r in range(T):
        m = idx[r] >= 0
        ref = O.indexer_kl_row(sel[r][m].astype(np.float64), q[r], c[idx[r][m]], cfg.scale)
        assert abs(kl[r] - ref) <= _tol(ref, float(np.abs(sel[r][m]).max())), f"row {r}"
