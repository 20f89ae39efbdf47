"""dsa_forward_prefill (indexer -> top-k -> sparse MLA) end to end against the fp64 oracle."""
import dataclasses
import os

import numpy as np
import pytest
import torch

import dsa_inputs as G
import oracle as O
from gpu_util import (MAX_ABS, RECALL, REL_L2, e2e_bound, f64, oracle_prefill, prefill_device, recall, rel_l2,
                      sample_rows)

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
    """Integer mode: the selections equal the oracle's and the outputs are within tolerance of the oracle's.
    Gaussian mode: the selections reach the recall bar, and the outputs are within tolerance of the oracle's
    attention over the selection the GPU made (a swapped borderline key carries an attention weight that has
    nothing to do with its index score, so the output error of a different selection is bounded by recall,
    not by the attention tolerance); the end-to-end relative-L2 against the oracle's own selection stays within
    the bound that the measured recall implies (gpu_util.e2e_bound)."""
    ref = oracle_prefill(cfg, seed, rows)
    got_out = f64(out[torch.as_tensor(rows, device=out.device)])
    recalls = []
    for r, t in enumerate(rows):
        if exact_idx or t + 1 <= cfg.k:
            assert np.array_equal(idx[t], ref["idx"][r]), f"row {t}"
        else:
            recalls.append(recall(idx[t], ref["idx"][r]))
    if exact_idx:
        assert np.abs(got_out - ref["out"]).max() <= MAX_ABS
        assert rel_l2(got_out, ref["out"]) <= REL_L2
        return
    assert np.mean(recalls) >= RECALL, f"mean recall {np.mean(recalls)}"
    keys = G.prefill_keys(cfg, seed)
    qs = G.prefill_queries(cfg, seed, rows=rows)
    c = O.bf16_to_f64(keys["c"].view(torch.int16).numpy().view(np.uint16))
    q = O.bf16_to_f64(qs["q"].view(torch.int16).numpy().view(np.uint16))
    att = np.stack([O.attention_row(q[r], c[idx[t][idx[t] >= 0]], cfg.scale, cfg.D_v)[0]
                    for r, t in enumerate(rows)])
    assert np.abs(got_out - att).max() <= MAX_ABS
    assert rel_l2(got_out, att) <= REL_L2
    e2e = rel_l2(got_out, ref["out"])
    print(f"end-to-end rel-L2 vs the oracle's own selection: {e2e:.2e}, mean recall {np.mean(recalls):.5f}, "
          f"bound {e2e_bound(np.mean(recalls)):.2e}")
    assert e2e <= e2e_bound(np.mean(recalls)), f"end-to-end rel-L2 {e2e} at recall {np.mean(recalls)}"


def test_tiny_all_rows(dsa):
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    idx, out, lse = _forward(dsa, cfg, 31)
    rows = list(range(cfg.L))
    _check_rows(cfg, 31, rows, idx, out, exact_idx=True)


def test_k_ending_in_half_a_tile_end_to_end(dsa):
    # k = 320: dense rows t + 1 <= 320 run ceil((t + 1) / 128) tiles, gathered rows three tiles, the last half
    # masked; integer mode, so the selections are exact
    cfg = dataclasses.replace(G.PREFILL_CONFIGS["prefill_8k"], L=1500, k=320)
    idx, out, _ = _forward(dsa, cfg, 35)
    rows = sorted(set(list(range(0, 1500, 23)) + [127, 128, 255, 256, 318, 319, 320, 321, 383, 384, 1499]))
    _check_rows(cfg, 35, rows, idx, out, exact_idx=True)


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
    # 512 seeded random query rows (plus the edge rows) are checked against the oracle
    n = int(os.environ.get("DSA_ORACLE_ROWS_128K", "512"))
    rows = sample_rows(cfg.L, cfg.k, n, 34)
    _check_rows(cfg, 34, rows, idx, out, exact_idx=(cfg.mode == "int"))


def test_short_prefill_takes_the_implied_selection(dsa):
    # With L <= k every row t selects all of 0..t, whatever the scores: the select writes that selection without
    # launching the indexer (one top-k and one attention launch in all), and the outputs match the oracle.
    cfg = G.PrefillConfig("short_1500", L=1500, H_I=64, d_I=128, k=2048, H=128)
    n0 = dsa.dsa_launch_count()
    idx, out, _ = _forward(dsa, cfg, 35)
    assert dsa.dsa_launch_count() - n0 == 2
    for t in (0, 1, 777, cfg.L - 1):
        assert np.array_equal(idx[t], np.r_[np.arange(t + 1), -np.ones(cfg.k - t - 1, dtype=np.int64)])
    _check_rows(cfg, 35, sample_rows(cfg.L, cfg.k, 16, 35), idx, out, exact_idx=True)


def test_varlen_batch_matches_each_sequence_alone(dsa):
    # Three causal sequences packed one after another, with an empty one among them: each row's selection,
    # output and LSE equal those of its sequence run alone through dsa_forward_prefill (bit for bit), and the
    # longest sequence matches the oracle on sampled rows.
    base = G.PREFILL_CONFIGS["prefill_8k"]       # integer mode, H_I = 64, d_I = 128, k = 2048, H = 128
    lens, seeds = [700, 0, 2500, 1300], [36, 0, 37, 38]
    cfgs = [dataclasses.replace(base, name=f"varlen_{n}", L=n) for n in lens]
    parts = [prefill_device(cfg, sd) for cfg, sd, n in zip(cfgs, seeds, lens) if n]
    cat = {key: torch.cat([x[key] for x in parts]) for key in ("q_idx", "k_idx", "w", "q", "c")}
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    n0 = dsa.dsa_launch_count()
    idx, out, lse = dsa.dsa_forward_prefill_varlen(cu, cat["q_idx"], None, cat["k_idx"], None, cat["w"], cat["q"],
                                                   cat["c"], base.k, base.scale)
    assert dsa.dsa_get_device_status() == 0
    # the batch is one group: the attention's row offsets, one indexer launch over the scored rows (t >= k) of every
    # sequence, the top-k's row offsets and lengths, one top-k launch over every row, one attention launch
    assert dsa.dsa_launch_count() - n0 == 5
    for b, (cfg, sd, n) in enumerate(zip(cfgs, seeds, lens)):
        if not n:
            continue
        r0, r1 = cu[b], cu[b + 1]
        i1, o1, l1 = _forward_full(dsa, cfg, sd)
        assert torch.equal(idx[r0:r1], i1), f"sequence {b}: selection"
        assert torch.equal(out[r0:r1], o1), f"sequence {b}: output"
        assert torch.equal(lse[r0:r1], l1), f"sequence {b}: lse"
    cfg, sd = cfgs[2], seeds[2]
    _check_rows(cfg, sd, sample_rows(cfg.L, cfg.k, 12, sd), idx[cu[2]:cu[3]].cpu().numpy(), out[cu[2]:cu[3]],
                exact_idx=True)


def _forward_full(dsa, cfg, seed):
    x = prefill_device(cfg, seed)
    idx, out, lse = dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                            x["c"], cfg.k, cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    return idx, out, lse


def test_varlen_many_sequences_one_select(dsa):
    # 24 sequences of 100..3000 tokens (integer mode, k = 2048): every sequence's rows match its own prefill bit for
    # bit, while the select of the whole batch is one indexer launch and one top-k launch
    base = G.PREFILL_CONFIGS["prefill_8k"]
    rng = np.random.default_rng(39)
    lens = [int(x) for x in rng.integers(100, 3001, size=24)]
    lens[5] = 0
    seeds = [100 + b for b in range(len(lens))]
    cfgs = [dataclasses.replace(base, name=f"varlen_{n}", L=max(n, 1)) for n in lens]
    parts = [prefill_device(cfg, sd) for cfg, sd, n in zip(cfgs, seeds, lens) if n]
    cat = {key: torch.cat([x[key] for x in parts]) for key in ("q_idx", "k_idx", "w", "q", "c")}
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    n0 = dsa.dsa_launch_count()
    idx, out, lse = dsa.dsa_forward_prefill_varlen(cu, cat["q_idx"], None, cat["k_idx"], None, cat["w"], cat["q"],
                                                   cat["c"], base.k, base.scale)
    assert dsa.dsa_get_device_status() == 0
    assert dsa.dsa_launch_count() - n0 == 5
    for b, (cfg, sd, n) in enumerate(zip(cfgs, seeds, lens)):
        if not n:
            continue
        i1, o1, l1 = _forward_full(dsa, cfg, sd)
        r0, r1 = cu[b], cu[b + 1]
        assert torch.equal(idx[r0:r1], i1), f"sequence {b}: selection"
        assert torch.equal(out[r0:r1], o1), f"sequence {b}: output"
        assert torch.equal(lse[r0:r1], l1), f"sequence {b}: lse"


def test_varlen_sequences_around_k(dsa):
    # sequences of k - 1, k, k + 1 and 1 tokens (and k + 129, one key tile more): the first take no indexer launch at
    # all, the longer ones score only their rows t >= k; every row matches its sequence's own prefill bit for bit
    base = G.PREFILL_CONFIGS["prefill_8k"]
    k = base.k
    lens = [k - 1, k, k + 1, 1, k + 129]
    seeds = [70 + b for b in range(len(lens))]
    cfgs = [dataclasses.replace(base, name=f"varlen_{n}", L=n) for n in lens]
    parts = [prefill_device(cfg, sd) for cfg, sd in zip(cfgs, seeds)]
    cat = {key: torch.cat([x[key] for x in parts]) for key in ("q_idx", "k_idx", "w", "q", "c")}
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    idx, out, lse = dsa.dsa_forward_prefill_varlen(cu, cat["q_idx"], None, cat["k_idx"], None, cat["w"], cat["q"],
                                                   cat["c"], k, base.scale)
    assert dsa.dsa_get_device_status() == 0
    for b, (cfg, sd) in enumerate(zip(cfgs, seeds)):
        i1, o1, l1 = _forward_full(dsa, cfg, sd)
        r0, r1 = cu[b], cu[b + 1]
        assert torch.equal(idx[r0:r1], i1), f"sequence {b}: selection"
        assert torch.equal(out[r0:r1], o1), f"sequence {b}: output"
        assert torch.equal(lse[r0:r1], l1), f"sequence {b}: lse"
    cfg, sd = cfgs[4], seeds[4]
    _check_rows(cfg, sd, sample_rows(cfg.L, k, 8, sd), idx[cu[4]:cu[5]].cpu().numpy(), out[cu[4]:cu[5]],
                exact_idx=True)


@pytest.mark.parametrize("name,L", [("prefill_8k", 8192), ("prefill_32k", 5000), ("tiny_1k", 1024)])
def test_host_buffer_prefill_identical(dsa, name, L):
    # dsa_forward_prefill_host: inputs in page-locked host memory, results copied back by the call, the transfers
    # overlapped with the kernels chunk by chunk; every result equals dsa_forward_prefill's bit for bit
    cfg = dataclasses.replace(G.PREFILL_CONFIGS[name], L=L)
    x = prefill_device(cfg, 81)
    idx, out, lse = dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                            x["c"], cfg.k, cfg.scale)
    host = {n: (None if t is None else t.cpu().pin_memory()) for n, t in x.items()}
    h_idx = torch.empty((L, cfg.k), dtype=torch.int32, pin_memory=True)
    h_out = torch.empty((L, cfg.H, 512), dtype=torch.bfloat16, pin_memory=True)
    h_lse = torch.empty((L, cfg.H), dtype=torch.float32, pin_memory=True)
    ws = torch.empty((dsa.dsa_prefill_host_workspace_size(L, cfg.H_I, cfg.d_I, cfg.H, cfg.k),), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_forward_prefill_host(host["q_idx"], host["q_scale"], host["k_idx"], host["k_scale"], host["w"], host["q"],
                                 host["c"], cfg.k, cfg.scale, h_idx, h_out, h_lse, ws)
    torch.cuda.current_stream().synchronize()
    assert dsa.dsa_get_device_status() == 0
    assert torch.equal(h_idx, idx.cpu())
    assert torch.equal(h_out, out.cpu())
    assert torch.equal(h_lse, lse.cpu())
