"""bench.py's host arithmetic, on the CPU: the algorithmic work each roofline figure divides by, the scores a
prefill step materialises, the decode step's HBM bytes and the clock-sample summary.  Every expected value is
counted here by brute force, independently of the closed forms bench.py uses."""
import dataclasses

import pytest
import torch

import bench
import dsa_inputs as G


def _count_prefill(cfg):
    """(indexer flops, attention flops, top-k bytes) counted row by row."""
    ind = att = tk = 0
    for t in range(cfg.L):
        n = t + 1
        if n > cfg.k:                      # only rows with more than k candidates need scores
            ind += 2 * cfg.H_I * cfg.d_I * n
            tk += 4 * n
        att += 2 * cfg.H * (cfg.D + cfg.D_v) * min(n, cfg.k)
        tk += 4 * cfg.k
    return ind, att, tk


@pytest.mark.parametrize("L,k", [(1024, 128), (3000, 2048), (2048, 2048), (700, 2048)])
def test_prefill_work_counts(L, k):
    cfg = dataclasses.replace(G.PREFILL_CONFIGS["prefill_8k"], L=L, k=k)
    w = bench.prefill_work(cfg)
    ind, att, tk = _count_prefill(cfg)
    assert w["indexer_flops"] == ind
    assert w["attention_flops"] == att
    assert w["topk_bytes"] == tk


def test_materialised_scores():
    # blocks of rows t < k materialise nothing; later blocks their rows times the keys up to their end
    blocks = [(0, 2048), (2048, 2048), (4096, 1000)]
    assert bench.materialised_scores(blocks, 2048) == 2048 * 4096 + 1000 * 5096
    assert bench.materialised_scores([(0, 500)], 2048) == 0
    assert bench.materialised_scores([(0, 128), (128, 896)], 128) == 896 * 1024


def test_decode_bytes_counted_per_sequence():
    cfg = G.DecodeConfig("tiny", B=3, len_lo=10, len_hi=3000, steps=4)
    lens = [10, 2047, 2900]
    got = bench.decode_bytes(cfg, lens, 2)
    want = 0
    for s in range(2):
        for n in lens:
            keys = n + s + 1                                 # the new token attends to its own entry too
            want += keys * (cfg.d_I + 4)                     # e4m3 key row + fp32 scale, every key
            want += min(keys, cfg.k) * cfg.D * 2             # the selected bf16 latent rows
        per_seq = (cfg.H * cfg.D * 2                         # q
                   + cfg.H_I * cfg.d_I + cfg.H_I * 4         # q_I and w
                   + cfg.k * 4                               # selected indices
                   + cfg.H * cfg.D_v * 2                     # output
                   + cfg.d_I + 4 + cfg.D * 2)                # the appended key, scale and latent row
        want += cfg.B * per_seq
    assert got == want


def test_clock_summary_reasons_and_median():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.rows = [["1965", "1965", "700.5", "Not Active", "Not Active", "Not Active", "Not Active"],
               ["1800", "1965", "990.1", "Not Active", "Not Active", "Not Active", "Active"],
               ["1900", "1965", "980.0", "Not Active", "Not Active", "Not Active", "Active"]]
    sm = cs.summary()
    assert sm["sm_mhz"] == 1900 and sm["sm_max_mhz"] == 1965
    assert sm["reasons"] == ["sw_power_cap"] and sm["samples"] == 3 and sm["power_w_max"] == 990.1
    cs.rows = [["1000", "1965", "[N/A]", "Active", "Not Active", "Active", "Not Active"]]
    sm = cs.summary()
    assert sm["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"] and sm["power_w_max"] == 0.0
    cs.rows = []
    assert cs.summary()["reasons"] == ["unsampled"]


@pytest.mark.parametrize("argv", [["--gpus", "1", "--steps", "20", "--warmup", "5"], [],
                                  ["--steps", "3", "--warmup", "40", "--decode-steps", "300"],
                                  ["--decode-only", "--decode-steps", "3"]])
def test_decode_caches_hold_every_step_the_run_appends(argv):
    # The run appends one entry per sequence at every warm-up and timed step; the caches bench.py allocates must
    # hold all of them, whatever the warm-up count, and the timed part is the 256 steps of the decode workload
    # unless asked otherwise.
    args = bench.parse_args(argv)
    cfg, nsteps = bench.decode_plan(bench.DECODE, args.warmup, args.decode_steps)
    assert nsteps == args.warmup + args.decode_steps
    if "--decode-steps" not in argv:
        assert args.decode_steps == 256
    seed = bench.replica_seed(2000, 0)
    lens, offs, tot = G.decode_layout(cfg, seed)
    assert lens == G.decode_lengths(bench.DECODE, seed)          # the same sequences as the workload
    ends = offs[1:] + [tot]
    for b, (n, o) in enumerate(zip(lens, offs)):
        assert o + n + nsteps <= ends[b], f"sequence {b}: the last appended entry falls outside its range"


def test_decode_plan_keeps_the_cache_contents():
    # A larger capacity moves the sequences' cache offsets but not their contents: the entry appended at step s
    # is the cache row at position n_b + s under either layout.
    small = G.DecodeConfig("tiny", B=3, len_lo=20, len_hi=60, steps=4, mode="int")
    big, nsteps = bench.decode_plan(small, 5, 6)
    assert big.steps == 11 and nsteps == 11
    seed = 9
    assert G.decode_layout(big, seed)[1] != G.decode_layout(small, seed)[1]
    lens = G.decode_lengths(small, seed)
    batch = G.decode_step_batch(big, seed, 2, step0=nsteps - 2)
    for i, s in enumerate((nsteps - 2, nsteps - 1)):
        for b in range(small.B):
            row = G.decode_cache_rows(small, seed, b, [lens[b] + s])
            assert torch.equal(batch["k_new"][i, b].view(torch.uint8), row["k_idx"][0].view(torch.uint8))
            assert torch.equal(batch["c_new"][i, b], row["c"][0])


def test_argument_checks():
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.parse_args(["--decode-steps", "0"])


@pytest.mark.parametrize("page_rows", [128, 256])
def test_paged_layout_maps_every_position_to_its_flat_row(page_rows):
    # The paged-decode bench line's caches: every position a sequence holds or appends (n_b + steps of them) sits in
    # the pool row its page-table entry names, each page is used once, and unused table entries are -1.
    cfg = G.DecodeConfig("paged_small", B=5, len_lo=200, len_hi=1500, steps=7)
    cache = G.decode_fill_cache(cfg, 3)
    lens, offs = cache["lens"], cache["offs"]
    table, kc, ks, cc = bench.paged_layout(cache, lens, offs, cfg.steps, page_rows, 3, device="cpu")
    used = table[table >= 0].tolist()
    assert sorted(used) == list(range(len(used))) and kc.shape[0] == len(used) * page_rows
    for b in range(cfg.B):
        cap = lens[b] + cfg.steps
        npg = -(-cap // page_rows)
        assert (table[b, :npg] >= 0).all() and (table[b, npg:] == -1).all()
        pos = torch.arange(cap)
        rows = table[b, pos // page_rows].long() * page_rows + pos % page_rows
        assert torch.equal(kc[rows].view(torch.uint8), cache["k_cache"][offs[b] + pos].view(torch.uint8))
        assert torch.equal(ks[rows], cache["k_scale_cache"][offs[b] + pos])
        assert torch.equal(cc[rows], cache["c_cache"][offs[b] + pos])
