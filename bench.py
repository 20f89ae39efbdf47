#!/usr/bin/env python
"""Throughput of the DSA forward hot path on B200: lightning indexer -> top-k -> sparse MLA.

Default run (N = 1): the 128K-token causal prefill (L = 131072, H_I = 64, d_I = 128 FP8, k = 2048, 128 query
heads over a 576-dim bf16 latent) is the headline line.  The same run also measures two other workloads:
- the 64-sequence decode batch (contexts 4K..128K, 256 steps, caches appended every step), under "decode";
- a packed batch of 32 independent 4K-token sequences through the varlen entry point, under "varlen".

One prefill step = the whole forward of one sequence through the C ABI with inputs resident in HBM:
dsa_prefill_select (indexer scores of a bounded block of rows + their top-k, block after block) followed by
dsa_sparse_mla_attn.  Both calls are bracketed by CUDA events on the launching stream.  After the timed region
the step's select blocks are re-run one by one through dsa_indexer_scores and dsa_topk (the same kernels and
arguments), with events around every launch; that gives the indexer's and the top-k's own share of the step.
The roofline line reports the kernel with the largest per-step time among attention, indexer and top-k.
Inputs (q alone is 19 GB) are far larger than the 126 MB L2, so no explicit L2 flush is needed between steps.

--impl reference runs the CPU oracle (fp64, test infrastructure) on the host cores on a bounded sample of
query rows per step and reports the same metric.
With torchrun (N > 1) every rank runs its own independent sequence (replicas, no collective on the data
path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsa_inputs as G  # noqa: E402

METRIC = "DSA forward tokens/s at 1 B200 (128K prefill; 64x128K decode) + % roofline"
PREFILL = G.PREFILL_CONFIGS["prefill_128k_gauss"]
DECODE = G.DECODE_CONFIG
NOMINAL_FP8_PER_BF16 = 2.0   # dense FP8 / BF16 tensor-core rate ratio (4.5 / 2.25 PFLOP/s)


# ------------------------------------------------------------------------------------------ environment
def dist_init():
    """One process per GPU under torchrun: NCCL over the GPUs; gloo where no GPU is visible (host-side tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The largest of every rank's x (every rank calls this, in the same order)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent sequence (replicas, no exchange on the data path)."""
    return base + rank


def job_rate(units_per_rank: float, ws: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return ws * units_per_rank / (ms_max * 1e-3)


def _traffic_entry(name, files):
    """The committed ncu traffic figure of a kernel (profiles/traffic.json), or None once its source differs
    from the one that capture measured."""
    import hashlib
    try:
        t = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[name]
        src = b"".join(open(os.path.join(ROOT, "sparse_attention_long_05_b200", "csrc", f), "rb").read() for f in files)
        if hashlib.sha256(src).hexdigest()[:16] != t["source_sha256_16"]:
            return None
        return t
    except (OSError, KeyError, ValueError):
        return None


def attention_traffic(tokens):
    """DRAM bytes of one sparse-MLA launch over `tokens` query tokens, scaled from the committed capture."""
    t = _traffic_entry("sparse_mla_attn", ("sparse_mla.cuh", "common.cuh"))
    return None if t is None else t["dram_bytes_per_query_token"] * tokens


def materialised_scores(blocks, k):
    """Scores one prefill step materialises: each score block's rows against the keys up to the block's end (a
    block whose rows all have t < k needs none)."""
    return sum(n * (r0 + n) for r0, n in blocks if r0 + n > k)


def select_traffic(blocks, k, name="prefill_select", files=("indexer.cuh", "topk.cuh", "common.cuh")):
    """DRAM bytes of one prefill step's indexer + top-k (or of one of them, by `name`), scaled from the committed
    capture's bytes per materialised score."""
    t = _traffic_entry(name, files)
    return None if t is None else t["dram_bytes_per_score"] * materialised_scores(blocks, k)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_burst": p["bf16_tflops"],
                "bf16_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_burst": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while the timed region runs."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.rows = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        self.cmd = ["nvidia-smi", "-i", ident, "--query-gpu=" + ",".join(self.FIELDS),
                    "--format=csv,noheader,nounits", "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[0]) for r in self.rows if num(r[0]) is not None]
        reasons = set()
        for r in self.rows:
            for name, v in zip(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"], r[3:]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(self.rows[0][1]),
                "reasons": sorted(reasons), "samples": len(self.rows),
                "power_w_max": max((num(r[2]) or 0.0) for r in self.rows)}


# ------------------------------------------------------------------------------------------ work counts
def prefill_work(cfg):
    """Algorithmic work of one prefill step: indexer FP8 flops, attention bf16 flops, top-k bytes."""
    L, k = cfg.L, cfg.k
    # (t, s) with s <= t over the rows whose selection needs scores (t + 1 > k; earlier rows take all of 0..t)
    pairs = L * (L + 1) // 2 - min(L, k) * (min(L, k) + 1) // 2
    sel = sum(min(t + 1, k) for t in range(min(L, k))) + max(0, L - k) * k
    return {"indexer_flops": 2.0 * cfg.H_I * cfg.d_I * pairs,
            "attention_flops": 2.0 * cfg.H * (cfg.D + cfg.D_v) * sel,
            "topk_bytes": 4.0 * pairs + 4.0 * L * k}


def decode_bytes(cfg, lens, steps):
    """Algorithmic HBM bytes of `steps` decode steps: key cache (e4m3 + fp32 scale) of every sequence,
    the selected latent rows, the new-token tensors, selected indices and outputs."""
    tot = 0.0
    for s in range(steps):
        for n in lens:
            m = n + s + 1
            tot += m * (cfg.d_I + 4) + min(m, cfg.k) * cfg.D * 2
        tot += cfg.B * (cfg.H * cfg.D * 2 + cfg.H_I * cfg.d_I + cfg.H_I * 4 + cfg.k * 4 + cfg.H * cfg.D_v * 2
                        + cfg.d_I + 4 + cfg.D * 2)
    return tot


# ------------------------------------------------------------------------------------------ GPU arms
def decode_traffic(step_bytes):
    """DRAM bytes of one decode step: the ncu capture's bytes per algorithmic byte (append, indexer, cluster top-k
    and attention of a 16-sequence step) times this step's algorithmic bytes; None once the kernels' source
    differs from the captured one."""
    t = _traffic_entry("decode_step", ("dsa_api.cu", "indexer.cuh", "topk_cluster.cuh", "sparse_mla.cuh",
                                       "common.cuh"))
    return None if t is None else t["dram_bytes_per_algorithmic_byte"] * step_bytes


def select_split(dsa, x, cfg, ws, idx):
    """Per-kernel time of one step's select: its score blocks re-run one by one through dsa_indexer_scores and
    dsa_topk (the kernels and arguments dsa_prefill_select launches block after block), each launch bracketed by
    CUDA events on the launching stream.  Returns (indexer ms, top-k ms, indexer launches, top-k launches)."""
    L, k = cfg.L, cfg.k
    blocks = dsa.prefill_blocks(L, k)      # the library's own block schedule
    evs = []
    for r0, rows in blocks:
        S = r0 + rows
        sc = ws[:rows * S * 4].view(torch.float32).view(rows, S)
        qs = None if x["q_scale"] is None else x["q_scale"][r0:r0 + rows]
        ks = None if x["k_scale"] is None else x["k_scale"][:S]
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        if S > k:    # as in the select: a block of rows t < k has its selection implied, without scores
            dsa.dsa_indexer_scores(x["q_idx"][r0:r0 + rows], qs, x["k_idx"][:S], ks, x["w"][r0:r0 + rows],
                                   pos0=r0, scores=sc)
        e[1].record()
        dsa.dsa_topk(sc, k, pos0=r0, idx=idx[r0:r0 + rows])
        e[2].record()
        evs.append(e)
    torch.cuda.synchronize()
    return (sum(e[0].elapsed_time(e[1]) for e in evs), sum(e[1].elapsed_time(e[2]) for e in evs),
            sum(1 for r0, rows in blocks if r0 + rows > k), len(evs))


def bench_prefill(dsa, cfg, steps, warmup, ws_n, rank, pk):
    dev = "cuda"
    x = G.prefill_keys(cfg, replica_seed(1000, rank), device=dev)
    x.update(G.prefill_queries(cfg, replica_seed(1000, rank), None, device=dev))
    L, k = cfg.L, cfg.k
    idx = torch.empty((L, k), dtype=torch.int32, device=dev)
    out = torch.empty((L, cfg.H, cfg.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((L, cfg.H), dtype=torch.float32, device=dev)
    ws = torch.empty((dsa.dsa_prefill_workspace_size(L, cfg.H_I, cfg.d_I, cfg.H, k),), dtype=torch.uint8,
                     device=dev)
    evs = []

    def step(record):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)] if record else None
        if record:
            e[0].record()
        dsa.dsa_prefill_select(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], k, idx_out=idx, ws=ws)
        if record:
            e[1].record()
        dsa.dsa_sparse_mla_attn(x["q"], x["c"], idx, cfg.scale, out=out, lse=lse)
        if record:
            e[2].record()
            evs.append(e)

    for _ in range(warmup):
        step(False)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_status() == 0
    barrier(ws_n)
    torch.cuda.synchronize()
    n0 = dsa.dsa_launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            step(True)
        t1.record()
        torch.cuda.synchronize()
    launches = dsa.dsa_launch_count() - n0
    barrier(ws_n)
    ms = max_over_ranks(t0.elapsed_time(t1), ws_n) / steps
    assert dsa.dsa_get_device_status() == 0
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    work = prefill_work(cfg)
    bf16_peak = pk["bf16_sustained"]
    att_tflops = work["attention_flops"] / (att_ms * 1e-3) / 1e12
    sel_tflops = work["indexer_flops"] / (sel_ms * 1e-3) / 1e12
    kernels = {
        "sparse_mla_attn": {"ms": att_ms, "share": att_ms / ms, "bound": "tensor", "achieved": att_tflops,
                            "peak": bf16_peak, "unit": "TFLOP/s", "frac": att_tflops / bf16_peak},
        "prefill_select": {"ms": sel_ms, "share": sel_ms / ms, "bound": "tensor", "achieved": sel_tflops,
                           "peak": bf16_peak * NOMINAL_FP8_PER_BF16, "unit": "TFLOP/s",
                           "frac": sel_tflops / (bf16_peak * NOMINAL_FP8_PER_BF16),
                           "note": "indexer (FP8 flops) + top-k of materialised score blocks: "
                                   f"{len(dsa.prefill_blocks(L, k))} blocks (the first k rows, then blocks of 1 GiB of scores)"},
    }
    # the select call's two kernels, timed one by one after the timed region (same kernels, inputs and blocks)
    idx_step = idx.clone()
    ind_ms, tk_ms, n_ind, n_tk = select_split(dsa, x, cfg, ws, idx)
    assert dsa.dsa_get_device_status() == 0
    assert torch.equal(idx, idx_step), "the launch-by-launch re-run must reproduce the step's selection"
    del idx_step
    ind_tflops = work["indexer_flops"] / (ind_ms * 1e-3) / 1e12
    tk_gbs = work["topk_bytes"] / (tk_ms * 1e-3) / 1e9
    split_note = ("the step's score blocks re-run one by one after the timed region through dsa_indexer_scores / "
                  "dsa_topk, CUDA events around every launch")
    kernels["indexer"] = {"ms": ind_ms, "launches": n_ind, "share": ind_ms / ms, "bound": "tensor",
                          "achieved": ind_tflops, "peak": bf16_peak * NOMINAL_FP8_PER_BF16, "unit": "TFLOP/s",
                          "frac": ind_tflops / (bf16_peak * NOMINAL_FP8_PER_BF16), "timed": split_note}
    kernels["topk"] = {"ms": tk_ms, "launches": n_tk, "share": tk_ms / ms, "bound": "hbm", "achieved": tk_gbs,
                       "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": tk_gbs / pk["hbm_gbs"], "timed": split_note}
    # dominant kernel: the largest per-step time among the three kernels (the select call is two of them)
    dom = max(("sparse_mla_attn", "indexer", "topk"), key=lambda n: kernels[n]["ms"])
    d = kernels[dom]
    blocks = dsa.prefill_blocks(L, k)
    traffic = {"sparse_mla_attn": lambda: attention_traffic(L),
               "indexer": lambda: select_traffic(blocks, k, "indexer", ("indexer.cuh", "common.cuh")),
               "topk": lambda: select_traffic(blocks, k, "topk", ("topk.cuh", "common.cuh"))}[dom]()
    peak_src = {"sparse_mla_attn": f"{pk['source']} bf16 sustained",
                "indexer": f"{pk['source']} bf16 sustained x2 (FP8)",
                "topk": f"{pk['source']} copy bandwidth"}[dom]
    roof = {"kernel": dom, "bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"],
            "frac": d["frac"], "traffic": traffic, "peak_source": peak_src}
    del x
    return {"ms": ms, "tokens_per_s": job_rate(L, ws_n, ms), "roofline": roof, "kernels": kernels,
            "clocks": clk.summary(), "launches": launches}


def bench_prefill_sharded(dsa, cfg, steps, warmup, ws_n, rank):
    """One sequence's prefill with its query rows split zig-zag over the ranks (sparse_attention_long_05_b200.shard):
    each rank generates the tensors of its own rows, and every step all-gathers the key-side tensors (NCCL) and
    runs dsa_forward_prefill_rows on the rank's two blocks.  Strong scaling: the job's work is one sequence."""
    from sparse_attention_long_05_b200 import shard
    dev = "cuda"
    L, k = cfg.L, cfg.k
    rows = shard.rank_rows(L, ws_n, rank)
    keys = G.prefill_keys(cfg, 1000, device=dev)
    local_keys = {n: (None if t is None else t[rows].contiguous()) for n, t in keys.items()}
    del keys
    local_q = G.prefill_queries(cfg, 1000, rows=rows, device=dev)

    def step():
        return shard.sharded_prefill(local_q, local_keys, L, k, cfg.scale)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws_n)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        res = step()
    t1.record()
    torch.cuda.synchronize()
    barrier(ws_n)
    ms = max_over_ranks(t0.elapsed_time(t1), ws_n) / steps
    assert dsa.dsa_get_device_status() == 0
    del res
    return {"ms": ms, "tokens_per_s": L / (ms * 1e-3), "rows_per_rank": len(rows)}


def bench_prefill_e2e(dsa, cfg, steps, rank):
    """The same metric through the C-ABI call with host buffers, dsa_forward_prefill_host: every input starts in
    page-locked host memory and every output lands there, the copies inside the timed region (the call overlaps
    them with its kernels).  Timed with CUDA events on the calling stream, whose work ends when the last result
    has landed on the host."""
    import psutil
    dev = "cuda"
    x = G.prefill_keys(cfg, replica_seed(1000, rank), device=dev)
    x.update(G.prefill_queries(cfg, replica_seed(1000, rank), None, device=dev))
    names = ["q_idx", "q_scale", "k_idx", "k_scale", "w", "q", "c"]
    h2d = sum(x[n].numel() * x[n].element_size() for n in names if x[n] is not None)
    L, k = cfg.L, cfg.k
    outs = {"idx": ((L, k), torch.int32), "out": ((L, cfg.H, cfg.D_v), torch.bfloat16),
            "lse": ((L, cfg.H), torch.float32)}
    d2h = sum(int(np.prod(s)) * torch.empty((), dtype=dt).element_size() for s, dt in outs.values())
    if psutil.virtual_memory().available < 1.5 * (h2d + d2h):
        return {"value": None, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "skipped": "not enough host memory for pinned copies of every input and output"}
    host = {n: (x[n].cpu().pin_memory() if x[n] is not None else None) for n in names}
    del x
    torch.cuda.empty_cache()
    hout = {n: torch.empty(s, dtype=dt, pin_memory=True) for n, (s, dt) in outs.items()}
    ws = torch.empty((dsa.dsa_prefill_host_workspace_size(L, cfg.H_I, cfg.d_I, cfg.H, k),), dtype=torch.uint8,
                     device=dev)

    def step():
        dsa.dsa_forward_prefill_host(host["q_idx"], host["q_scale"], host["k_idx"], host["k_scale"], host["w"],
                                     host["q"], host["c"], k, cfg.scale, hout["idx"], hout["out"], hout["lse"], ws)

    step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    assert dsa.dsa_get_device_status() == 0
    return {"value": L / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "call": "dsa_forward_prefill_host (page-locked host buffers)"}


def bench_varlen(dsa, cfg, nseq, steps, warmup, ws_n, rank, pk):
    """A packed batch of nseq independent causal sequences of cfg.L / nseq tokens each (the same token count and
    shapes as the single-sequence prefill), one dsa_forward_prefill_varlen call per step, CUDA events around the
    timed steps."""
    import dataclasses
    dev = "cuda"
    n = cfg.L // nseq
    scfg = dataclasses.replace(cfg, name=f"{cfg.name}_varlen", L=n)
    parts = []
    for b in range(nseq):
        x = G.prefill_keys(scfg, replica_seed(3000, rank) + 7 * b, device=dev)
        x.update(G.prefill_queries(scfg, replica_seed(3000, rank) + 7 * b, None, device=dev))
        parts.append(x)
    keys = ("q_idx", "q_scale", "k_idx", "k_scale", "w", "q", "c")
    cat = {key: torch.cat([x[key] for x in parts]) if parts[0][key] is not None else None for key in keys}
    del parts
    cu = [b * n for b in range(nseq + 1)]
    total = cu[-1]
    idx = torch.empty((total, cfg.k), dtype=torch.int32, device=dev)
    out = torch.empty((total, cfg.H, cfg.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((total, cfg.H), dtype=torch.float32, device=dev)
    ws = torch.empty((dsa.dsa_prefill_varlen_workspace_size(nseq, total, n, cfg.H_I, cfg.d_I, cfg.H, cfg.k),),
                     dtype=torch.uint8, device=dev)

    def step():
        dsa.dsa_forward_prefill_varlen(cu, cat["q_idx"], cat["q_scale"], cat["k_idx"], cat["k_scale"], cat["w"],
                                       cat["q"], cat["c"], cfg.k, cfg.scale, idx_out=idx, out=out, lse=lse, ws=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws_n)
    n0 = dsa.dsa_launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    launches = dsa.dsa_launch_count() - n0
    barrier(ws_n)
    ms = max_over_ranks(t0.elapsed_time(t1), ws_n) / steps
    assert dsa.dsa_get_device_status() == 0
    work = prefill_work(scfg)
    flops = nseq * (work["indexer_flops"] / NOMINAL_FP8_PER_BF16 + work["attention_flops"])
    del cat
    return {"metric": f"DSA forward tokens/s, {nseq} packed causal sequences of {n} tokens (varlen)",
            "value": job_rate(total, ws_n, ms), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "warmup": warmup, "launches_per_step": launches / steps,
            "bf16_equivalent_tflops": flops / (ms * 1e-3) / 1e12,
            "note": "indexer FP8 flops counted at half weight (the nominal FP8/bf16 rate ratio) plus attention "
                    "bf16 flops, over the whole call"}


def timed_steps(step, steps, warmup, ws_n):
    """Run `warmup` untimed and `steps` timed calls of step(), CUDA events around the timed ones (barriers and
    max over ranks as for the headline); returns ms per step."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws_n)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    barrier(ws_n)
    return max_over_ranks(t0.elapsed_time(t1), ws_n) / steps


def bench_kl(dsa, cfg, steps, warmup, ws_n, rank, pk):
    """The prefill with the indexer objective (dsa_forward_prefill_kl: selection, attention and the per-row
    KL(p_t || Softmax(I_t))) against the plain forward on the same inputs; the difference is the objective's pass."""
    dev = "cuda"
    x = G.prefill_keys(cfg, replica_seed(4000, rank), device=dev)
    x.update(G.prefill_queries(cfg, replica_seed(4000, rank), None, device=dev))
    args = (x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"], x["c"], cfg.k, cfg.scale)
    L = cfg.L
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device=dev)
    out = torch.empty((L, cfg.H, cfg.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((L, cfg.H), dtype=torch.float32, device=dev)
    kl = torch.empty((L,), dtype=torch.float32, device=dev)
    ws_kl = torch.empty((dsa.dsa_prefill_kl_workspace_size(L, cfg.H_I, cfg.d_I, cfg.H, cfg.k),), dtype=torch.uint8,
                        device=dev)
    ms_kl = timed_steps(lambda: dsa.dsa_forward_prefill_kl(*args, idx_out=idx, out=out, lse=lse, kl=kl, ws=ws_kl),
                        steps, warmup, ws_n)
    del ws_kl
    ws = torch.empty((dsa.dsa_prefill_workspace_size(L, cfg.H_I, cfg.d_I, cfg.H, cfg.k),), dtype=torch.uint8,
                     device=dev)
    ms_fw = timed_steps(lambda: dsa.dsa_forward_prefill(*args, idx_out=idx, out=out, lse=lse, ws=ws),
                        steps, warmup, ws_n)
    assert dsa.dsa_get_device_status() == 0
    sel = sum(min(t + 1, cfg.k) for t in range(L))
    obj_ms = max(ms_kl - ms_fw, 1e-9)
    flops = 2.0 * cfg.H * cfg.D * sel            # the objective recomputes the selected keys' logits
    del x, ws
    return {"metric": f"DSA forward + indexer KL objective tokens/s ({cfg.name}, {L} tokens)",
            "value": job_rate(L, ws_n, ms_kl), "unit": "tokens/s", "ms_per_step": ms_kl, "forward_ms": ms_fw,
            "objective_ms": obj_ms, "steps": steps, "warmup": warmup,
            "roofline": {"kernel": "indexer objective pass (logits of the selected keys again)", "bound": "tensor",
                         "achieved": flops / (obj_ms * 1e-3) / 1e12, "peak": pk["bf16_sustained"],
                         "unit": "TFLOP/s", "frac": flops / (obj_ms * 1e-3) / 1e12 / pk["bf16_sustained"],
                         "note": "its time is the KL call's minus the plain forward's"}}


def bench_short_prefill(dsa, cfg, steps, warmup, ws_n, rank, pk):
    """A prefill no longer than k: every row t attends to all of 0..t (no indexer launch; the attention reads the
    keys as contiguous tiles)."""
    dev = "cuda"
    L = cfg.L
    x = G.prefill_keys(cfg, replica_seed(5000, rank), device=dev)
    x.update(G.prefill_queries(cfg, replica_seed(5000, rank), None, device=dev))
    idx = torch.empty((L, cfg.k), dtype=torch.int32, device=dev)
    out = torch.empty((L, cfg.H, cfg.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((L, cfg.H), dtype=torch.float32, device=dev)
    ws = torch.empty((max(1, dsa.dsa_prefill_workspace_size(L, cfg.H_I, cfg.d_I, cfg.H, cfg.k)),), dtype=torch.uint8,
                     device=dev)
    n0 = dsa.dsa_launch_count()
    ms = timed_steps(lambda: dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"],
                                                     x["q"], x["c"], cfg.k, cfg.scale, idx_out=idx, out=out, lse=lse,
                                                     ws=ws), steps, warmup, ws_n)
    launches = (dsa.dsa_launch_count() - n0) / (steps + warmup)
    assert dsa.dsa_get_device_status() == 0
    flops = prefill_work(cfg)["attention_flops"]
    del x, ws
    return {"metric": f"DSA prefill tokens/s, L = {L} <= k (masked-MHA mode: every row attends to 0..t)",
            "value": job_rate(L, ws_n, ms), "unit": "tokens/s", "ms_per_step": ms, "steps": steps, "warmup": warmup,
            "launches_per_step": launches,
            "roofline": {"kernel": "sparse_mla_attn (dense tiles)", "bound": "tensor",
                         "achieved": flops / (ms * 1e-3) / 1e12, "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                         "frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_sustained"],
                         "note": "whole call (the top-k writes the implied selection, then the attention)"}}


def paged_layout(cache, lens, offs, nsteps, page_rows, seed, device="cuda"):
    """The flat decode caches' sequences moved into shuffled pages of page pools: (page table [B, max_pages],
    k_I pool, scale pool, latent pool).  One gather per pool; rows of a sequence's last page past its capacity
    repeat its last row."""
    B = len(lens)
    need = [-(-(n + nsteps) // page_rows) for n in lens]
    max_pages = max(need)
    num_pages = sum(need)
    perm = np.random.default_rng(seed).permutation(num_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    src = np.zeros(num_pages * page_rows, dtype=np.int64)
    at = 0
    for b in range(B):
        cap = lens[b] + nsteps
        for j in range(need[b]):
            pg = int(perm[at])
            at += 1
            table[b, j] = pg
            rows = np.arange(j * page_rows, (j + 1) * page_rows)
            src[pg * page_rows:(pg + 1) * page_rows] = offs[b] + np.minimum(rows, cap - 1)
    src_t = torch.from_numpy(src).to(device)
    kc = cache["k_cache"].view(torch.uint8)[src_t].view(torch.float8_e4m3fn)
    ks = cache["k_scale_cache"][src_t]
    cc = cache["c_cache"][src_t]
    return torch.from_numpy(table).to(device), kc, ks, cc


def bench_decode_paged(dsa, cfg, steps, warmup, ws_n, rank, pk, page_rows=256):
    """The decode workload over paged caches (pools of page_rows-row pages in shuffled order, a page table per
    sequence): the same sequences, inputs and algorithmic bytes as the flat-cache decode line."""
    dev = "cuda"
    seed = replica_seed(2000, rank)
    cfg, nsteps = decode_plan(cfg, warmup, steps)
    cache = G.decode_fill_cache(cfg, seed, device=dev)
    lens, offs = cache["lens"], cache["offs"]
    table, kc, ks, cc = paged_layout(cache, lens, offs, nsteps, page_rows, seed)
    del cache
    torch.cuda.empty_cache()
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    blocks = [G.decode_step_batch(cfg, seed, min(32, nsteps - s0), device=dev, step0=s0)
              for s0 in range(0, nsteps, 32)]
    inp = {key: torch.cat([b[key] for b in blocks]) if blocks[0][key] is not None else None for key in blocks[0]}
    B, k = cfg.B, cfg.k
    idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    out = torch.empty((B, cfg.H, cfg.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, cfg.H), dtype=torch.float32, device=dev)
    ws = torch.empty((dsa.dsa_decode_paged_workspace_size(B, table.shape[1], page_rows, cfg.H_I, cfg.d_I, cfg.H, k),),
                     dtype=torch.uint8, device=dev)
    it = [0]

    def step():
        s = it[0]
        g = lambda key: None if inp[key] is None else inp[key][s]   # noqa: E731
        dsa.dsa_forward_decode_paged(table, page_rows, ctx, g("q_idx"), g("q_scale"), g("w"), g("q"), g("k_new"),
                                     g("k_scale_new"), g("c_new"), kc, ks, cc, k, cfg.scale, idx_out=idx, out=out,
                                     lse=lse, ws=ws)
        ctx.add_(1)
        it[0] += 1

    ms = timed_steps(step, steps, warmup, ws_n)
    assert dsa.dsa_get_device_status() == 0
    byts = decode_bytes(cfg, lens, nsteps) - decode_bytes(cfg, lens, warmup)
    gbs = byts / steps / (ms * 1e-3) / 1e9
    del kc, ks, cc, inp
    return {"metric": f"DSA decode tokens/s over paged caches ({page_rows}-row pages, shuffled; the decode line's "
                      "workload)", "value": job_rate(B, ws_n, ms), "unit": "tokens/s", "ms_per_step": ms,
            "steps": steps, "warmup": warmup,
            "roofline": {"kernel": "decode step (append, indexer, top-k, sparse MLA)", "bound": "hbm",
                         "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"]}}


def decode_plan(cfg, warmup, steps):
    """The decode workload of a run of `warmup` untimed and `steps` timed steps: the same sequences (lengths and
    cache contents depend only on the seed), with caches that hold every entry the run appends.  Returns the
    workload and the total number of steps."""
    nsteps = warmup + steps
    return dataclasses.replace(cfg, steps=max(cfg.steps, nsteps)), nsteps


def bench_decode(dsa, cfg, steps, warmup, ws_n, rank, pk):
    dev = "cuda"
    seed = replica_seed(2000, rank)
    cfg, nsteps = decode_plan(cfg, warmup, steps)
    cache = G.decode_fill_cache(cfg, seed, device=dev)
    lens, offs = cache["lens"], cache["offs"]
    cache_off = torch.tensor(offs, dtype=torch.int64, device=dev)
    ctx = torch.tensor(lens, dtype=torch.int32, device=dev)
    blocks = [G.decode_step_batch(cfg, seed, min(32, nsteps - s0), device=dev, step0=s0)
              for s0 in range(0, nsteps, 32)]
    inp = {key: torch.cat([b[key] for b in blocks]) if blocks[0][key] is not None else None for key in blocks[0]}
    B, k = cfg.B, cfg.k
    idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    out = torch.empty((B, cfg.H, cfg.D_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, cfg.H), dtype=torch.float32, device=dev)
    ws = torch.empty((dsa.dsa_decode_workspace_size(B, cache["rows"], cfg.H_I, cfg.d_I, cfg.H, k),),
                     dtype=torch.uint8, device=dev)

    def step(s):
        g = lambda key: None if inp[key] is None else inp[key][s]   # noqa: E731
        dsa.dsa_forward_decode(cache_off, ctx, g("q_idx"), g("q_scale"), g("w"), g("q"), g("k_new"),
                               g("k_scale_new"), g("c_new"), cache["k_cache"], cache["k_scale_cache"],
                               cache["c_cache"], k, cfg.scale, idx_out=idx, out=out, lse=lse, ws=ws)
        ctx.add_(1)

    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_status() == 0
    barrier(ws_n)
    torch.cuda.synchronize()
    n0 = dsa.dsa_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for s in range(warmup, nsteps):
        step(s)
    t1.record()
    torch.cuda.synchronize()
    launches = dsa.dsa_launch_count() - n0
    barrier(ws_n)
    ms = max_over_ranks(t0.elapsed_time(t1), ws_n) / steps
    assert dsa.dsa_get_device_status() == 0
    byts = decode_bytes(cfg, lens, nsteps) - decode_bytes(cfg, lens, warmup)
    gbs = byts / steps / (ms * 1e-3) / 1e9
    return {"metric": "DSA decode tokens/s (64 sequences, 4K-128K contexts, caches appended every step)",
            "value": job_rate(B, ws_n, ms), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "warmup": warmup,
            "roofline": {"kernel": "decode step (append, indexer, top-k, sparse MLA)", "bound": "hbm",
                         "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": decode_traffic(byts / steps),
                         "peak_source": pk["source"] + " copy bandwidth"},
            "launches": launches}


# ------------------------------------------------------------------------------------------ profiling cases
def kernels_small(dsa):
    """One launch each of the main kernels on small inputs (for ncu captures): sparse MLA over 1184 query
    tokens of the 128K latent, indexer scores of a 2048-row block against 131072 keys, top-k of those rows, and one
    decode step of 16 sequences with contexts of 4K-128K."""
    cfg = PREFILL
    keys = G.prefill_keys(cfg, 5, device="cuda")
    rows = range(cfg.L - 2048, cfg.L)
    qs = G.prefill_queries(cfg, 5, rows=rows, device="cuda")
    rng = np.random.default_rng(5)
    T = 1184
    idx = torch.from_numpy(np.sort(np.stack([rng.choice(cfg.L, cfg.k, replace=False) for _ in range(T)]), axis=1)
                           .astype(np.int32)).cuda()
    dsa.dsa_sparse_mla_attn(qs["q"][:T].contiguous(), keys["c"], idx, cfg.scale)
    sc = dsa.dsa_indexer_scores(qs["q_idx"], qs["q_scale"], keys["k_idx"], keys["k_scale"], qs["w"],
                                pos0=cfg.L - 2048)
    dsa.dsa_topk(sc, cfg.k, pos0=cfg.L - 2048)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_status() == 0
    del sc, qs, idx
    # one decode step of 16 sequences with contexts of 4K-128K (append, indexer, cluster top-k, attention)
    dcfg = G.DecodeConfig("decode_16", B=16, len_lo=4096, len_hi=131072, steps=4)
    cache = G.decode_fill_cache(dcfg, 5, device="cuda")
    st = G.decode_step_inputs(dcfg, 5, 0, device="cuda")
    dsa.dsa_forward_decode(torch.tensor(cache["offs"], dtype=torch.int64, device="cuda"),
                           torch.tensor(cache["lens"], dtype=torch.int32, device="cuda"), st["q_idx"], st["q_scale"],
                           st["w"], st["q"], st["k_new"], st["k_scale_new"], st["c_new"], cache["k_cache"],
                           cache["k_scale_cache"], cache["c_cache"], dcfg.k, dcfg.scale)
    torch.cuda.synchronize()
    assert dsa.dsa_get_device_status() == 0
    print(json.dumps({"kernels_small": "ok", "attention_tokens": T, "indexer_rows": 2048, "keys": cfg.L,
                      "decode_sequences": dcfg.B, "decode_keys": sum(n + 1 for n in cache["lens"]),
                      "decode_algorithmic_bytes": decode_bytes(dcfg, cache["lens"], 1)}))


# ------------------------------------------------------------------------------------------ oracle arm
_KEYS_CACHE = {}


def oracle_prefill_rate(cfg, budget_s, seed, max_rows=256, batch=16):
    """Oracle tokens/s on the host: seeded uniformly random query rows of the workload, in batches until the
    time budget is used (at least one batch); the mean per-row time (unbiased under uniform sampling)
    extrapolates to L rows.  Input generation is not timed."""
    import oracle as O
    if cfg.name not in _KEYS_CACHE:
        _KEYS_CACHE[cfg.name] = G.prefill_keys(cfg, 7)
    keys = _KEYS_CACHE[cfg.name]
    rng = np.random.default_rng(seed)
    rows = [int(r) for r in rng.choice(cfg.L, size=max_rows, replace=False)]
    done, spent = 0, 0.0
    while done < len(rows) and (done == 0 or spent < budget_s):
        rs = rows[done:done + batch]
        qs = G.prefill_queries(cfg, seed, rows=rs)
        t = time.perf_counter()
        O.prefill_rows(keys, qs, rs, cfg.k, cfg.scale, D_v=cfg.D_v)
        spent += time.perf_counter() - t
        done += len(rs)
    return done / spent, done, spent


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args, ws_n, rank):
    """The oracle arm: each step is a bounded sample of seeded random query rows of the headline prefill, timed
    on the host cores.  ms_per_step is the measured host time of a step (the sample's oracle time); the rate
    extrapolates the mean per-row time to whole sequences of L rows."""
    if rank != 0:
        return
    cfg = PREFILL
    for w in range(args.warmup):
        oracle_prefill_rate(cfg, 0.0, 11 + w, max_rows=2, batch=2)
    rows_tot, spent_tot, wall_tot = 0, 0.0, 0.0
    for s in range(args.steps):
        t0 = time.perf_counter()
        v, n, sp = oracle_prefill_rate(cfg, args.ref_step_seconds, 100 + s)
        wall_tot += time.perf_counter() - t0
        rows_tot += n
        spent_tot += sp
    value = rows_tot / spent_tot
    cores = oracle_threads()
    sample = (f"{rows_tot} seeded random query rows of the L={cfg.L} prefill over {args.steps} steps "
              f"({spent_tot:.1f} s of host time), extrapolated to L rows")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * spent_tot / args.steps,
            "host_wall_ms_per_step": 1e3 * wall_tot / args.steps,
            "extrapolated_ms_per_sequence": 1e3 * cfg.L / value,
            "step": "one bounded sample of query rows (the oracle's time, input generation excluded)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "seq_len": cfg.L, "global_batch": 1, "H_I": cfg.H_I,
                       "d_I": cfg.d_I, "k": cfg.k, "heads": cfg.H, "parallelism": "replicas"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------ main
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["dsa", "reference"], default="dsa")
    ap.add_argument("--decode-steps", type=int, default=DECODE.steps,
                    help="timed decode steps (the caches are sized for these plus the warm-up steps)")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="host time budget of the cpu_baseline leg")
    ap.add_argument("--ref-step-seconds", type=float, default=8.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the 8K and 32K prefill lines")
    ap.add_argument("--prefill-shard", action="store_true",
                    help="with N > 1: one 128K sequence row-sharded over the N ranks (an all-gather of the key-side "
                         "tensors per step, strong scaling) instead of one independent sequence per rank")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the lines of the next rows (indexer objective, short prefill, paged decode)")
    ap.add_argument("--kernels-small", action="store_true",
                    help="run one launch of each main kernel on small inputs (profiling) and exit")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode workload (--warmup, then --decode-steps timed steps), print its "
                         "measurement and exit (profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.steps < 1 or args.decode_steps < 1:
        ap.error("at least one timed step")
    return args


def main(argv=None):
    args = parse_args(argv)
    ws_n, rank, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, ws_n, rank)
        else:
            run_dsa(args, ws_n, rank)
    finally:
        if ws_n > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


# the other prefill configurations of the workload, each measured like the headline (parity cases otherwise)
SIDE_CONFIGS = ("prefill_8k", "prefill_32k")


def side_line(pre, cfg):
    """Summary of one side configuration's prefill measurement."""
    return {"workload": cfg.name, "seq_len": cfg.L, "indexer_inputs": "integer-valued fp8" if cfg.mode == "int"
            else "gaussian fp8 with per-token scale", "value": pre["tokens_per_s"], "unit": "tokens/s",
            "ms_per_step": pre["ms"], "roofline": pre["roofline"],
            "kernels": {n: {key: v[key] for key in ("ms", "frac", "achieved", "unit")}
                        for n, v in pre["kernels"].items()}}


def run_dsa(args, ws_n, rank):
    import sparse_attention_long_05_b200 as dsa
    if args.kernels_small:
        kernels_small(dsa)
        return
    pk = peaks()
    if args.decode_only:
        dec = bench_decode(dsa, DECODE, args.decode_steps, args.warmup, ws_n, rank, pk)
        if rank == 0:
            print(json.dumps({"decode": dec}), flush=True)
        return
    if args.prefill_shard and ws_n > 1:
        sh = bench_prefill_sharded(dsa, PREFILL, args.steps, args.warmup, ws_n, rank)
        if rank == 0:
            print(json.dumps({
                "metric": METRIC, "value": sh["tokens_per_s"], "unit": "tokens/s", "n_gpus": ws_n,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": sh["ms"], "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "e4m3+bf16", "data": "synthetic",
                "config": {"workload": PREFILL.name, "seq_len": PREFILL.L, "global_batch": 1,
                           "parallelism": f"rows{ws_n} (zig-zag query-row blocks, all-gather of k_I, scales and c)",
                           "rows_per_rank": sh["rows_per_rank"]}}), flush=True)
        return
    pre = bench_prefill(dsa, PREFILL, args.steps, args.warmup, ws_n, rank, pk)
    torch.cuda.empty_cache()
    dec = None
    if not args.no_decode:
        dec = bench_decode(dsa, DECODE, args.decode_steps, args.warmup, ws_n, rank, pk)
        torch.cuda.empty_cache()
    var = None
    if not args.no_varlen:
        var = bench_varlen(dsa, PREFILL, 32, max(3, args.steps // 2), args.warmup, ws_n, rank, pk)
        torch.cuda.empty_cache()
    side = None
    if not args.no_configs:
        side = {}
        for name in SIDE_CONFIGS:
            cfg = G.PREFILL_CONFIGS[name]
            side[name] = side_line(bench_prefill(dsa, cfg, args.steps, args.warmup, ws_n, rank, pk), cfg)
            torch.cuda.empty_cache()
    rows_next = None
    if not args.no_next_rows:
        # the next rows built beyond the hot path, each measured: the indexer objective, masked-MHA short prefill,
        # paged decode (varlen prefill is the "varlen" line)
        import dataclasses
        rows_next = {
            "kl": bench_kl(dsa, G.PREFILL_CONFIGS["prefill_32k"], max(3, args.steps // 2), args.warmup, ws_n, rank,
                           pk),
            "short_prefill": bench_short_prefill(dsa, dataclasses.replace(G.PREFILL_CONFIGS["prefill_8k"],
                                                                          name="prefill_2k", L=2048),
                                                 args.steps, args.warmup, ws_n, rank, pk),
        }
        torch.cuda.empty_cache()
        if not args.no_decode:
            rows_next["paged_decode"] = bench_decode_paged(dsa, DECODE, args.decode_steps, args.warmup, ws_n, rank,
                                                           pk)
            torch.cuda.empty_cache()
    e2e = None
    if not args.no_e2e:
        e2e = bench_prefill_e2e(dsa, PREFILL, args.e2e_steps, rank)
        torch.cuda.empty_cache()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and ws_n == 1:
        v, n, sp = oracle_prefill_rate(PREFILL, args.cpu_seconds, 7)
        cpu = {"value": v, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{n} seeded random query rows of the L={PREFILL.L} prefill ({sp:.1f} s of host time), "
                         "extrapolated to L rows"}
    line = {
        "metric": METRIC, "value": pre["tokens_per_s"], "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": pre["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3+bf16", "data": "synthetic",
        "config": {"workload": PREFILL.name, "model": "DSA forward (lightning indexer -> top-k -> sparse MLA, MQA)",
                   "global_batch": ws_n, "seq_len": PREFILL.L, "H_I": PREFILL.H_I, "d_I": PREFILL.d_I,
                   "k": PREFILL.k, "heads": PREFILL.H, "latent_dim": PREFILL.D, "value_dim": PREFILL.D_v,
                   "indexer_inputs": "gaussian, fp8 e4m3 with per-token scale", "parallelism": "replicas",
                   "l2": "inputs larger than L2 (q alone is 19 GB), no flush"},
        "roofline": pre["roofline"], "kernels": pre["kernels"], "clocks": pre["clocks"],
        "e2e": e2e, "gpu_launches": pre["launches"], "cpu_baseline": cpu, "decode": dec, "varlen": var,
        "configs": side, "next_rows": rows_next,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
