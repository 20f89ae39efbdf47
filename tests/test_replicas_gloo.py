"""The multi-process (N > 1) host logic of bench.py, run as two gloo ranks on the CPU.

Under torchrun every rank runs its own independent sequence: no collective touches the data path.  What the
ranks do share is the timing protocol: a barrier on both sides of the timed region, the slowest rank's time,
and a whole-job rate counting the units every rank processed.  The reference leg runs on rank 0 alone.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WS = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(WS),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import dsa_inputs as G
    import torch.distributed as dist

    ws, r, local = bench.dist_init()
    res = {"ws": ws, "rank": r, "backend": dist.get_backend()}
    try:
        bench.barrier(ws)
        # Distinct per-rank times: every rank must see the largest one.
        res["max"] = bench.max_over_ranks(1.5 + 10.0 * r, ws)
        # Each rank draws a different sequence of the same workload shape.
        cfg = G.PREFILL_CONFIGS["tiny_1k"]
        x = G.prefill_keys(cfg, bench.replica_seed(1000, r))
        res["k_sum"] = float(x["k_idx"].view(torch.uint8).to(torch.int64).sum())
        res["rate"] = bench.job_rate(cfg.L, ws, res["max"])
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def _spawn(target, args):
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=target, args=(r,) + args) for r in range(WS)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    return codes


def test_two_replicas_share_only_the_timing(tmp_path):
    codes = _spawn(_rank_main, (_free_port(), str(tmp_path)))
    assert codes == [0] * WS
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WS)]
    assert [x["rank"] for x in res] == list(range(WS))
    assert all(x["ws"] == WS and x["backend"] == "gloo" for x in res)
    slowest = 1.5 + 10.0 * (WS - 1)
    assert all(x["max"] == slowest for x in res)
    # Whole-job rate: WS sequences of L tokens over the slowest rank's milliseconds.
    assert all(x["rate"] == pytest.approx(WS * 1024 / (slowest * 1e-3)) for x in res)
    assert res[0]["k_sum"] != res[1]["k_sum"]


def _reference_rank(rank, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(WS),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import contextlib
    import io

    import bench
    buf = io.StringIO()
    sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(WS), "--steps", "1", "--warmup", "3",
                "--ref-step-seconds", "0.0"]
    if rank == 0:
        # Keep the oracle's share of this test small: one batch of rows per step.
        bench.oracle_prefill_rate.__defaults__ = (2, 2)
    with contextlib.redirect_stdout(buf):
        bench.main()
    with open(os.path.join(out_dir, f"ref{rank}.txt"), "w") as f:
        f.write(buf.getvalue())


@pytest.mark.timeout(600)
def test_reference_leg_runs_on_rank_zero_only(tmp_path):
    codes = _spawn(_reference_rank, (_free_port(), str(tmp_path)))
    assert codes == [0] * WS
    out0 = (tmp_path / "ref0.txt").read_text().strip().splitlines()
    out1 = (tmp_path / "ref1.txt").read_text().strip()
    assert out1 == ""
    assert len(out0) == 1
    line = json.loads(out0[0])
    assert line["impl"] == "reference" and line["n_gpus"] == WS
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
