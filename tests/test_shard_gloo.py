"""Row-sharded prefill (sparse_attention_long_05_b200/shard.py) on host processes: two and three gloo ranks.

Each rank holds the query-side and key-side tensors of its zig-zag blocks only.  The all-gather must hand every
rank the sequence's key-side tensors bit for bit, and the ranks' per-block results, put together, must be the
forward of every row.  The compute step here is the oracle (this is a host-only test of the plumbing; the CUDA
entry point that the default compute step calls is checked against the unsharded forward in
test_gpu_shard.py)."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, L):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import dsa_inputs as G
    import oracle as O
    from sparse_attention_long_05_b200 import shard

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import dataclasses
        cfg = dataclasses.replace(G.PREFILL_CONFIGS["tiny_1k"], L=L, mode="gauss")
        seed = 61
        rows = shard.rank_rows(L, world, rank)
        keys_all = G.prefill_keys(cfg, seed)
        local_keys = {n: (None if t is None else t[rows]) for n, t in keys_all.items()}
        local_q = G.prefill_queries(cfg, seed, rows=rows)
        got_keys = shard.gather_keys(local_keys, L)
        same = all(torch.equal(got_keys[n].view(torch.uint8) if got_keys[n].dtype == torch.float8_e4m3fn
                               else got_keys[n], keys_all[n].view(torch.uint8) if n == "k_idx" else keys_all[n])
                   for n in ("k_idx", "k_scale", "c"))

        def oracle_compute(row0, q_rows, keys, k, scale):
            n = q_rows["q_idx"].shape[0]
            r = O.prefill_rows(keys, q_rows, range(row0, row0 + n), k, scale)
            return {"idx": r["idx"].tolist(), "out": r["out"].tolist()}

        blocks = shard.sharded_prefill(local_q, local_keys, L, cfg.k, cfg.scale, compute=oracle_compute)
        res = {"keys_identical": bool(same), "rows": rows,
               "blocks": [[r0, b["idx"], b["out"]] for r0, b in blocks]}
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world,L", [(2, 300), (3, 257)])
def test_sharded_prefill_reassembles_every_row(tmp_path, world, L):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), L)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert all(r["keys_identical"] for r in res)
    # every row on exactly one rank
    assert sorted(x for r in res for x in r["rows"]) == list(range(L))
    # the blocks put together equal the oracle's forward of every row
    sys.path.insert(0, ROOT)
    import dataclasses

    import dsa_inputs as G
    import oracle as O
    cfg = dataclasses.replace(G.PREFILL_CONFIGS["tiny_1k"], L=L, mode="gauss")
    ref = O.prefill_rows(G.prefill_keys(cfg, 61), G.prefill_queries(cfg, 61), range(L), cfg.k, cfg.scale)
    idx = np.full((L, cfg.k), -2, dtype=np.int64)
    out = np.zeros((L,) + ref["out"].shape[1:])
    for r in res:
        for r0, bi, bo in r["blocks"]:
            idx[r0:r0 + len(bi)] = bi
            out[r0:r0 + len(bo)] = bo
    assert np.array_equal(idx, ref["idx"])
    assert np.array_equal(out, ref["out"])


def test_zigzag_blocks_balance_causal_work():
    sys.path.insert(0, ROOT)
    from sparse_attention_long_05_b200 import shard
    for L, world in [(131072, 8), (131072, 2), (8192, 4), (1000, 3)]:
        work = [sum(t + 1 for t in shard.rank_rows(L, world, r)) for r in range(world)]
        assert sorted(t for r in range(world) for t in shard.rank_rows(L, world, r)) == list(range(L))
        assert max(work) / min(work) < 1.01 if L % (2 * world) == 0 else max(work) / min(work) < 1.05
    assert shard.zigzag_blocks(10, 2, 0) == [(0, 3), (9, 1)] and shard.zigzag_blocks(10, 2, 1) == [(3, 3), (6, 3)]
