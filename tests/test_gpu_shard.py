"""dsa_forward_prefill_rows and the row-sharded prefill on one GPU.  The ranks of a world of N are emulated one
after another in this process: each builds the tensors of its own zig-zag blocks, the all-gather is replaced by
stacking every rank's packed blocks (what all_gather_into_tensor returns), and each block runs through the C ABI.
Every row's selection, output and LSE must equal those of the unsharded dsa_forward_prefill bit for bit (the
same kernels over the same keys; only the rows of a launch differ).  No kernel waits on another rank."""
import dataclasses

import pytest
import torch

import dsa_inputs as G
from gpu_util import prefill_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


@pytest.mark.parametrize("name,L,world", [("prefill_8k", 8192, 2), ("prefill_8k", 5000, 3), ("prefill_32k", 12000, 4)])
def test_sharded_rows_identical_to_unsharded(dsa, name, L, world):
    from sparse_attention_long_05_b200 import shard
    cfg = dataclasses.replace(G.PREFILL_CONFIGS[name], L=L)
    x = prefill_device(cfg, 62)
    idx, out, lse = dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                            x["c"], cfg.k, cfg.scale)
    key_names = ("k_idx", "k_scale", "c")
    for name_k in key_names:
        if x[name_k] is None:
            continue
        packed = torch.stack([shard.pack_blocks(x[name_k][shard.rank_rows(L, world, r)], L, world, r)
                              for r in range(world)])
        full = shard.assemble_blocks(packed, L, world)
        assert torch.equal(full.view(torch.uint8) if full.dtype == torch.float8_e4m3fn else full,
                           x[name_k].view(torch.uint8) if name_k == "k_idx" else x[name_k])
    for r in range(world):
        for r0, n in shard.zigzag_blocks(L, world, r):
            if n == 0:
                continue
            sl = slice(r0, r0 + n)
            q_scale = None if x["q_scale"] is None else x["q_scale"][sl]
            i2, o2, l2 = dsa.dsa_forward_prefill_rows(r0, x["q_idx"][sl], q_scale, x["k_idx"], x["k_scale"],
                                                      x["w"][sl], x["q"][sl], x["c"], cfg.k, cfg.scale)
            assert dsa.dsa_get_device_status() == 0
            assert torch.equal(i2, idx[sl]), f"rank {r} block {r0}: selection"
            assert torch.equal(o2, out[sl]), f"rank {r} block {r0}: output"
            assert torch.equal(l2, lse[sl]), f"rank {r} block {r0}: lse"
