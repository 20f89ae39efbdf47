"""Row-sharded prefill of one causal sequence over the ranks of a torch.distributed process group.

The forward of a long sequence splits by query rows: once every rank holds all of the sequence's key-side tensors
(indexer keys k_I, their scales and the latent entries c), each query row's selection and attention depend on
nothing else.  The rows are cut into 2N equal blocks for N ranks and dealt zig-zag, rank r taking blocks r and
2N - 1 - r: a row's causal work grows with its position, so every rank gets the same amount.  Each rank holds the
query-side tensors and the key-side tensors of its own rows; one all-gather per key-side tensor is the path's only
exchange step (NCCL over NVLink between GPUs, gloo between host processes), and each rank then runs
dsa_forward_prefill_rows on its blocks.  The outputs stay on the rank that computed them.

This module is plumbing: block bookkeeping and the collective.  Every step of the method runs in libdsa.so, which
is imported only when the default compute step is used.
"""
from __future__ import annotations

import torch



def block_rows(L: int, world: int) -> int:
    """Rows per block: 2 * world blocks cover the sequence (the last ones may be shorter or empty)."""
    return -(-L // (2 * world))


def zigzag_blocks(L: int, world: int, rank: int):
    """(first row, rows) of the blocks of `rank`, in position order: blocks rank and 2 world - 1 - rank."""
    b = block_rows(L, world)
    out = []
    for i in sorted((rank, 2 * world - 1 - rank)):
        r0 = min(L, i * b)
        out.append((r0, min(L, r0 + b) - r0))
    return out


def rank_rows(L: int, world: int, rank: int) -> list:
    """Positions of the rows `rank` holds, in the order of its blocks."""
    return [r for r0, n in zigzag_blocks(L, world, rank) for r in range(r0, r0 + n)]


def _wire(t: torch.Tensor) -> torch.Tensor:
    """Rows of any dtype as rows of bytes (every backend moves uint8)."""
    return t.contiguous().reshape(t.shape[0], -1).view(torch.uint8)


def pack_blocks(local: torch.Tensor, L: int, world: int, rank: int) -> torch.Tensor:
    """The rank's rows (its blocks in position order, concatenated) as [2, block_rows, ...], zero-padded."""
    b = block_rows(L, world)
    out = torch.zeros((2, b) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    at = 0
    for slot, (r0, n) in enumerate(zigzag_blocks(L, world, rank)):
        out[slot, :n] = local[at:at + n]
        at += n
    return out


def assemble_blocks(gathered: torch.Tensor, L: int, world: int) -> torch.Tensor:
    """Every rank's packed blocks [world, 2, block_rows, ...] -> the sequence's rows [L, ...] in position order.
    Blocks 0 .. world - 1 are the ranks' first blocks; blocks world .. 2 world - 1 their second ones, rank
    world - 1 first."""
    firsts = gathered[:, 0]
    seconds = torch.flip(gathered[:, 1], dims=(0,))
    full = torch.cat([firsts, seconds]).reshape((-1,) + tuple(gathered.shape[3:]))
    return full[:L]


def gather_keys(local_keys: dict, L: int, group=None) -> dict:
    """All-gather the key-side tensors of every rank's rows: {name: [rows of this rank, ...] or None} ->
    {name: [L, ...] or None}, the sequence's tensors in position order on every rank."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    out = {}
    for name, t in local_keys.items():
        if t is None:
            out[name] = None
            continue
        blocks = pack_blocks(t, L, world, rank)                     # [2, block_rows, ...]
        packed = _wire(blocks.reshape((-1,) + tuple(t.shape[1:]))).reshape(2, blocks.shape[1], -1)
        # the ranks' packed blocks concatenated along the first dimension (the form every backend accepts)
        gathered = torch.empty((world * packed.shape[0],) + tuple(packed.shape[1:]), dtype=packed.dtype,
                               device=packed.device)
        dist.all_gather_into_tensor(gathered, packed, group=group)
        full = assemble_blocks(gathered.view((world,) + tuple(packed.shape)), L, world)
        out[name] = full.contiguous().view(t.dtype).reshape((L,) + tuple(t.shape[1:]))
    return out


def _default_compute(row0, q_rows: dict, keys: dict, k: int, scale: float):
    from . import _lib
    idx, out, lse = _lib.dsa_forward_prefill_rows(row0, q_rows["q_idx"], q_rows["q_scale"], keys["k_idx"],
                                                  keys["k_scale"], q_rows["w"], q_rows["q"], keys["c"], k, scale)
    return {"idx": idx, "out": out, "lse": lse}


def sharded_prefill(local_q: dict, local_keys: dict, L: int, k: int, scale: float, group=None, compute=None):
    """The forward of this rank's rows of one causal sequence of L tokens.

    local_q: {"q_idx", "q_scale", "w", "q"} and local_keys: {"k_idx", "k_scale", "c"}, each holding this rank's
    rows in the order rank_rows() lists them.  Returns [(row0, {"idx", "out", "lse"}), ...], one entry per block of
    this rank.  `compute(row0, q_rows, keys, k, scale)` runs steps 1-3 for one block (default: libdsa.so's
    dsa_forward_prefill_rows).
    """
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    keys = gather_keys(local_keys, L, group)
    compute = compute or _default_compute
    res, at = [], 0
    for r0, n in zigzag_blocks(L, world, rank):
        if n == 0:
            continue
        q_rows = {name: (None if t is None else t[at:at + n]) for name, t in local_q.items()}
        res.append((r0, compute(r0, q_rows, keys, k, scale)))
        at += n
    return res
