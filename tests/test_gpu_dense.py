"""The dense (masked-MHA) path of the attention for rows whose selection is every earlier key (t + 1 <= k).

Such a row attends to all of its sequence's keys 0..t, so the attention reads them as contiguous 64-row tiles and
runs ceil((t + 1) / 64) tiles instead of gathering k / 64 tiles of its padded index row (velog.io page §3.3 and the
yuuk.io notes, 推論コスト: short-sequence prefill runs DSA as masked MHA).  The keys land in the same slots of the
same tiles as on the gathered path and every tile the dense path skips is wholly masked there, so the results are
bit-identical to the gathered path over the same selection; the gathered path itself is checked against the oracle
in test_gpu_mla.py and the whole forward in test_gpu_prefill.py."""
import dataclasses

import numpy as np
import pytest
import torch

import dsa_inputs as G
import oracle as O
from gpu_util import MAX_ABS, REL_L2, f64, prefill_device, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


@pytest.mark.parametrize("L,k,H", [(3000, 2048, 128), (1024, 128, 8), (700, 2048, 128), (65, 128, 8)])
def test_prefill_dense_rows_identical_to_gathered(dsa, L, k, H):
    base = G.PREFILL_CONFIGS["prefill_8k" if H == 128 else "tiny_1k"]
    cfg = dataclasses.replace(base, name=f"dense_{L}", L=L, k=k)
    x = prefill_device(cfg, 51)
    idx, out, lse = dsa.dsa_forward_prefill(x["q_idx"], x["q_scale"], x["k_idx"], x["k_scale"], x["w"], x["q"],
                                            x["c"], cfg.k, cfg.scale)
    # the same selection through the gathered path (dsa_sparse_mla_attn never takes the dense path)
    out_g, lse_g = dsa.dsa_sparse_mla_attn(x["q"], x["c"], idx, cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    assert torch.equal(out, out_g)
    assert torch.equal(lse, lse_g)


def test_decode_dense_tokens_identical_to_gathered(dsa):
    # Short contexts (n_b + 1 <= k) take the dense path in decode too; each sequence's output equals the gathered
    # path over its own cache rows.  The cache rows after each sequence's entries are filled with NaN: the dense
    # path never lets them into a tile.
    cfg = G.DecodeConfig("dense_dec", B=6, len_lo=30, len_hi=4000, steps=2)   # 3 of the 6 contexts are below k
    seed = 52
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    lens, offs = cache["lens"], cache["offs"]
    nan_bf16 = torch.tensor([0x7FC0], dtype=torch.int16).view(torch.bfloat16).item()
    for b in range(cfg.B):
        cache["c_cache"][offs[b] + lens[b]:offs[b] + lens[b] + cfg.steps] = nan_bf16
    cache_off = torch.tensor(offs, dtype=torch.int64, device="cuda")
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st = G.decode_step_inputs(cfg, seed, 0, device="cuda")
    idx, out, lse = dsa.dsa_forward_decode(cache_off, ctx, st["q_idx"], st["q_scale"], st["w"], st["q"],
                                           st["k_new"], st["k_scale_new"], st["c_new"], cache["k_cache"],
                                           cache["k_scale_cache"], cache["c_cache"], cfg.k, cfg.scale)
    assert dsa.dsa_get_device_status() == 0
    assert torch.isfinite(out.float()).all()
    dense = [b for b in range(cfg.B) if lens[b] + 1 <= cfg.k]
    assert dense and len(dense) < cfg.B
    step_q = G.decode_step_inputs(cfg, seed, 0)
    for b in range(cfg.B):
        n = lens[b] + 1
        c_b = cache["c_cache"][offs[b]:offs[b] + n]
        o_g, l_g = dsa.dsa_sparse_mla_attn(st["q"][b:b + 1].contiguous(), c_b, idx[b:b + 1].contiguous(), cfg.scale)
        assert torch.equal(out[b:b + 1], o_g), f"sequence {b}"
        assert torch.equal(lse[b:b + 1], l_g), f"sequence {b}"
        if b in dense:   # every earlier key selected: the oracle's output is the same computation
            rows = G.decode_cache_rows(cfg, seed, b, range(n))
            ref = O.decode_row(rows, step_q, b, n, cfg.k, cfg.scale)
            assert np.array_equal(idx[b].cpu().numpy(), ref["idx"])
            got = f64(out[b])
            assert np.abs(got - ref["out"]).max() <= MAX_ABS and rel_l2(got, ref["out"]) <= REL_L2
