"""dsa_forward_decode (append -> indexer over the key cache -> top-k -> sparse MLA) against the oracle."""
import numpy as np
import pytest
import torch

import dsa_inputs as G
import oracle as O
from gpu_util import MAX_ABS, RECALL, REL_L2, e2e_bound, f64, recall, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import sparse_attention_long_05_b200 as m
    return m


def _run_steps(dsa, cfg, seed, steps, check_seqs, exact):
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    lens, offs = cache["lens"], cache["offs"]
    cache_off = torch.tensor(offs, dtype=torch.int64, device="cuda")
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for step in range(steps):
        st = G.decode_step_inputs(cfg, seed, step, device="cuda")
        idx, out, lse = dsa.dsa_forward_decode(cache_off, ctx, st["q_idx"], st["q_scale"], st["w"], st["q"],
                                               st["k_new"], st["k_scale_new"], st["c_new"], cache["k_cache"],
                                               cache["k_scale_cache"], cache["c_cache"], cfg.k, cfg.scale)
        assert dsa.dsa_get_device_status() == 0
        idx, out = idx.cpu().numpy(), f64(out)
        step_q = G.decode_step_inputs(cfg, seed, step)
        recs, refs, gots, e2e = [], [], [], []
        for b in check_seqs:
            n = lens[b] + step + 1
            rows = G.decode_cache_rows(cfg, seed, b, range(n))
            # the appended entry landed in the cache
            o = offs[b] + n - 1
            assert torch.equal(cache["c_cache"][o].cpu(), rows["c"][n - 1])
            ref = O.decode_row(rows, step_q, b, n, cfg.k, cfg.scale)
            if exact:
                assert np.array_equal(idx[b], ref["idx"]), f"seq {b} step {step}"
                refs.append(ref["out"])
            else:
                # Gaussian mode: recall gates the selection; the attention is checked on the GPU's selection
                recs.append(recall(idx[b], ref["idx"]))
                sel = idx[b][idx[b] >= 0]
                q = O.bf16_to_f64(step_q["q"][b].view(torch.int16).numpy().view(np.uint16))
                c = O.bf16_to_f64(rows["c"][sel].view(torch.int16).numpy().view(np.uint16))
                refs.append(O.attention_row(q, c, cfg.scale, cfg.D_v)[0])
                e2e.append(ref["out"])
            gots.append(out[b])
        refs, gots = np.stack(refs), np.stack(gots)
        assert np.abs(gots - refs).max() <= MAX_ABS
        assert rel_l2(gots, refs) <= REL_L2
        if recs:
            assert np.mean(recs) >= RECALL
            assert rel_l2(gots, np.stack(e2e)) <= e2e_bound(np.mean(recs))
        ctx += 1


def test_small_batch_integer_mode_exact(dsa):
    cfg = G.DecodeConfig("small_int", B=5, len_lo=1000, len_hi=9000, steps=3, mode="int")
    _run_steps(dsa, cfg, 41, 3, range(5), exact=True)


def test_small_batch_gaussian(dsa):
    cfg = G.DecodeConfig("small_gauss", B=6, len_lo=100, len_hi=6000, steps=2)
    _run_steps(dsa, cfg, 42, 2, range(6), exact=False)


def test_full_batch_sampled_sequences(dsa):
    cfg = G.DECODE_CONFIG
    _run_steps(dsa, cfg, 43, 2, [0, 7, 21, 63], exact=False)


@pytest.mark.parametrize("B", [160, 300])
def test_batch_larger_than_the_sm_count_integer_mode_exact(dsa, B):
    # More sequences than the 148 SMs: the top-k takes one CTA per row (no histogram from the indexer) and each
    # attention cluster serves several tokens (300 sequences: more than two per cluster).  Contexts of 100..5000
    # keys, so some rows select every key.
    cfg = G.DecodeConfig("many_int", B=B, len_lo=100, len_hi=5000, steps=2, mode="int")
    _run_steps(dsa, cfg, 49, 2, [0, 1, 57, 111, 148, 159, B - 1], exact=True)


@pytest.mark.parametrize("len_lo,len_hi", [(30000, 31000), (100, 1000)])
def test_single_sequence_integer_mode_exact(dsa, len_lo, len_hi):
    # One sequence: its key tiles are spread over every indexer CTA (most get one or two tiles, some none), one
    # cluster selects its row, one attention cluster runs.  The short context takes the dense path (every key).
    cfg = G.DecodeConfig("single_int", B=1, len_lo=len_lo, len_hi=len_hi, steps=2, mode="int")
    _run_steps(dsa, cfg, 51, 2, [0], exact=True)


@pytest.mark.parametrize("k", [128, 320, 1024])
def test_smaller_k_integer_mode_exact(dsa, k):
    # k below 2048 (320: a selection ending in half a 128-key tile); contexts of 100..9000 keys, so some tokens
    # take every key and the others select k of them
    cfg = G.DecodeConfig("small_k_int", B=5, len_lo=100, len_hi=9000, steps=2, k=k, mode="int")
    _run_steps(dsa, cfg, 52, 2, range(5), exact=True)


def test_contexts_around_k_integer_mode_exact(dsa):
    # contexts n_b of 2044..2050 keys before the step (k = 2048): over three appended steps the tokens cross from the
    # dense path (n_b + 1 <= k: every key selected, read as contiguous tiles) to the selected path, one key at a time
    cfg = G.DecodeConfig("around_k", B=12, len_lo=2044, len_hi=2050, steps=3, mode="int")
    lens = G.decode_lengths(cfg, 50)
    assert min(lens) + 1 <= cfg.k < max(lens) + 3
    _run_steps(dsa, cfg, 50, 3, range(12), exact=True)


def test_long_rows_integer_mode_exact(dsa):
    # Score rows of 16K-40K keys take the top-k's sampled path; integer mode has many tied scores, which it
    # must still break exactly as the oracle does.  The rows' cache offsets are not multiples of 4.
    cfg = G.DecodeConfig("long_int", B=4, len_lo=16384, len_hi=40000, steps=2, mode="int")
    assert any(o % 4 for o in G.decode_layout(cfg, 45)[1])
    _run_steps(dsa, cfg, 45, 2, range(4), exact=True)


def test_invalid_sequence_is_reported_and_skipped(dsa):
    # Sequence 1 points past the end of the cache: the call reports DSA_ERR_BAD_INDEX, touches none of its
    # rows, selects nothing for it, and the other sequences (whose score rows move up) are unaffected.
    cfg = G.DecodeConfig("bad_seq", B=3, len_lo=17000, len_hi=30000, steps=1, mode="int")
    seed = 46
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    lens, offs = cache["lens"], list(cache["offs"])
    offs[1] = cache["rows"]
    cache_off = torch.tensor(offs, dtype=torch.int64, device="cuda")
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    before = cache["c_cache"].clone()
    st = G.decode_step_inputs(cfg, seed, 0, device="cuda")
    idx, out, _ = dsa.dsa_forward_decode(cache_off, ctx, st["q_idx"], st["q_scale"], st["w"], st["q"],
                                         st["k_new"], st["k_scale_new"], st["c_new"], cache["k_cache"],
                                         cache["k_scale_cache"], cache["c_cache"], cfg.k, cfg.scale)
    assert dsa.dsa_get_device_status() == 6
    idx, out = idx.cpu().numpy(), f64(out)
    assert (idx[1] == -1).all()
    step_q = G.decode_step_inputs(cfg, seed, 0)
    changed = (cache["c_cache"] != before).any(dim=1).nonzero().flatten().tolist()
    assert changed == [cache["offs"][0] + lens[0], cache["offs"][2] + lens[2]]
    for b in (0, 2):
        n = lens[b] + 1
        rows = G.decode_cache_rows(cfg, seed, b, range(n))
        ref = O.decode_row(rows, step_q, b, n, cfg.k, cfg.scale)
        assert np.array_equal(idx[b], ref["idx"])
        assert np.abs(out[b] - ref["out"]).max() <= MAX_ABS
        assert rel_l2(out[b], ref["out"]) <= REL_L2


def test_full_batch_256_steps_checked_at_first_and_last(dsa):
    # The decode workload as measured: 64 sequences with contexts of 4K-128K, 256 steps, the caches appended at
    # every step.  Steps 0 and 255 are checked on 8 seeded random sequences against the oracle (recall gate, the
    # attention over the GPU's selection, the end-to-end bound), and after the last step every appended entry of
    # those sequences is in its cache row.
    cfg = G.DECODE_CONFIG
    seed = 44
    nsteps = cfg.steps
    assert nsteps == 256
    check = sorted(int(b) for b in np.random.default_rng(seed).choice(cfg.B, size=8, replace=False))
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    lens, offs = cache["lens"], cache["offs"]
    cache_off = torch.tensor(offs, dtype=torch.int64, device="cuda")
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    got = {}
    for s0 in range(0, nsteps, 32):
        blk = G.decode_step_batch(cfg, seed, min(32, nsteps - s0), device="cuda", step0=s0)
        for i in range(blk["q"].shape[0]):
            g = lambda key: None if blk[key] is None else blk[key][i]   # noqa: E731
            idx, out, lse = dsa.dsa_forward_decode(cache_off, ctx, g("q_idx"), g("q_scale"), g("w"), g("q"),
                                                   g("k_new"), g("k_scale_new"), g("c_new"), cache["k_cache"],
                                                   cache["k_scale_cache"], cache["c_cache"], cfg.k, cfg.scale)
            step = s0 + i
            if step in (0, nsteps - 1):
                got[step] = (idx.cpu().numpy(), f64(out))
            ctx += 1
    assert dsa.dsa_get_device_status() == 0
    assert ctx.cpu().tolist() == [n + nsteps for n in lens]
    for b in check:
        rows = G.decode_cache_rows(cfg, seed, b, range(lens[b] + nsteps))
        o = offs[b]
        # every entry appended over the 256 steps sits at its position in the flat caches
        appended = slice(o + lens[b], o + lens[b] + nsteps)
        assert torch.equal(cache["c_cache"][appended].cpu(), rows["c"][lens[b]:])
        assert torch.equal(cache["k_cache"][appended].cpu().view(torch.uint8), rows["k_idx"][lens[b]:].view(torch.uint8))
        assert torch.equal(cache["k_scale_cache"][appended].cpu(), rows["k_scale"][lens[b]:])
    for step, (idx, out) in got.items():
        step_q = G.decode_step_inputs(cfg, seed, step, seqs=range(cfg.B))
        recs, e2e_ref, att, gots = [], [], [], []
        for b in check:
            n = lens[b] + step + 1
            rows = G.decode_cache_rows(cfg, seed, b, range(n))
            ref = O.decode_row(rows, step_q, b, n, cfg.k, cfg.scale)
            recs.append(recall(idx[b], ref["idx"]))
            sel = idx[b][idx[b] >= 0]
            assert len(sel) == min(n, cfg.k) and (np.diff(sel) > 0).all() and sel.max() < n
            q = O.bf16_to_f64(step_q["q"][b].view(torch.int16).numpy().view(np.uint16))
            c = O.bf16_to_f64(rows["c"][sel].view(torch.int16).numpy().view(np.uint16))
            att.append(O.attention_row(q, c, cfg.scale, cfg.D_v)[0])
            e2e_ref.append(ref["out"])
            gots.append(out[b])
        att, e2e_ref, gots = np.stack(att), np.stack(e2e_ref), np.stack(gots)
        assert np.mean(recs) >= RECALL, f"step {step}: mean recall {np.mean(recs)}"
        assert np.abs(gots - att).max() <= MAX_ABS and rel_l2(gots, att) <= REL_L2, f"step {step}"
        assert rel_l2(gots, e2e_ref) <= e2e_bound(np.mean(recs)), f"step {step}"


def _paged_copy(cache, lens, offs, steps, page_rows, seed, spare=5):
    """The flat caches' sequences moved into shuffled pages of page pools (with spare pages full of NaN), and
    the page table [B, max_pages] that maps them."""
    B = len(lens)
    need = [-(-(n + steps) // page_rows) for n in lens]
    max_pages = max(need) + 1
    num_pages = sum(need) + spare
    perm = np.random.default_rng(seed).permutation(num_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    kc = torch.zeros((num_pages * page_rows, cache["k_cache"].shape[1]), dtype=torch.uint8, device="cuda")
    ks = torch.full((num_pages * page_rows,), float("nan"), dtype=torch.float32, device="cuda")
    nan_bf16 = torch.tensor([0x7FC0], dtype=torch.int16).view(torch.bfloat16).item()
    cc = torch.full((num_pages * page_rows, cache["c_cache"].shape[1]), nan_bf16, dtype=torch.bfloat16, device="cuda")
    at = 0
    for b in range(B):
        for j in range(need[b]):
            pg = int(perm[at])
            at += 1
            table[b, j] = pg
            r0, r1 = offs[b] + j * page_rows, min(offs[b] + lens[b] + steps, offs[b] + (j + 1) * page_rows)
            d0 = pg * page_rows
            kc[d0:d0 + r1 - r0] = cache["k_cache"][r0:r1].view(torch.uint8)
            ks[d0:d0 + r1 - r0] = cache["k_scale_cache"][r0:r1]
            cc[d0:d0 + r1 - r0] = cache["c_cache"][r0:r1]
    return torch.from_numpy(table).cuda(), kc.view(torch.float8_e4m3fn), ks, cc


@pytest.mark.parametrize("B,len_hi,page_rows", [(6, 20000, 128), (6, 20000, 256), (160, 5000, 512)])
def test_paged_cache_identical_to_flat(dsa, B, len_hi, page_rows):
    # The same sequences in flat caches and in shuffled pages of page pools (spare pages hold NaN): every step's
    # selection, output and LSE are bit-identical, and the appended entries land in the right pages.  160
    # sequences: more than the SMs (one top-k CTA per row, several tokens per attention cluster).
    cfg = G.DecodeConfig("paged", B=B, len_lo=100, len_hi=len_hi, steps=3)
    seed = 47
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    lens, offs = cache["lens"], cache["offs"]
    table, kc, ks, cc = _paged_copy(cache, lens, offs, cfg.steps, page_rows, seed)
    cache_off = torch.tensor(offs, dtype=torch.int64, device="cuda")
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    for step in range(cfg.steps):
        st = G.decode_step_inputs(cfg, seed, step, device="cuda")
        args = (st["q_idx"], st["q_scale"], st["w"], st["q"], st["k_new"], st["k_scale_new"], st["c_new"])
        i1, o1, l1 = dsa.dsa_forward_decode(cache_off, ctx, *args, cache["k_cache"], cache["k_scale_cache"],
                                            cache["c_cache"], cfg.k, cfg.scale)
        i2, o2, l2 = dsa.dsa_forward_decode_paged(table, page_rows, ctx, *args, kc, ks, cc, cfg.k, cfg.scale)
        assert dsa.dsa_get_device_status() == 0
        assert torch.equal(i1, i2), f"step {step}: selection"
        assert torch.equal(o1, o2), f"step {step}: output"
        assert torch.equal(l1, l2), f"step {step}: lse"
        ctx += 1
    tab = table.cpu().numpy()
    for b in range(cfg.B):
        for s in range(cfg.steps):
            pos = lens[b] + s
            row = int(tab[b, pos // page_rows]) * page_rows + pos % page_rows
            assert torch.equal(cc[row], cache["c_cache"][offs[b] + pos])
            assert torch.equal(kc[row].view(torch.uint8), cache["k_cache"][offs[b] + pos].view(torch.uint8))


def test_paged_bad_page_is_reported_and_skipped(dsa):
    cfg = G.DecodeConfig("paged_bad", B=3, len_lo=3000, len_hi=9000, steps=1, mode="int")
    seed = 48
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    lens, offs = cache["lens"], cache["offs"]
    table, kc, ks, cc = _paged_copy(cache, lens, offs, cfg.steps, 128, seed)
    table[1, 0] = kc.shape[0] // 128          # one past the last page of the pools
    before = cc.clone()
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st = G.decode_step_inputs(cfg, seed, 0, device="cuda")
    idx, out, _ = dsa.dsa_forward_decode_paged(table, 128, ctx, st["q_idx"], st["q_scale"], st["w"], st["q"],
                                               st["k_new"], st["k_scale_new"], st["c_new"], kc, ks, cc, cfg.k,
                                               cfg.scale)
    assert dsa.dsa_get_device_status() == 6
    idx = idx.cpu().numpy()
    assert (idx[1] == -1).all()
    changed = (cc.view(torch.int16) != before.view(torch.int16)).any(dim=1).nonzero().flatten().tolist()
    tab = table.cpu().numpy()
    assert changed == sorted(int(tab[b, lens[b] // 128]) * 128 + lens[b] % 128 for b in (0, 2))
    step_q = G.decode_step_inputs(cfg, seed, 0)
    for b in (0, 2):
        n = lens[b] + 1
        ref = O.decode_row(G.decode_cache_rows(cfg, seed, b, range(n)), step_q, b, n, cfg.k, cfg.scale)
        assert np.array_equal(idx[b], ref["idx"])
