"""Pins of the fp64 CPU oracle against things other than itself (no GPU needed).

Each pin is chosen so that a plausible mistake in the oracle fails at least one of them:
* format definitions and torch's own conversions for the FP8 / bf16 decoders;
* hand-worked examples of the index score, the selection and the attention (tests/golden/);
* an independent algebraic route for the score (w*ReLU(x) = (w*x + w*|x|)/2) and exact int64 arithmetic;
* invariants of the formula (w >= 0, head / dim permutations, q_I = 0);
* the definition of top-k under a total order, checked pairwise by brute force;
* torch's scaled_dot_product_attention (fp64) for dense causal rows, closed forms for q = 0 and k = 1;
* pure-Python brute force of the whole path on micro sequences.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e4m3_bits(vals):
    return torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# ------------------------------------------------------------------------------------------- decoders
def test_e4m3_definition_values():
    t = O.e4m3_table()
    assert t[0x00] == 0.0 and t[0x80] == 0.0 and math.copysign(1, t[0x80]) == -1
    assert t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9
    assert t[0x08] == 2.0 ** -6
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert t[0x3F] == 1.875 and t[0x40] == 2.0
    # integers -16..16 are all representable
    for v in range(-16, 17):
        assert O.e4m3_to_f64(_e4m3_bits([v]))[0] == v


def test_e4m3_matches_torch_conversion():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])


def test_bf16_widening_matches_torch():
    g = torch.Generator().manual_seed(0)
    x = (torch.randn(4096, generator=g) * 100).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_to_f64(bits), x.to(torch.float64).numpy())


# ------------------------------------------------------------------------------------------- index score
def test_golden_index_score_and_selection():
    g = json.load(open(os.path.join(GOLDEN, "indexer_tiny.json")))
    qI = np.array(g["q_I_t"], dtype=np.float64)
    kI = np.array(g["k_I"], dtype=np.float64)
    for case in g["cases"]:
        I = O.indexer_scores_row(qI, np.array(case["w"], dtype=np.float64), kI)
        assert I.tolist() == case["I"]
        assert O.topk_row(I, 1).tolist() == case["top1"]
        assert O.topk_row(I, 2).tolist() == case["top2"]
        assert O.topk_row(I, 4).tolist() == case["top4"]


@pytest.mark.parametrize("seed", range(4))
def test_score_abs_identity_route(seed):
    """w*ReLU(x) = (w*x + w*|x|)/2: the linear half computed as k . (sum_j w_j q_j), a different route."""
    rng = np.random.default_rng(seed)
    H_I, d_I, n = 5, 7, 33
    qI = rng.normal(size=(H_I, d_I))
    kI = rng.normal(size=(n, d_I))
    w = rng.normal(size=H_I)
    lin = kI @ (w @ qI)
    absterm = np.abs(np.einsum("sd,jd->sj", kI, qI)) @ w
    np.testing.assert_allclose(O.indexer_scores_row(qI, w, kI), 0.5 * (lin + absterm), rtol=1e-12, atol=1e-12)


def test_score_integer_exact():
    rng = np.random.default_rng(7)
    H_I, d_I, n = 64, 128, 300
    qi = rng.integers(-7, 8, size=(H_I, d_I))
    ki = rng.integers(-7, 8, size=(n, d_I))
    w = rng.integers(-3, 4, size=H_I)
    exact = np.maximum(ki.astype(np.int64) @ qi.T.astype(np.int64), 0) @ w.astype(np.int64)
    got = O.indexer_scores_row(qi.astype(np.float64), w.astype(np.float64), ki.astype(np.float64))
    assert np.array_equal(got, exact.astype(np.float64))
    assert np.abs(exact).max() < 2 ** 24


def test_score_invariants():
    rng = np.random.default_rng(3)
    H_I, d_I, n = 6, 9, 50
    qI = rng.normal(size=(H_I, d_I))
    kI = rng.normal(size=(n, d_I))
    w = rng.normal(size=H_I)
    I = O.indexer_scores_row(qI, w, kI)
    # w >= 0  =>  every score is >= 0 (each head term is a ReLU)
    assert (O.indexer_scores_row(qI, np.abs(w), kI) >= 0).all()
    # permuting heads (q_I and w together) and dims (q_I and k_I together) leaves scores unchanged
    ph, pd = rng.permutation(H_I), rng.permutation(d_I)
    np.testing.assert_allclose(O.indexer_scores_row(qI[ph], w[ph], kI), I, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.indexer_scores_row(qI[:, pd], w, kI[:, pd]), I, rtol=1e-12, atol=1e-12)
    # q_I = 0  =>  all scores 0; positive rescaling of q_I scales the score
    assert (O.indexer_scores_row(np.zeros_like(qI), w, kI) == 0).all()
    np.testing.assert_allclose(O.indexer_scores_row(3.0 * qI, w, kI), 3.0 * I, rtol=1e-12, atol=1e-12)
    # one head whose query is -k_s: ReLU kills the term at s
    one = O.indexer_scores_row(-kI[4:5], np.array([2.0]), kI)
    assert one[4] == 0.0
    # the single head, unit weight case is ReLU of a plain dot product
    np.testing.assert_allclose(O.indexer_scores_row(qI[:1], np.array([1.0]), kI), np.maximum(kI @ qI[0], 0))


# ------------------------------------------------------------------------------------------- selection
def _dominates(a, b, sc):
    return sc[a] > sc[b] or (sc[a] == sc[b] and a < b)


@pytest.mark.parametrize("seed", range(30))
def test_topk_pairwise_dominance(seed):
    """Top-k under the total order (score desc, s asc): every selected entry beats every unselected one."""
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    k = int(rng.integers(1, 12))
    sc = rng.integers(-3, 4, size=n).astype(np.float64)   # heavy ties
    if seed % 3 == 0:
        sc[rng.integers(0, n)] = -0.0
    out = O.topk_row(sc, k)
    sel = [int(s) for s in out if s >= 0]
    assert len(sel) == min(k, n)
    assert sel == sorted(sel) and (out[len(sel):] == -1).all()
    rest = sorted(set(range(n)) - set(sel))
    for a, b in itertools.product(sel, rest):
        assert _dominates(a, b, sc)


def test_topk_ties_and_short_rows():
    assert O.topk_row(np.zeros(10), 4).tolist() == [0, 1, 2, 3]
    assert O.topk_row(np.array([0.0, -0.0, 0.0]), 2).tolist() == [0, 1]
    assert O.topk_row(np.array([5.0, 1.0]), 4).tolist() == [0, 1, -1, -1]
    assert O.topk_row(np.array([1.0, 2.0, 3.0, 3.0]), 1).tolist() == [2]


def test_topk_distinct_matches_argpartition():
    rng = np.random.default_rng(11)
    sc = rng.normal(size=5000)
    k = 257
    ref = np.sort(np.argpartition(-sc, k)[:k])
    assert np.array_equal(O.topk_row(sc, k), ref)


# ------------------------------------------------------------------------------------------- attention
def test_golden_attention():
    g = json.load(open(os.path.join(GOLDEN, "attention_tiny.json")))
    u, lse = O.attention_row(np.array(g["q"]), np.array(g["c"]), g["scale"], g["D_v"])
    np.testing.assert_allclose(u, np.array(g["u"]), rtol=1e-12)
    np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=1e-12)


@pytest.mark.parametrize("m", [1, 7, 300])
def test_attention_matches_torch_sdpa(m):
    rng = np.random.default_rng(m)
    H, D, D_v = 4, 24, 16
    q = rng.normal(size=(H, D))
    c = rng.normal(size=(m, D))
    scale = D ** -0.5
    u, lse = O.attention_row(q, c, scale, D_v)
    qt = torch.tensor(q).view(H, 1, D)
    kt = torch.tensor(c).expand(H, m, D)
    vt = torch.tensor(c[:, :D_v]).expand(H, m, D_v)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale).view(H, D_v).numpy()
    np.testing.assert_allclose(u, ref, rtol=1e-10, atol=1e-12)
    ref_lse = torch.logsumexp(torch.tensor(q) @ torch.tensor(c).T * scale, dim=1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(5)
    H, D, D_v, m = 3, 10, 6, 9
    c = rng.normal(size=(m, D))
    # q = 0: uniform weights, u = mean of the values
    u, lse = O.attention_row(np.zeros((H, D)), c, 0.3, D_v)
    np.testing.assert_allclose(u, np.tile(c[:, :D_v].mean(0), (H, 1)), rtol=1e-12)
    np.testing.assert_allclose(lse, np.log(m))
    # a single selected entry: u = its value part
    u1, _ = O.attention_row(rng.normal(size=(H, D)), c[2:3], 0.3, D_v)
    np.testing.assert_allclose(u1, np.tile(c[2, :D_v], (H, 1)), rtol=1e-12)
    # order of the selected entries does not matter
    q = rng.normal(size=(H, D))
    p = rng.permutation(m)
    ua, la = O.attention_row(q, c, 0.3, D_v)
    ub, lb = O.attention_row(q, c[p], 0.3, D_v)
    np.testing.assert_allclose(ua, ub, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-12)
    # a dominant logit: u is (almost exactly) that entry's value
    qd = np.zeros((1, D)); qd[0, 0] = 1.0
    cd = c.copy(); cd[4, 0] = 1e4
    ud, _ = O.attention_row(qd, cd, 1.0, D_v)
    np.testing.assert_allclose(ud[0], cd[4, :D_v], rtol=1e-12)
    # no selected entry: zeros and -inf
    uz, lz = O.attention_row(q, c[:0], 0.3, D_v)
    assert (uz == 0).all() and np.isneginf(lz).all()


# ------------------------------------------------------------------------------------------- whole path
def _micro_inputs(rng, L, H_I, d_I, H, D):
    qi = rng.integers(-7, 8, size=(L, H_I, d_I))
    ki = rng.integers(-7, 8, size=(L, d_I))
    w = rng.integers(-3, 4, size=(L, H_I)).astype(np.float32)
    q = torch.randn(L, H, D, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30)))).to(torch.bfloat16)
    c = torch.randn(L, D, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30)))).to(torch.bfloat16)
    keys = {"k_idx": _e4m3_bits(ki).reshape(L, d_I), "k_scale": None, "c": c}
    queries = {"q_idx": _e4m3_bits(qi).reshape(L, H_I, d_I), "q_scale": None, "w": w, "q": q}
    return qi, ki, w, q, c, keys, queries


@pytest.mark.parametrize("seed", range(3))
def test_prefill_rows_bruteforce_micro(seed):
    """Pure-Python loops over the whole path on a micro sequence (L=12, k=3) against prefill_rows."""
    rng = np.random.default_rng(100 + seed)
    L, H_I, d_I, H, D, D_v, k = 12, 2, 4, 2, 6, 4, 3
    qi, ki, w, q, c, keys, queries = _micro_inputs(rng, L, H_I, d_I, H, D)
    scale = 0.37
    got = O.prefill_rows(keys, queries, range(L), k, scale, D_v=D_v, want_scores=True)
    qf, cf = q.double().tolist(), c.double().tolist()
    for t in range(L):
        I = []
        for s in range(t + 1):
            tot = 0
            for j in range(H_I):
                x = sum(int(qi[t, j, d]) * int(ki[s, d]) for d in range(d_I))
                tot += int(w[t, j]) * max(x, 0)
            I.append(tot)
        assert got["scores"][t].tolist() == I
        ranked = sorted(range(t + 1), key=lambda s: (-I[s], s))[:k]
        sel = sorted(ranked)
        assert got["idx"][t].tolist() == sel + [-1] * (k - len(sel))
        for h in range(H):
            logit = [scale * sum(qf[t][h][d] * cf[s][d] for d in range(D)) for s in sel]
            mx = max(logit)
            e = [math.exp(v - mx) for v in logit]
            z = sum(e)
            for v in range(D_v):
                ref = sum(e[i] * cf[s][v] for i, s in enumerate(sel)) / z
                assert abs(got["out"][t, h, v] - ref) < 1e-12
            assert abs(got["lse"][t, h] - (mx + math.log(z))) < 1e-12


def test_short_rows_equal_dense_causal_attention():
    """For t + 1 <= k the selection is all of 0..t and the output equals dense causal attention."""
    rng = np.random.default_rng(9)
    L, H_I, d_I, H, D, D_v, k = 20, 3, 8, 4, 16, 12, 32
    _, _, _, q, c, keys, queries = _micro_inputs(rng, L, H_I, d_I, H, D)
    scale = D ** -0.5
    got = O.prefill_rows(keys, queries, range(L), k, scale, D_v=D_v)
    for t in range(L):
        assert got["idx"][t].tolist() == list(range(t + 1)) + [-1] * (k - t - 1)
    qt = q.double().permute(1, 0, 2)                 # [H, L, D]
    kt = c.double().expand(H, L, D)
    vt = c.double()[:, :D_v].expand(H, L, D_v)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    np.testing.assert_allclose(got["out"], ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_q_index_zero_selects_first_k():
    """q_I = 0 makes every score 0, so the tie-break alone decides: S_t = {0..k-1}."""
    rng = np.random.default_rng(4)
    L, H_I, d_I, H, D, k = 40, 2, 8, 2, 8, 5
    _, _, _, _, _, keys, queries = _micro_inputs(rng, L, H_I, d_I, H, D)
    queries["q_idx"] = np.zeros_like(queries["q_idx"])
    got = O.prefill_rows(keys, queries, range(L), k, 1.0, D_v=4)
    for t in range(k, L):
        assert got["idx"][t].tolist() == list(range(k))


def test_decode_row_equals_prefill_row():
    """A decode token at position n over cache rows 0..n is the prefill row t = n of the same content."""
    rng = np.random.default_rng(21)
    L, H_I, d_I, H, D, D_v, k = 30, 2, 8, 3, 10, 6, 7
    _, _, _, _, _, keys, queries = _micro_inputs(rng, L, H_I, d_I, H, D)
    t = 25
    step_q = {"q_idx": queries["q_idx"][t:t + 1], "q_scale": None, "w": queries["w"][t:t + 1],
              "q": queries["q"][t:t + 1]}
    pre = O.prefill_rows(keys, step_q, [t], k, 0.5, D_v=D_v)
    dec = O.decode_row(keys, step_q, 0, t + 1, k, 0.5, D_v=D_v)
    assert np.array_equal(dec["idx"], pre["idx"][0])
    np.testing.assert_allclose(dec["out"], pre["out"][0], rtol=1e-14)


# ------------------------------------------------------------------------------------------ indexer KL objective
def test_indexer_kl_hand_worked():
    # velog.io page, Stage 1 Dense Warm-up: target p = the heads' attention summed and L1-normalised, loss
    # KL(p || Softmax(I)).  Two heads, three keys, scale 1.  Head 0 has logits (0, ln 2, ln 4): probabilities
    # (1, 2, 4) / 7; head 1 has logits 0: probabilities 1/3 each.  Summed: (10, 13, 19) / 21, L1-normalised:
    # p = (10, 13, 19) / 42.  I = (0, 0, ln 2): Softmax(I) = (1, 1, 2) / 4.
    q = np.array([[math.log(2.0), math.log(4.0)], [0.0, 0.0]])
    c = np.array([[0.0, 0.0], [1.0, 0.0], [0.0, 1.0]])
    I = np.array([0.0, 0.0, math.log(2.0)])
    want = (10 / 42) * math.log((10 / 42) / 0.25) + (13 / 42) * math.log((13 / 42) / 0.25) + \
        (19 / 42) * math.log((19 / 42) / 0.5)
    assert O.indexer_kl_row(I, q, c, 1.0) == pytest.approx(want, abs=1e-14)


def test_indexer_kl_zero_when_the_indexer_matches_the_target():
    rng = np.random.default_rng(11)
    q, c = rng.standard_normal((4, 16)), rng.standard_normal((30, 16))
    logits = 0.25 * q @ c.T
    P = np.exp(logits) / np.exp(logits).sum(axis=1, keepdims=True)
    p = P.sum(axis=0) / 4
    assert O.indexer_kl_row(np.log(p) + 7.5, q, c, 0.25) == pytest.approx(0.0, abs=1e-12)
    # any other I: strictly positive, and unchanged by a constant shift
    I = rng.standard_normal(30) * 3
    kl = O.indexer_kl_row(I, q, c, 0.25)
    assert kl > 1e-3
    assert O.indexer_kl_row(I - 40.0, q, c, 0.25) == pytest.approx(kl, rel=1e-12)
    assert O.indexer_kl_row(np.zeros(0), q, c[:0], 0.25) == 0.0


def test_indexer_kl_brute_force_loops():
    rng = np.random.default_rng(12)
    H, m, D = 3, 7, 5
    q, c, I = rng.standard_normal((H, D)), rng.standard_normal((m, D)), rng.standard_normal(m) * 2
    # pure-Python: each head's softmax, the sum over heads, its L1 normalisation, then the divergence
    p = [0.0] * m
    for h in range(H):
        lg = [0.4 * sum(q[h][d] * c[s][d] for d in range(D)) for s in range(m)]
        z = sum(math.exp(v) for v in lg)
        for s in range(m):
            p[s] += math.exp(lg[s]) / z
    tot = sum(p)
    p = [v / tot for v in p]
    zq = sum(math.exp(v) for v in I)
    want = sum(p[s] * math.log(p[s] / (math.exp(I[s]) / zq)) for s in range(m))
    assert O.indexer_kl_row(I, q, c, 0.4) == pytest.approx(want, rel=1e-12)
