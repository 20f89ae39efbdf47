"""CPU oracle of the DeepSeek Sparse Attention (DSA) forward path, in fp64.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or execute this module: it is used by
``tests/``, by ``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py``.  It shares no code with the CUDA path (``sparse_attention_long_05_b200``); its inputs come
from the seeded generator ``dsa_inputs`` or are written by hand in the tests.

What it computes follows "DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models" as summarised
on the velog.io page (DeepSeek Sparse Attention, §1.1-§1.3) and the yuuk.io notes (提案手法 / DSA):

* §1.1 Lightning Indexer, the index score:  I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]), over the
  H_I indexer heads j, for previous tokens s of the query token t (read as s <= t).
* §1.2 Fine-grained token selection: keep the KV entries c_s whose I[t,s] is among the top-k of row t;
  u_t = Attn(h_t, {c_s : s selected}).  k = 2048 (velog.io Stage 2; aisparkup.com; macaron.im).
* §1.3 MLA in MQA mode: every latent entry c_s (one vector per token) is shared by all query heads, so
  u_t[h] = softmax_s(scale * q[t,h] . c_s) . c_s[:D_v] over the selected s.
* Stage 1 (dense warm-up) training objective of the indexer: the target p_{t,:} is the main attention's
  probabilities summed over the heads and L1-normalised, and L_I = sum_t KL(p_{t,:} || Softmax(I_{t,:})).

Readings where the pages are silent:
* causal includes s = t; when t + 1 <= k every s <= t is selected; the output index list is in ascending s
  and padded with -1;
* ties in the top-k are broken by the smaller s (a total order on (score desc, s asc) makes the set unique);
  -0.0 and +0.0 compare equal;
* FP8 means e4m3fn (bias 7, no infinities, 0x7F/0xFF are NaN, largest finite 448); in Gaussian mode q_I is
  dequantised with one fp32 scale per query token and k_I with one per key token;
* the value of an entry is its first D_v = 512 of D = 576 dims, the softmax scale is D^-1/2, and lse is the
  natural-log log-sum-exp of the scaled logits;
* a row with no selected entry has output 0 and lse = -inf.

Every function is the plain definition written out in fp64: library primitives (matmul, sort, exp) serve
as single steps, with no blocking, fusion or reordering beyond what the definition states.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "e4m3_table", "e4m3_to_f64", "bf16_to_f64", "f32_to_f64",
    "indexer_scores_row", "topk_row", "attention_row", "prefill_rows", "decode_row", "indexer_kl_row",
]


def e4m3_table() -> np.ndarray:
    """fp64 value of every e4m3fn bit pattern, from the format definition (sign, 4-bit exponent with bias
    7, 3-bit mantissa; exponent 0 is subnormal; S.1111.111 is NaN; no infinities)."""
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            out[code] = np.nan
        elif e == 0:
            out[code] = sign * 2.0 ** (1 - 7) * (m / 8.0)
        else:
            out[code] = sign * 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return out


_E4M3 = e4m3_table()


def e4m3_to_f64(bits) -> np.ndarray:
    """Decode uint8 e4m3fn bit patterns to fp64 values."""
    return _E4M3[np.asarray(bits, dtype=np.uint8)]


def bf16_to_f64(bits) -> np.ndarray:
    """Widen uint16 bf16 bit patterns exactly to fp64 (a bf16 is the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f32_to_f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def indexer_scores_row(qI_t: np.ndarray, w_t: np.ndarray, kI: np.ndarray) -> np.ndarray:
    """Index scores of one query token against the given key rows (velog.io §1.1 Lightning Indexer).

    qI_t: [H_I, d_I] dequantised indexer queries of token t; w_t: [H_I] head weights of token t;
    kI: [n, d_I] dequantised indexer keys of the rows s to score.  Returns I[t, s] for those rows, [n].
    """
    x = kI @ qI_t.T                    # x[s, j] = q_I[t,j] . k_I[s]
    return np.maximum(x, 0.0) @ w_t    # sum_j w[t,j] * ReLU(x[s, j])


def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Top-k selection of one row (velog.io §1.2): the min(k, n) positions s of largest I[t, s], ties broken
    by the smaller s.  Returned in ascending s, padded with -1 to length k."""
    n = scores.shape[0]
    s = np.arange(n)
    order = np.lexsort((s, -scores))   # primary: score descending; secondary: s ascending
    sel = np.sort(order[:min(k, n)])
    out = np.full(k, -1, dtype=np.int32)
    out[:sel.shape[0]] = sel
    return out


def attention_row(q_t: np.ndarray, c_sel: np.ndarray, scale: float, D_v: int):
    """MLA in MQA mode over the selected latent entries (velog.io §1.2-§1.3).

    q_t: [H, D] queries of token t; c_sel: [m, D] the selected shared latent entries.  Every head attends to
    the same entries; logits are scale * q[h] . c_s over all D dims, values are c_s[:D_v].
    Returns (u [H, D_v], lse [H]).
    """
    H = q_t.shape[0]
    if c_sel.shape[0] == 0:
        return np.zeros((H, D_v)), np.full(H, -np.inf)
    logits = scale * (q_t @ c_sel.T)                  # [H, m]
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)                           # subtracting the row max is exact in real arithmetic
    l = p.sum(axis=1, keepdims=True)
    u = (p @ c_sel[:, :D_v]) / l
    lse = (mx + np.log(l))[:, 0]
    return u, lse


def indexer_kl_row(I_keys: np.ndarray, q_t: np.ndarray, c_keys: np.ndarray, scale: float) -> float:
    """KL(p_t || Softmax(I_t)) of one query token over a set of keys (velog.io page, Stage 1 Dense Warm-up: the
    target is the main attention heads' scores summed and L1-normalised; the loss is the KL divergence of the
    indexer's output distribution from it).

    I_keys: [m] index scores I[t, s] of the keys; q_t: [H, D] queries of token t; c_keys: [m, D] the keys' shared
    latent entries (all D dims enter the logits, as in attention_row).  The keys are all s <= t in the dense
    warm-up; over a selected set S_t both distributions are taken over S_t.  Returns the divergence in nats (0 for
    an empty set).
    """
    m = I_keys.shape[0]
    if m == 0:
        return 0.0
    logits = scale * (q_t @ c_keys.T)                 # [H, m]
    P = np.exp(logits - logits.max(axis=1, keepdims=True))
    P = P / P.sum(axis=1, keepdims=True)              # each head's attention distribution over the keys
    a = P.sum(axis=0)                                 # summed over the heads ...
    p = a / a.sum()                                   # ... and L1-normalised: the target p_{t,:}
    mI = I_keys.max()
    log_q = I_keys - (mI + np.log(np.exp(I_keys - mI).sum()))   # log Softmax(I_{t,:})
    nz = p > 0                                        # 0 log 0 = 0
    return float((p[nz] * (np.log(p[nz]) - log_q[nz])).sum())


def _dequant(bits, scale=None):
    v = e4m3_to_f64(bits)
    if scale is not None:
        v = v * f32_to_f64(scale).reshape((-1,) + (1,) * (v.ndim - 1))
    return v


def _np(t):
    """uint8 / uint16 / fp32 numpy view of a CPU torch tensor (or pass-through for numpy arrays)."""
    if t is None or isinstance(t, np.ndarray):
        return t
    import torch
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def prefill_rows(keys: dict, queries: dict, positions, k: int, scale: float, D_v: int = 512,
                 want_scores: bool = False, want_attention: bool = True):
    """The whole forward path for a set of query rows of one causal prefill sequence.

    keys: {"k_idx": e4m3 [L, d_I], "k_scale": fp32 [L] or None, "c": bf16 [L, D]};
    queries: {"q_idx": e4m3 [R, H_I, d_I], "q_scale": fp32 [R] or None, "w": fp32 [R, H_I],
    "q": bf16 [R, H, D] (optional)} for query rows at absolute positions ``positions`` [R].
    Returns {"idx": int32 [R, k], "out": [R, H, D_v], "lse": [R, H], "scores": list of [t+1] rows}.
    """
    positions = [int(p) for p in positions]
    kI = _dequant(_np(keys["k_idx"]), _np(keys["k_scale"]))
    qI = _dequant(_np(queries["q_idx"]), _np(queries["q_scale"]))
    w = f32_to_f64(_np(queries["w"]))
    c = bf16_to_f64(_np(keys["c"])) if want_attention else None
    q = bf16_to_f64(_np(queries["q"])) if want_attention else None
    R = len(positions)
    if qI.shape[0] != R or w.shape[0] != R or (q is not None and q.shape[0] != R):
        raise ValueError("queries must hold exactly one row per entry of positions")
    idx = np.empty((R, k), dtype=np.int32)
    out = lse = None
    if want_attention:
        out = np.empty((R, q.shape[1], D_v))
        lse = np.empty((R, q.shape[1]))
    scores = []
    for r, t in enumerate(positions):
        I = indexer_scores_row(qI[r], w[r], kI[:t + 1])
        if want_scores:
            scores.append(I)
        idx[r] = topk_row(I, k)
        if want_attention:
            sel = idx[r][idx[r] >= 0]
            out[r], lse[r] = attention_row(q[r], c[sel], scale, D_v)
    return {"idx": idx, "out": out, "lse": lse, "scores": scores}


def decode_row(cache: dict, step_q: dict, b: int, n_keys: int, k: int, scale: float, D_v: int = 512):
    """One decode token of sequence b against its cache positions 0..n_keys-1 (after the append).

    cache: {"k_idx": e4m3 [n_keys, d_I], "k_scale": fp32 [n_keys] or None, "c": bf16 [n_keys, D]} (rows of
    sequence b only); step_q: the new-token query tensors of all sequences ({"q_idx", "q_scale", "w", "q"}).
    """
    qs = _np(step_q["q_scale"])
    qI = _dequant(_np(step_q["q_idx"])[b:b + 1], None if qs is None else qs[b:b + 1])[0]
    w = f32_to_f64(_np(step_q["w"])[b])
    kI = _dequant(_np(cache["k_idx"])[:n_keys], None if cache["k_scale"] is None else _np(cache["k_scale"])[:n_keys])
    I = indexer_scores_row(qI, w, kI)
    idx = topk_row(I, k)
    sel = idx[idx >= 0]
    c = bf16_to_f64(_np(cache["c"])[sel])
    q = bf16_to_f64(_np(step_q["q"])[b])
    out, lse = attention_row(q, c, scale, D_v)
    return {"idx": idx, "out": out, "lse": lse, "scores": I}
