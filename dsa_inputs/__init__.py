"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) forward path.

This module is the one thing the CPU oracle and the CUDA path share.  It holds no arithmetic of the method
itself (no scores, no selection, no attention); it only produces the tensors the method consumes:

* the lightning-indexer operands q_I [T, H_I, d_I], k_I [S, d_I] in FP8 e4m3 (plus a per-token fp32 scale
  in Gaussian mode) and the head weights w [T, H_I] in fp32;
* the MLA-in-MQA-mode operands: queries q [T, H, 576] and the shared latent entries c [S, 576], bf16.

Every element is a pure function of (seed, tensor id, flat element index).  A splitmix64-style finaliser
(Steele, Lea & Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) is evaluated with
int64 torch operations, whose wrap-around multiply, xor and masked shifts give the same bits on the CPU
and on a GPU.  Normal deviates come from a 65,536-entry table of the inverse normal CDF at the bin
midpoints (built once in fp64 on the host, rounded once to the target dtype on the host), indexed by 16
hash bits, so no transcendental function is evaluated on either device.  Any query row, key row or decode
step can therefore be regenerated on its own, which lets the oracle check sampled rows of a 128K-token
workload whose query tensor (19 GB) is generated on the GPU.

Recipes (input modes of the workloads):

* ``mode="int"``: q_I, k_I uniform integers in [-7, 7] stored exactly in e4m3; w uniform integers in
  [-3, 3].  Index scores are then exact integers below 2^24, so the selected sets are decided exactly.
* ``mode="gauss"``: q_I, k_I drawn N(0, 1) in fp32, then quantised to e4m3 with one fp32 scale per token
  (amax / 448, round-to-nearest-even, clamped to +-448); w drawn N(0, 1/H_I) in fp32.
* q and c: N(0, 1) rounded to bf16.
"""
from __future__ import annotations

import math
import statistics
from dataclasses import dataclass, field

import torch

__all__ = [
    "PrefillConfig", "DecodeConfig", "PREFILL_CONFIGS", "DECODE_CONFIG",
    "prefill_keys", "prefill_queries", "prefill_inputs",
    "decode_lengths", "decode_layout", "decode_cache_rows", "decode_fill_cache", "decode_step_inputs",
    "decode_step_batch",
    "hash64", "uniform_int", "normal_index",
]

_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
E4M3_MAX = 448.0

# tensor ids: one independent stream per tensor
_TID = {
    "q_idx": 1, "k_idx": 2, "w": 3, "q": 4, "c": 5,
    "dec_len": 16, "dec_q_idx": 17, "dec_w": 18, "dec_q": 19,
}


def _s64(x: int) -> int:
    """Two's-complement int64 value of a 64-bit pattern."""
    x &= _MASK64
    return x - (1 << 64) if x >> 63 else x


def _mix_int(x: int) -> int:
    """splitmix64 finaliser on a Python int (used once per stream to derive a key)."""
    x = (x + _GOLDEN) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def stream_key(seed: int, tensor: str) -> int:
    return _mix_int(_mix_int(seed & _MASK64) ^ (_TID[tensor] * 0xD1B54A32D192ED03 & _MASK64))


def _lsr(z: torch.Tensor, n: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return torch.bitwise_and(torch.bitwise_right_shift(z, n), (1 << (64 - n)) - 1)


def hash64(counter: torch.Tensor, key: int) -> torch.Tensor:
    """64 random bits (as int64) for each int64 counter, under a 64-bit stream key."""
    z = counter + _s64(key + _GOLDEN)
    z = torch.bitwise_xor(z, _lsr(z, 30)) * _s64(0xBF58476D1CE4E5B9)
    z = torch.bitwise_xor(z, _lsr(z, 27)) * _s64(0x94D049BB133111EB)
    return torch.bitwise_xor(z, _lsr(z, 31))


def uniform_int(bits: torch.Tensor, a: int) -> torch.Tensor:
    """Integers uniform in [-a, a] from the top 32 hash bits (multiply-shift range reduction)."""
    u = _lsr(bits, 32)
    return torch.bitwise_right_shift(u * (2 * a + 1), 32) - a


def normal_index(bits: torch.Tensor) -> torch.Tensor:
    """Index of a normal-table bin from the top 16 hash bits."""
    return _lsr(bits, 48)


_NORMAL_F64 = None
_TABLES: dict = {}


def _normal_table(dtype: torch.dtype, device) -> torch.Tensor:
    """Inverse normal CDF at bin midpoints (j + 1/2) / 65536, rounded once to ``dtype`` on the host."""
    global _NORMAL_F64
    if _NORMAL_F64 is None:
        nd = statistics.NormalDist()
        _NORMAL_F64 = torch.tensor([nd.inv_cdf((j + 0.5) / 65536.0) for j in range(65536)], dtype=torch.float64)
    key = (dtype, str(device))
    if key not in _TABLES:
        _TABLES[key] = _NORMAL_F64.to(dtype).to(device)
    return _TABLES[key]


def _counters(rows: torch.Tensor, row_len: int) -> torch.Tensor:
    return rows.to(torch.int64)[:, None] * row_len + torch.arange(row_len, dtype=torch.int64, device=rows.device)


def _rows_normal(key: int, rows: torch.Tensor, row_len: int, dtype: torch.dtype) -> torch.Tensor:
    idx = normal_index(hash64(_counters(rows, row_len), key))
    return _normal_table(dtype, rows.device)[idx]


def _rows_uniform(key: int, rows: torch.Tensor, row_len: int, a: int) -> torch.Tensor:
    return uniform_int(hash64(_counters(rows, row_len), key), a)


def quantise_e4m3_per_row(x: torch.Tensor):
    """fp32 rows -> (e4m3 rows, fp32 scale per row) with scale = amax / 448 (input recipe, not the method)."""
    amax = x.abs().amax(dim=1).clamp_min(1e-30)
    # tensor / tensor: a correctly rounded division on every device (a CUDA division by a Python scalar multiplies
    # by its reciprocal, which can differ in the last bit from the CPU's result)
    s = amax / torch.full_like(amax, E4M3_MAX)
    q = (x / s[:, None]).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return q, s


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    L: int
    H_I: int
    d_I: int
    k: int
    H: int
    D: int = 576
    D_v: int = 512
    mode: str = "int"

    @property
    def scale(self) -> float:
        return self.D ** -0.5


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    len_lo: int
    len_hi: int
    steps: int
    H_I: int = 64
    d_I: int = 128
    k: int = 2048
    H: int = 128
    D: int = 576
    D_v: int = 512
    mode: str = "gauss"

    @property
    def scale(self) -> float:
        return self.D ** -0.5


PREFILL_CONFIGS = {
    "tiny_1k": PrefillConfig("tiny_1k", L=1024, H_I=4, d_I=64, k=128, H=8),
    "prefill_8k": PrefillConfig("prefill_8k", L=8192, H_I=64, d_I=128, k=2048, H=128),
    "prefill_32k": PrefillConfig("prefill_32k", L=32768, H_I=64, d_I=128, k=2048, H=128, mode="gauss"),
    "prefill_128k": PrefillConfig("prefill_128k", L=131072, H_I=64, d_I=128, k=2048, H=128),
    "prefill_128k_gauss": PrefillConfig("prefill_128k_gauss", L=131072, H_I=64, d_I=128, k=2048, H=128,
                                        mode="gauss"),
}
DECODE_CONFIG = DecodeConfig("decode_64x128k", B=64, len_lo=4096, len_hi=131072, steps=256)


def _row_range(start: int, stop: int, device) -> torch.Tensor:
    return torch.arange(start, stop, dtype=torch.int64, device=device)


def _as_rows(rows, device) -> torch.Tensor:
    if isinstance(rows, torch.Tensor):
        return rows.to(device=device, dtype=torch.int64)
    return torch.as_tensor(list(rows), dtype=torch.int64, device=device)


def _indexer_rows(key: int, rows: torch.Tensor, width: int, mode: str, int_range: int = 7):
    """e4m3 rows (+ per-row scale in Gaussian mode) for q_I (width H_I*d_I) or k_I (width d_I)."""
    if mode == "int":
        v = _rows_uniform(key, rows, width, int_range).to(torch.float32)
        return v.to(torch.float8_e4m3fn), None
    if mode == "gauss":
        return quantise_e4m3_per_row(_rows_normal(key, rows, width, torch.float32))
    raise ValueError(f"unknown indexer input mode {mode!r}")


def _weights(key: int, rows: torch.Tensor, H_I: int, mode: str) -> torch.Tensor:
    if mode == "int":
        return _rows_uniform(key, rows, H_I, 3).to(torch.float32)
    return _rows_normal(key, rows, H_I, torch.float32) * torch.tensor(H_I ** -0.5, dtype=torch.float32)


def prefill_keys(cfg: PrefillConfig, seed: int, device="cpu", chunk_rows: int = 16384):
    """Key-side tensors of one prefill sequence: k_idx [L, d_I] e4m3, k_scale [L] or None, c [L, 576] bf16."""
    k_idx = torch.empty((cfg.L, cfg.d_I), dtype=torch.float8_e4m3fn, device=device)
    k_scale = torch.empty((cfg.L,), dtype=torch.float32, device=device) if cfg.mode == "gauss" else None
    c = torch.empty((cfg.L, cfg.D), dtype=torch.bfloat16, device=device)
    kk, kc = stream_key(seed, "k_idx"), stream_key(seed, "c")
    for r0 in range(0, cfg.L, chunk_rows):
        rows = _row_range(r0, min(cfg.L, r0 + chunk_rows), device)
        q8, s = _indexer_rows(kk, rows, cfg.d_I, cfg.mode)
        k_idx[r0:r0 + len(rows)] = q8
        if k_scale is not None:
            k_scale[r0:r0 + len(rows)] = s
        c[r0:r0 + len(rows)] = _rows_normal(kc, rows, cfg.D, torch.bfloat16)
    return {"k_idx": k_idx, "k_scale": k_scale, "c": c}


def prefill_queries(cfg: PrefillConfig, seed: int, rows=None, device="cpu", chunk_rows: int = 2048,
                    with_q: bool = True):
    """Query-side tensors for the given query rows (default: all L rows, in order).

    Returns q_idx [R, H_I, d_I] e4m3, q_scale [R] or None, w [R, H_I] fp32 and (with_q) q [R, H, 576] bf16.
    """
    rows_t = _row_range(0, cfg.L, device) if rows is None else _as_rows(rows, device)
    R = rows_t.numel()
    q_idx = torch.empty((R, cfg.H_I, cfg.d_I), dtype=torch.float8_e4m3fn, device=device)
    q_scale = torch.empty((R,), dtype=torch.float32, device=device) if cfg.mode == "gauss" else None
    w = torch.empty((R, cfg.H_I), dtype=torch.float32, device=device)
    q = torch.empty((R, cfg.H, cfg.D), dtype=torch.bfloat16, device=device) if with_q else None
    kq, kw, kqq = stream_key(seed, "q_idx"), stream_key(seed, "w"), stream_key(seed, "q")
    for r0 in range(0, R, chunk_rows):
        rr = rows_t[r0:r0 + chunk_rows]
        n = rr.numel()
        q8, s = _indexer_rows(kq, rr, cfg.H_I * cfg.d_I, cfg.mode)
        q_idx[r0:r0 + n] = q8.view(n, cfg.H_I, cfg.d_I)
        if q_scale is not None:
            q_scale[r0:r0 + n] = s
        w[r0:r0 + n] = _weights(kw, rr, cfg.H_I, cfg.mode)
        if with_q:
            q[r0:r0 + n] = _rows_normal(kqq, rr, cfg.H * cfg.D, torch.bfloat16).view(n, cfg.H, cfg.D)
    return {"q_idx": q_idx, "q_scale": q_scale, "w": w, "q": q}


def prefill_inputs(cfg: PrefillConfig, seed: int, device="cpu"):
    """All tensors of one prefill sequence (query rows 0..L-1)."""
    out = prefill_keys(cfg, seed, device)
    out.update(prefill_queries(cfg, seed, None, device))
    return out


# ---------------------------------------------------------------------------------------------- decode
_DEC_ROW_STRIDE = 1 << 18  # > max context + steps; decouples row content from the cache layout


def decode_lengths(cfg: DecodeConfig, seed: int) -> list:
    """Context length n_b (before the first step) of each sequence, uniform in [len_lo, len_hi]."""
    bits = hash64(torch.arange(cfg.B, dtype=torch.int64), stream_key(seed, "dec_len"))
    u = _lsr(bits, 32)
    span = cfg.len_hi - cfg.len_lo + 1
    return (cfg.len_lo + torch.bitwise_right_shift(u * span, 32)).tolist()


def decode_layout(cfg: DecodeConfig, seed: int):
    """(lengths n_b, cache row offsets, total cache rows): sequence b owns rows [off_b, off_b + n_b + steps)."""
    lens = decode_lengths(cfg, seed)
    offs, tot = [], 0
    for n in lens:
        offs.append(tot)
        tot += n + cfg.steps
    return lens, offs, tot


def decode_cache_rows(cfg: DecodeConfig, seed: int, b: int, positions, device="cpu"):
    """Cache content at the given positions of sequence b (prefix rows and rows appended at later steps).

    Returns k_idx [R, d_I] e4m3, k_scale [R] or None, c [R, 576] bf16.
    """
    pos = _as_rows(positions, device)
    gid = b * _DEC_ROW_STRIDE + pos
    q8, s = _indexer_rows(stream_key(seed, "k_idx"), gid, cfg.d_I, cfg.mode)
    c = _rows_normal(stream_key(seed, "c"), gid, cfg.D, torch.bfloat16)
    return {"k_idx": q8, "k_scale": s, "c": c}


def decode_fill_cache(cfg: DecodeConfig, seed: int, device="cpu", chunk_rows: int = 32768):
    """Allocate the flat caches (capacity n_b + steps per sequence) and fill each sequence's first n_b rows."""
    lens, offs, tot = decode_layout(cfg, seed)
    k_cache = torch.zeros((tot, cfg.d_I), dtype=torch.float8_e4m3fn, device=device)
    k_scale = torch.zeros((tot,), dtype=torch.float32, device=device)
    c_cache = torch.zeros((tot, cfg.D), dtype=torch.bfloat16, device=device)
    for b, (n, o) in enumerate(zip(lens, offs)):
        for p0 in range(0, n, chunk_rows):
            p1 = min(n, p0 + chunk_rows)
            r = decode_cache_rows(cfg, seed, b, _row_range(p0, p1, device), device)
            k_cache[o + p0:o + p1] = r["k_idx"]
            if r["k_scale"] is not None:
                k_scale[o + p0:o + p1] = r["k_scale"]
            else:
                k_scale[o + p0:o + p1] = 1.0
            c_cache[o + p0:o + p1] = r["c"]
    return {"k_cache": k_cache, "k_scale_cache": k_scale, "c_cache": c_cache,
            "lens": lens, "offs": offs, "rows": tot}


def decode_step_inputs(cfg: DecodeConfig, seed: int, step: int, device="cpu", seqs=None):
    """New-token tensors of one decode step for the given sequences (default all B).

    The new key-side entries are the cache rows at position n_b + step, so the cache after the append
    equals ``decode_cache_rows`` over positions 0..n_b+step.
    """
    lens = decode_lengths(cfg, seed)
    seqs = list(range(cfg.B)) if seqs is None else list(seqs)
    tok = torch.as_tensor([step * cfg.B + b for b in seqs], dtype=torch.int64, device=device)
    q8, qs = _indexer_rows(stream_key(seed, "dec_q_idx"), tok, cfg.H_I * cfg.d_I, cfg.mode)
    w = _weights(stream_key(seed, "dec_w"), tok, cfg.H_I, cfg.mode)
    q = _rows_normal(stream_key(seed, "dec_q"), tok, cfg.H * cfg.D, torch.bfloat16).view(len(seqs), cfg.H, cfg.D)
    kn = {"k_idx": [], "k_scale": [], "c": []}
    for b in seqs:
        r = decode_cache_rows(cfg, seed, b, [lens[b] + step], device)
        for key in kn:
            kn[key].append(r[key])
    k_new = torch.cat(kn["k_idx"])
    k_scale_new = torch.cat(kn["k_scale"]) if cfg.mode == "gauss" else torch.ones(len(seqs), device=device)
    return {"q_idx": q8.view(len(seqs), cfg.H_I, cfg.d_I), "q_scale": qs, "w": w, "q": q,
            "k_new": k_new, "k_scale_new": k_scale_new, "c_new": torch.cat(kn["c"])}


def decode_step_batch(cfg: DecodeConfig, seed: int, steps: int, device="cpu", step0: int = 0):
    """New-token tensors of decode steps step0..step0+steps-1 for all B sequences, stacked on a step axis.

    Element for element identical to ``decode_step_inputs(cfg, seed, step)`` for each step.
    """
    lens = decode_lengths(cfg, seed)
    B = cfg.B
    tok = torch.arange(step0 * B, (step0 + steps) * B, dtype=torch.int64, device=device)   # step * B + b
    q8, qs = _indexer_rows(stream_key(seed, "dec_q_idx"), tok, cfg.H_I * cfg.d_I, cfg.mode)
    w = _weights(stream_key(seed, "dec_w"), tok, cfg.H_I, cfg.mode)
    q = _rows_normal(stream_key(seed, "dec_q"), tok, cfg.H * cfg.D, torch.bfloat16)
    b = tok % B
    pos = torch.as_tensor(lens, dtype=torch.int64, device=device)[b] + tok // B
    gid = b * _DEC_ROW_STRIDE + pos
    k8, ks = _indexer_rows(stream_key(seed, "k_idx"), gid, cfg.d_I, cfg.mode)
    c = _rows_normal(stream_key(seed, "c"), gid, cfg.D, torch.bfloat16)
    if ks is None:
        ks = torch.ones(steps * B, dtype=torch.float32, device=device)
    return {"q_idx": q8.view(steps, B, cfg.H_I, cfg.d_I), "q_scale": None if qs is None else qs.view(steps, B),
            "w": w.view(steps, B, cfg.H_I), "q": q.view(steps, B, cfg.H, cfg.D),
            "k_new": k8.view(steps, B, cfg.d_I), "k_scale_new": ks.view(steps, B), "c_new": c.view(steps, B, cfg.D)}
