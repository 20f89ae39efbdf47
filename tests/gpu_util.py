"""Helpers shared by the GPU parity tests: seeded inputs on the device, oracle rows on the host, metrics."""
import numpy as np
import torch

import dsa_inputs as G
import oracle as O

# Tolerances of the attention outputs against the fp64 oracle (fixed by the target of the build):
MAX_ABS = 2e-2
REL_L2 = 5e-3
RECALL = 0.995


def rel_l2(got, ref) -> float:
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def prefill_device(cfg, seed):
    """All inputs of one prefill sequence, generated on the GPU."""
    d = G.prefill_keys(cfg, seed, device="cuda")
    d.update(G.prefill_queries(cfg, seed, None, device="cuda"))
    return d


def oracle_prefill(cfg, seed, rows, want_attention=True, want_scores=False):
    """Oracle results for the given query rows (inputs regenerated on the host)."""
    keys = G.prefill_keys(cfg, seed)
    qs = G.prefill_queries(cfg, seed, rows=rows, with_q=want_attention)
    return O.prefill_rows(keys, qs, rows, cfg.k, cfg.scale, D_v=cfg.D_v, want_scores=want_scores,
                          want_attention=want_attention)


def recall(got_idx: np.ndarray, ref_idx: np.ndarray) -> float:
    """|got & ref| / |ref| over the valid (non -1) entries of one row."""
    ref = set(int(x) for x in ref_idx if x >= 0)
    got = set(int(x) for x in got_idx if x >= 0)
    return len(ref & got) / max(len(ref), 1)


def sample_rows(L, k, n_random, seed):
    """Row sample: edges (first rows, around k, tile boundaries, the last row) plus seeded random rows."""
    fixed = {0, 1, 63, 64, 127, 128, k - 2, k - 1, k, k + 1, L // 2, L - 2, L - 1}
    rng = np.random.default_rng(seed)
    rand = set(int(x) for x in rng.choice(L, size=min(n_random, L), replace=False))
    return sorted(r for r in fixed | rand if 0 <= r < L)
