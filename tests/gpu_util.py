"""Helpers shared by the GPU parity tests: seeded inputs on the device, oracle rows on the host, metrics."""
import numpy as np
import torch

import dsa_inputs as G
import oracle as O

# Tolerances of the attention outputs against the fp64 oracle (fixed by the target of the build):
MAX_ABS = 2e-2
REL_L2 = 5e-3
RECALL = 0.995


def e2e_bound(mean_recall: float) -> float:
    """Bound on the end-to-end relative-L2 error of Gaussian-mode outputs against the oracle's own selection,
    given the measured recall.  The attention weight of a key is independent of its index score, so a swapped
    key (a fraction f = 1 - recall of the k selected) is a random draw from the same weight distribution as the
    key it replaced.  With logits x ~ N(0, 1), sum_i p_i^2 = e / k per output dimension, so swapping m = f k
    keys moves the output by sqrt(2 m e) / k against an output of sqrt(e / k): a relative-L2 of sqrt(2 f).
    The bound allows 1.5 times that (the swap count and the weights fluctuate) plus the attention tolerance."""
    return 1.5 * float(np.sqrt(2.0 * max(0.0, 1.0 - mean_recall))) + REL_L2


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
