"""The tolerance the Gaussian-mode GPU tests derive from recall (gpu_util.e2e_bound), checked on the CPU by
simulation: swapping a fraction f of the k selected latent entries for unselected ones (keys whose attention
weights are unrelated to the swap, as for a borderline index score) moves the fp64 attention output by a
relative-L2 of about sqrt(2 f), and stays under the bound."""
import numpy as np
import pytest

import oracle as O
from gpu_util import REL_L2, e2e_bound


@pytest.mark.parametrize("f", [0.005, 0.02])
def test_swap_error_scales_as_sqrt_two_f(f):
    rng = np.random.default_rng(5)
    k, D, D_v, H, pool = 2048, 576, 512, 16, 6144
    m = int(round(f * k))
    errs = []
    for trial in range(6):
        c = rng.standard_normal((pool, D))
        q = rng.standard_normal((H, D))
        sel = rng.choice(pool, size=k, replace=False)
        rest = np.setdiff1d(np.arange(pool), sel)
        swapped = sel.copy()
        swapped[rng.choice(k, size=m, replace=False)] = rng.choice(rest, size=m, replace=False)
        a = O.attention_row(q, c[sel], D ** -0.5, D_v)[0]
        b = O.attention_row(q, c[swapped], D ** -0.5, D_v)[0]
        errs.append(np.linalg.norm(a - b) / np.linalg.norm(a))
    pred = np.sqrt(2 * f)
    assert 0.6 * pred <= np.mean(errs) <= 1.4 * pred, (np.mean(errs), pred)
    assert max(errs) <= e2e_bound(1.0 - f)


def test_bound_reduces_to_the_attention_tolerance_at_full_recall():
    assert e2e_bound(1.0) == REL_L2
    assert e2e_bound(0.995) == pytest.approx(1.5 * 0.1 + REL_L2)
