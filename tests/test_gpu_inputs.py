"""The seeded inputs are the same bits whether generated on the GPU (as the parity tests and the bench do) or on
the host (where the oracle regenerates the rows it checks)."""
import pytest
import torch

import dsa_inputs as G

pytestmark = pytest.mark.gpu


def _same(a, b):
    if a is None or b is None:
        return a is None and b is None
    a, b = a.cpu(), b.cpu()
    if a.dtype in (torch.float8_e4m3fn, torch.bfloat16):
        a, b = a.view(torch.uint8 if a.dtype == torch.float8_e4m3fn else torch.int16), \
            b.view(torch.uint8 if b.dtype == torch.float8_e4m3fn else torch.int16)
    return torch.equal(a, b)


@pytest.mark.parametrize("name", ["prefill_32k", "prefill_8k"])
def test_prefill_inputs_identical_on_both_devices(name):
    cfg = G.PREFILL_CONFIGS[name]
    rows = [0, 1, 2047, 5000, 8191]
    kg, kc = G.prefill_keys(cfg, 3, device="cuda"), G.prefill_keys(cfg, 3)
    for key in kg:
        assert _same(kg[key], kc[key]), key
    qg, qc = G.prefill_queries(cfg, 3, rows=rows, device="cuda"), G.prefill_queries(cfg, 3, rows=rows)
    for key in qg:
        assert _same(qg[key], qc[key]), key


def test_decode_inputs_identical_on_both_devices():
    cfg = G.DECODE_CONFIG
    seed = 44
    bg, bc = G.decode_step_batch(cfg, seed, 2, device="cuda", step0=254), G.decode_step_batch(cfg, seed, 2, step0=254)
    for key in bg:
        assert _same(bg[key], bc[key]), key
    rg, rc = G.decode_cache_rows(cfg, seed, 5, range(1000), device="cuda"), G.decode_cache_rows(cfg, seed, 5, range(1000))
    for key in rg:
        assert _same(rg[key], rc[key]), key
