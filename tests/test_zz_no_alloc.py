"""dsa_forward_decode_noalloc: the decode step for callers that cannot allocate device memory (its scratch is
a fixed array inside the library).  Its results must match dsa_forward_decode's on the same inputs, on two
calls in a row (the second call reuses the array the first one left behind).  This file is collected last so
that a run stopping at the first failure has run every other test first."""
import pytest
import torch

import dsa_inputs as G

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice():
    import sparse_attention_long_05_b200 as dsa
    cfg = G.DecodeConfig("noalloc", B=8, len_lo=3000, len_hi=40000, steps=4)
    seed = 77
    cache = G.decode_fill_cache(cfg, seed, device="cuda")
    cache_off = torch.tensor(cache["offs"], dtype=torch.int64, device="cuda")
    ctx = torch.tensor(cache["lens"], dtype=torch.int32, device="cuda")
    need = dsa.dsa_decode_workspace_size(cfg.B, cache["rows"], cfg.H_I, cfg.d_I, cfg.H, cfg.k)
    assert need <= dsa.dsa_decode_noalloc_scratch_bytes()
    for step in range(2):
        st = G.decode_step_inputs(cfg, seed, step, device="cuda")
        args = (cache_off, ctx, st["q_idx"], st["q_scale"], st["w"], st["q"], st["k_new"], st["k_scale_new"],
                st["c_new"], cache["k_cache"], cache["k_scale_cache"], cache["c_cache"], cfg.k, cfg.scale)
        ref_idx, ref_out, ref_lse = dsa.dsa_forward_decode(*args)
        got_idx, got_out, got_lse = dsa.dsa_forward_decode_noalloc(*args)
        assert dsa.dsa_get_device_status() == 0
        # both entry points launch the same kernels on the same inputs, so the results are identical
        assert torch.equal(got_idx, ref_idx)
        assert torch.equal(got_out, ref_out)
        assert torch.equal(got_lse, ref_lse)
        ctx += 1


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import ctypes
    import sparse_attention_long_05_b200 as dsa
    from sparse_attention_long_05_b200 import _lib
    one = ctypes.c_void_p(16)
    rows = dsa.dsa_decode_noalloc_scratch_bytes() // 4 + 1       # more score rows than the array holds
    rc = _lib._lib.dsa_forward_decode_noalloc(4, one, one, one, None, one, one, one, one, one, one, one, one, rows,
                                              64, 128, 128, 2048, 1.0, None, one, None, None)
    assert rc == 7     # DSA_ERR_WORKSPACE, nothing launched
    # argument and shape errors are reported as dsa_forward_decode reports them, whatever the size
    rc = _lib._lib.dsa_forward_decode_noalloc(4, one, None, one, None, one, one, one, one, one, one, one, one, rows,
                                              64, 128, 128, 2048, 1.0, None, one, None, None)
    assert rc == 1     # DSA_ERR_INVALID_ARG (null ctx_len)
    rc = _lib._lib.dsa_forward_decode_noalloc(2000, one, one, one, None, one, one, one, one, one, one, one, one,
                                              rows, 64, 128, 128, 2048, 1.0, None, one, None, None)
    assert rc == 2     # DSA_ERR_UNSUPPORTED_SHAPE (more sequences than a decode step takes)
