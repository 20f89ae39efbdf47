"""Failure detection on the GPU without a fault: the library's bounded pipeline wait runs out on a barrier that
nothing arrives on, the kernel returns normally with DSA_ERR_TIMEOUT in the device status word, and the context
stays usable for the next call."""
import pytest
import torch

import dsa_inputs as G

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    import sparse_attention_long_05_b200 as dsa
    assert dsa.dsa_get_device_status() == 0
    res, status = dsa.dsa_check_bounded_wait()
    assert status == 5                                    # DSA_ERR_TIMEOUT
    ok0, t0, ok1, t1 = res.cpu().tolist()
    assert ok0 == 0 and ok1 == 0                         # neither wait claims success
    # warp 0 spent its whole budget (2^31 cycles = 2048 units of 2^20); warp 1, which started half a budget
    # later, left on the abort flag after about half a budget instead of its own full one
    assert 2040 <= t0 <= 2300
    assert 0 < t1 < 0.75 * t0
    # the status word was cleared by the read, and the context still runs the library's kernels
    assert dsa.dsa_get_device_status() == 0
    cfg = G.PREFILL_CONFIGS["tiny_1k"]
    x = G.prefill_inputs(cfg, 3, device="cuda")
    scores = dsa.dsa_indexer_scores(x["q_idx"][:8].contiguous(), None, x["k_idx"], None, x["w"][:8].contiguous())
    torch.cuda.synchronize()
    assert torch.isfinite(scores[:, :1]).all()
    assert dsa.dsa_get_device_status() == 0
