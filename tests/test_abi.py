"""The C-ABI library (no GPU needed): it builds, loads, exports every declared symbol, and its host-side
argument checks reject bad calls before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return re.findall(r"DSA_API\s+[\w\s\*]*?\b(dsa_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "dsa_build", os.path.join(ROOT, "sparse_attention_long_05_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    from sparse_attention_long_05_b200 import _lib
    return _lib._lib


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    from sparse_attention_long_05_b200._lib import SIGNATURES
    for n in names:
        assert hasattr(lib, n), n
        assert n in SIGNATURES, n


def test_status_strings(lib):
    for code, name in [(0, b"DSA_OK"), (2, b"DSA_ERR_UNSUPPORTED_SHAPE"), (5, b"DSA_ERR_TIMEOUT"),
                       (7, b"DSA_ERR_WORKSPACE"), (8, b"DSA_ERR_CHECK"), (99, b"DSA_UNKNOWN_STATUS")]:
        assert lib.dsa_status_string(code) == name


def test_checking_build_exports_the_same_entry_points(lib):
    """The -DDSA_CHECKS build (libdsa_checks.so) is a drop-in for libdsa.so; only it reports checks enabled."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "dsa_build", os.path.join(ROOT, "sparse_attention_long_05_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    from sparse_attention_long_05_b200 import _lib
    chk = _lib.load(b.build_checks())
    for n in _declared():
        assert hasattr(chk, n), n
    assert chk.dsa_checks_enabled() == 1 and lib.dsa_checks_enabled() == 0
    assert chk.dsa_status_string(8) == b"DSA_ERR_CHECK"


def test_workspace_sizes(lib):
    assert lib.dsa_prefill_workspace_size(0, 64, 128, 128, 2048) == 0
    w8 = lib.dsa_prefill_workspace_size(8192, 64, 128, 128, 2048)
    assert w8 >= 8192 * 2048 * 4 and w8 % 256 == 0
    w128 = lib.dsa_prefill_workspace_size(131072, 64, 128, 128, 2048)
    assert w128 <= (1 << 30) + 131072 * 2048 * 4 + 512      # never the L x L score matrix
    assert lib.dsa_decode_workspace_size(64, 1 << 20, 64, 128, 128, 2048) >= (1 << 20) * 4 + 64 * 2048 * 4


def test_host_argument_checks(lib):
    P = ctypes.c_void_p
    one = P(16)  # a dummy aligned non-null address: every call below must fail before touching it
    # unsupported indexer shape
    assert lib.dsa_indexer_scores(one, None, one, None, one, 4, 4, 32, 128, 0, one, None) == 2
    # negative sizes / null outputs
    assert lib.dsa_indexer_scores(one, None, one, None, one, -1, 4, 64, 128, 0, one, None) == 1
    assert lib.dsa_topk(None, 3, 10, None, 0, 4, one, None) == 1
    assert lib.dsa_topk(one, 3, 10, None, 0, 0, one, None) == 1
    # misaligned TMA operand
    assert lib.dsa_indexer_scores(P(17), None, one, None, one, 4, 4, 64, 128, 0, one, None) == 3
    # attention: too many heads, k not a multiple of 64
    assert lib.dsa_sparse_mla_attn(one, one, 10, one, 2, 129, 64, 1.0, one, None, None) == 2
    assert lib.dsa_sparse_mla_attn(one, one, 10, one, 2, 8, 100, 1.0, one, None, None) == 2
    # prefill without a big enough workspace
    assert lib.dsa_forward_prefill(one, None, one, None, one, one, one, 1024, 4, 64, 8, 128, 1.0, None, one, None,
                                   one, 16, None) == 7
    # decode: only H_I = 64 / d_I = 128
    assert lib.dsa_forward_decode(2, one, one, one, None, one, one, one, one, one, one, one, one, 100, 4, 64, 8, 128,
                                  1.0, None, one, None, one, 1 << 20, None) == 2
    # varlen prefill: malformed cu_seqlens (first entry not 0, decreasing, empty batch)
    cu = (ctypes.c_int64 * 3)(0, 100, 50)
    assert lib.dsa_forward_prefill_varlen(2, ctypes.cast(cu, P), one, None, one, None, one, one, one, 64, 128, 128,
                                          2048, 1.0, None, one, None, one, 1 << 30, None) == 1
    cu = (ctypes.c_int64 * 2)(5, 100)
    assert lib.dsa_forward_prefill_varlen(1, ctypes.cast(cu, P), one, None, one, None, one, one, one, 64, 128, 128,
                                          2048, 1.0, None, one, None, one, 1 << 30, None) == 1
    cu = (ctypes.c_int64 * 2)(0, 0)
    assert lib.dsa_forward_prefill_varlen(1, ctypes.cast(cu, P), one, None, one, None, one, one, one, 64, 128, 128,
                                          2048, 1.0, None, one, None, one, 1 << 30, None) == 1
    # ... an unsupported shape, and a workspace below dsa_prefill_varlen_workspace_size
    cu = (ctypes.c_int64 * 3)(0, 100, 300)
    assert lib.dsa_forward_prefill_varlen(2, ctypes.cast(cu, P), one, None, one, None, one, one, one, 4, 128, 128,
                                          2048, 1.0, None, one, None, one, 1 << 30, None) == 2
    assert lib.dsa_forward_prefill_varlen(2, ctypes.cast(cu, P), one, None, one, None, one, one, one, 64, 128, 128,
                                          2048, 1.0, None, one, None, one, 16, None) == 7
    assert lib.dsa_prefill_varlen_workspace_size(2, 300, 200, 64, 128, 128, 2048) >= 300 * 2048 * 4 + 300 * 8
    # bounded-wait self-check: null or misaligned result array
    assert lib.dsa_check_bounded_wait(None, None) == 1
    assert lib.dsa_check_bounded_wait(P(20), None) == 3
    # empty work is a no-op
    assert lib.dsa_indexer_scores(one, None, one, None, one, 0, 4, 64, 128, 0, one, None) == 0
    assert lib.dsa_sparse_mla_attn(None, None, 10, None, 0, 8, 128, 1.0, None, None, None) == 0


def test_prefill_block_schedule(lib):
    # dsa_prefill_block_rows (host only): the blocks tile [0, L) in order; rows t < k form the first block; every
    # later block's scores (rows x keys up to its end) fit the workspace's prefill_chunk_rows(L) x L scores, and
    # blocks get no longer as their key ranges grow
    for L, k in ((1024, 128), (1500, 2048), (8192, 2048), (32768, 2048), (131072, 2048), (300000, 2048)):
        cap = (lib.dsa_prefill_workspace_size(L, 64, 128, 128, k) - (((L * k * 4) + 255) // 256) * 256) // 4
        r0, blocks = 0, []
        while r0 < L:
            n = lib.dsa_prefill_block_rows(L, k, r0)
            assert n >= 1
            blocks.append((r0, n))
            r0 += n
        assert r0 == L
        assert blocks[0] == (0, min(k, L))
        for (a, n), (b, m) in zip(blocks[1:], blocks[2:]):
            assert b == a + n and m <= n
        for a, n in blocks[1:]:
            assert n * (a + n) <= cap
    assert lib.dsa_prefill_block_rows(100, 10, 100) == 0 and lib.dsa_prefill_block_rows(0, 10, 0) == 0
