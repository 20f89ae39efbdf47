"""ctypes binding of libdsa.so: argument marshalling only.

Each function has the name of the C entry point it wraps (include/dsa.h), takes torch CUDA tensors, passes
their device pointers, sizes and the current CUDA stream, and raises DsaError for a non-OK status.  Every
step of the computation runs in libdsa.so's kernels; there is no fallback: importing this module fails
loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")
CHECKS_LIB_PATH = os.path.join(_HERE, "libdsa_checks.so")   # the -DDSA_CHECKS build (debugging)

_STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED_SHAPE", 3: "DSA_ERR_ALIGNMENT",
           4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_BAD_INDEX", 7: "DSA_ERR_WORKSPACE",
           8: "DSA_ERR_CHECK"}

# exported symbols and their C signatures
_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "dsa_status_string": (ctypes.c_char_p, [_I]),
    "dsa_get_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_int)]),
    "dsa_check_bounded_wait": (_I, [_P, _P]),
    "dsa_num_sms": (_I, []),
    "dsa_checks_enabled": (_I, []),
    "dsa_checks_selftest_bytes": (_SZ, []),
    "dsa_checks_selftest": (_I, [_I, _P, _P]),
    "dsa_indexer_scores": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "dsa_topk": (_I, [_P, _I, _I64, _P, _I, _I, _P, _P]),
    "dsa_sparse_mla_attn": (_I, [_P, _P, _I, _P, _I, _I, _I, _F, _P, _P, _P]),
    "dsa_indexer_kl": (_I, [_P, _P, _I, _P, _P, _P, _I, _I, _I, _F, _P, _P]),
    "dsa_prefill_kl_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "dsa_forward_prefill_kl": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _SZ,
                                    _P]),
    "dsa_launch_count": (ctypes.c_uint64, []),
    "dsa_prefill_block_rows": (_I, [_I, _I, _I]),
    "dsa_prefill_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "dsa_prefill_select": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _SZ, _P]),
    "dsa_forward_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _SZ, _P]),
    "dsa_prefill_host_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "dsa_forward_prefill_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _SZ,
                                      _P]),
    "dsa_prefill_rows_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "dsa_forward_prefill_rows": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _SZ,
                                      _P]),
    "dsa_prefill_varlen_workspace_size": (_SZ, [_I, _I64, _I, _I, _I, _I, _I]),
    "dsa_forward_prefill_varlen": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P, _P, _P, _SZ,
                                        _P]),
    "dsa_decode_workspace_size": (_SZ, [_I, _I64, _I, _I, _I, _I]),
    "dsa_forward_decode": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I, _I, _I, _I, _F,
                                _P, _P, _P, _P, _SZ, _P]),
    "dsa_decode_paged_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "dsa_forward_decode_paged": (_I, [_I, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                      _F, _P, _P, _P, _P, _SZ, _P]),
    "dsa_decode_noalloc_scratch_bytes": (_SZ, []),
    "dsa_forward_decode_noalloc": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I, _I, _I, _I,
                                        _F, _P, _P, _P, _P]),
}


class DsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {_STATUS.get(code, code)}")
        self.code = code


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libdsa.so is not built ({path}); run `python -m sparse_attention_long_05_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = load()


def use_library(path: str = LIB_PATH) -> str:
    """Route every binding below to the library at `path` (e.g. CHECKS_LIB_PATH, the -DDSA_CHECKS build, which
    exports the same entry points); returns the path in use before."""
    global _lib
    prev = _lib._name
    _lib = load(path)
    return prev


def dsa_checks_enabled() -> bool:
    return bool(_lib.dsa_checks_enabled())


def dsa_checks_selftest(which: int, stream=None) -> int:
    """Plant violation `which` (0: a malformed top-k row, 1: a non-causal selected entry) in the checking build
    and return the device status it leaves."""
    scratch = torch.empty((int(_lib.dsa_checks_selftest_bytes()),), dtype=torch.uint8, device="cuda")
    _check("dsa_checks_selftest", _lib.dsa_checks_selftest(which, _ptr(scratch), _stream(stream)))
    return dsa_get_device_status(stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libdsa takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise DsaError(fn, code)


def dsa_num_sms() -> int:
    return _lib.dsa_num_sms()


def dsa_get_device_status(stream=None) -> int:
    v = ctypes.c_int(0)
    _check("dsa_get_device_status", _lib.dsa_get_device_status(_stream(stream), ctypes.byref(v)))
    return v.value


def dsa_check_bounded_wait(stream=None):
    """Run the bounded-wait self-check kernel (about a second) and return (result [4] int32 on the device,
    device status).  result = [warp 0 succeeded, its wait in 2^20 cycles, warp 1 succeeded, its wait]."""
    res = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    _check("dsa_check_bounded_wait", _lib.dsa_check_bounded_wait(_ptr(res), _stream(stream)))
    return res, dsa_get_device_status(stream)


def dsa_indexer_scores(q_idx, q_scale, k_idx, k_scale, w, pos0: int = 0, scores=None, stream=None):
    """Index scores [T, S] (fp32) of query rows at positions pos0.. against keys 0..S-1."""
    T, H_I, d_I = q_idx.shape
    S = k_idx.shape[0]
    if scores is None:
        scores = torch.empty((T, S), dtype=torch.float32, device=q_idx.device)
    _check("dsa_indexer_scores", _lib.dsa_indexer_scores(
        _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w), T, S, H_I, d_I, pos0, _ptr(scores),
        _stream(stream)))
    return scores


def dsa_topk(scores, k: int, row_len=None, pos0: int = 0, idx=None, stream=None):
    """Top-k columns [rows, k] (int32, ascending, -1 padded) of each row of scores [rows, ld]."""
    rows, ld = scores.shape
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    _check("dsa_topk", _lib.dsa_topk(_ptr(scores), rows, ld, _ptr(row_len), pos0, k, _ptr(idx), _stream(stream)))
    return idx


def dsa_sparse_mla_attn(q, c, idx, scale: float, out=None, lse=None, want_lse: bool = True, stream=None):
    """Attention of q [T, H, 576] over the selected rows idx [T, k] of c [S, 576] -> (out [T, H, 512], lse)."""
    T, H, _ = q.shape
    S = c.shape[0]
    k = idx.shape[1]
    if out is None:
        out = torch.empty((T, H, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    _check("dsa_sparse_mla_attn", _lib.dsa_sparse_mla_attn(
        _ptr(q), _ptr(c), S, _ptr(idx), T, H, k, float(scale), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def dsa_indexer_kl(q, c, idx, sel_scores, lse, scale: float, kl=None, stream=None):
    """KL(p_t || Softmax(I_t)) [T] of each token over its selected entries, from the attention's lse [T, H] and the
    selected entries' index scores sel_scores [T, k]."""
    T, H, _ = q.shape
    S = c.shape[0]
    k = idx.shape[1]
    if kl is None:
        kl = torch.empty((T,), dtype=torch.float32, device=q.device)
    _check("dsa_indexer_kl", _lib.dsa_indexer_kl(
        _ptr(q), _ptr(c), S, _ptr(idx), _ptr(sel_scores), _ptr(lse), T, H, k, float(scale), _ptr(kl),
        _stream(stream)))
    return kl


def dsa_prefill_kl_workspace_size(L: int, H_I: int, d_I: int, H: int, k: int) -> int:
    return int(_lib.dsa_prefill_kl_workspace_size(L, H_I, d_I, H, k))


def dsa_forward_prefill_kl(q_idx, q_scale, k_idx, k_scale, w, q, c, k: int, scale: float, idx_out=None, out=None,
                           lse=None, kl=None, ws=None, stream=None):
    """DSA forward of one causal prefill sequence plus the indexer objective per row -> (idx, out, lse, kl [L])."""
    L, H_I, d_I = q_idx.shape
    H = q.shape[1]
    dev = q.device
    if idx_out is None:
        idx_out = torch.empty((L, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((L, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((L, H), dtype=torch.float32, device=dev)
    if kl is None:
        kl = torch.empty((L,), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty((dsa_prefill_kl_workspace_size(L, H_I, d_I, H, k),), dtype=torch.uint8, device=dev)
    _check("dsa_forward_prefill_kl", _lib.dsa_forward_prefill_kl(
        _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w), _ptr(q), _ptr(c), L, H_I, d_I, H, k,
        float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(kl), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out, lse, kl


def dsa_prefill_workspace_size(L: int, H_I: int, d_I: int, H: int, k: int) -> int:
    return int(_lib.dsa_prefill_workspace_size(L, H_I, d_I, H, k))


def dsa_prefill_block_rows(L: int, k: int, r0: int) -> int:
    return int(_lib.dsa_prefill_block_rows(L, k, r0))


def prefill_blocks(L: int, k: int):
    """(first row, rows) of every score block of an L-row prefill, in the order the select processes them."""
    out, r0 = [], 0
    while r0 < L:
        n = dsa_prefill_block_rows(L, k, r0)
        out.append((r0, n))
        r0 += n
    return out


def dsa_launch_count() -> int:
    return int(_lib.dsa_launch_count())


def dsa_prefill_select(q_idx, q_scale, k_idx, k_scale, w, k: int, idx_out=None, ws=None, stream=None):
    """Indexer scores + top-k of every row of one causal prefill sequence -> idx [L, k] (int32)."""
    L, H_I, d_I = q_idx.shape
    dev = q_idx.device
    if idx_out is None:
        idx_out = torch.empty((L, k), dtype=torch.int32, device=dev)
    if ws is None:
        ws = torch.empty((dsa_prefill_workspace_size(L, H_I, d_I, 1, k),), dtype=torch.uint8, device=dev)
    _check("dsa_prefill_select", _lib.dsa_prefill_select(
        _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w), L, H_I, d_I, k, _ptr(idx_out), _ptr(ws),
        ws.numel(), _stream(stream)))
    return idx_out


def dsa_forward_prefill(q_idx, q_scale, k_idx, k_scale, w, q, c, k: int, scale: float, idx_out=None, out=None,
                        lse=None, ws=None, stream=None):
    """Whole DSA forward of one causal prefill sequence -> (idx [L, k], out [L, H, 512], lse [L, H])."""
    L, H_I, d_I = q_idx.shape
    H = q.shape[1]
    dev = q.device
    if idx_out is None:
        idx_out = torch.empty((L, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((L, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((L, H), dtype=torch.float32, device=dev)
    need = dsa_prefill_workspace_size(L, H_I, d_I, H, k)
    if ws is None:
        ws = torch.empty((need,), dtype=torch.uint8, device=dev)
    _check("dsa_forward_prefill", _lib.dsa_forward_prefill(
        _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w), _ptr(q), _ptr(c), L, H_I, d_I, H, k,
        float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out, lse


def _hptr(t):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("dsa_forward_prefill_host takes host tensors")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def dsa_prefill_host_workspace_size(L: int, H_I: int, d_I: int, H: int, k: int) -> int:
    return int(_lib.dsa_prefill_host_workspace_size(L, H_I, d_I, H, k))


def dsa_forward_prefill_host(q_idx, q_scale, k_idx, k_scale, w, q, c, k: int, scale: float, idx_out, out, lse, ws,
                             stream=None):
    """dsa_forward_prefill over HOST tensors (page-locked for overlapped copies): fills idx_out, out and lse (host
    tensors, the latter two may be None); ws is a device workspace of dsa_prefill_host_workspace_size bytes."""
    L, H_I, d_I = q_idx.shape
    H = q.shape[1]
    _check("dsa_forward_prefill_host", _lib.dsa_forward_prefill_host(
        _hptr(q_idx), _hptr(q_scale), _hptr(k_idx), _hptr(k_scale), _hptr(w), _hptr(q), _hptr(c), L, H_I, d_I, H, k,
        float(scale), _hptr(idx_out), _hptr(out), _hptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out, lse


def dsa_prefill_rows_workspace_size(row0: int, nrows: int, H_I: int, d_I: int, H: int, k: int) -> int:
    return int(_lib.dsa_prefill_rows_workspace_size(row0, nrows, H_I, d_I, H, k))


def dsa_forward_prefill_rows(row0: int, q_idx, q_scale, k_idx, k_scale, w, q, c, k: int, scale: float, idx_out=None,
                             out=None, lse=None, ws=None, stream=None):
    """Steps 1-3 for the rows row0 .. row0 + nrows - 1 of one causal sequence (query-side tensors of those rows,
    key-side tensors of the sequence from position 0) -> (idx [nrows, k], out [nrows, H, 512], lse [nrows, H])."""
    nrows, H_I, d_I = q_idx.shape
    H = q.shape[1]
    dev = q.device
    if idx_out is None:
        idx_out = torch.empty((nrows, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((nrows, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((nrows, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty((dsa_prefill_rows_workspace_size(row0, nrows, H_I, d_I, H, k),), dtype=torch.uint8,
                         device=dev)
    _check("dsa_forward_prefill_rows", _lib.dsa_forward_prefill_rows(
        _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale), _ptr(w), _ptr(q), _ptr(c), row0, nrows, H_I, d_I, H,
        k, float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out, lse


def dsa_prefill_varlen_workspace_size(nseq: int, total: int, max_len: int, H_I: int, d_I: int, H: int,
                                      k: int) -> int:
    return int(_lib.dsa_prefill_varlen_workspace_size(nseq, total, max_len, H_I, d_I, H, k))


def dsa_forward_prefill_varlen(cu_seqlens, q_idx, q_scale, k_idx, k_scale, w, q, c, k: int, scale: float,
                               idx_out=None, out=None, lse=None, ws=None, stream=None):
    """DSA forward of a packed batch of causal sequences (sequence b = rows cu_seqlens[b]..cu_seqlens[b+1]-1)
    -> (idx [total, k] within each sequence, out [total, H, 512], lse [total, H])."""
    cu = [int(v) for v in cu_seqlens]
    nseq = len(cu) - 1
    total, H_I, d_I = q_idx.shape
    H = q.shape[1]
    dev = q.device
    max_len = max((cu[b + 1] - cu[b] for b in range(nseq)), default=0)
    if idx_out is None:
        idx_out = torch.empty((total, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((total, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((total, H), dtype=torch.float32, device=dev)
    if ws is None:
        need = dsa_prefill_varlen_workspace_size(nseq, total, max(max_len, 1), H_I, d_I, H, k)
        ws = torch.empty((max(need, 1),), dtype=torch.uint8, device=dev)
    cu_arr = (ctypes.c_int64 * len(cu))(*cu)
    _check("dsa_forward_prefill_varlen", _lib.dsa_forward_prefill_varlen(
        nseq, ctypes.cast(cu_arr, ctypes.c_void_p), _ptr(q_idx), _ptr(q_scale), _ptr(k_idx), _ptr(k_scale),
        _ptr(w), _ptr(q), _ptr(c), H_I, d_I, H, k, float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(stream)))
    return idx_out, out, lse


def dsa_decode_workspace_size(B: int, cache_rows: int, H_I: int, d_I: int, H: int, k: int) -> int:
    return int(_lib.dsa_decode_workspace_size(B, cache_rows, H_I, d_I, H, k))


def dsa_forward_decode(cache_off, ctx_len, q_idx, q_scale, w, q, k_new, k_scale_new, c_new, k_cache,
                       k_scale_cache, c_cache, k: int, scale: float, idx_out=None, out=None, lse=None, ws=None,
                       stream=None):
    """One decode step for B sequences (appends the new entries, then attends) -> (idx, out, lse)."""
    B, H_I, d_I = q_idx.shape
    H = q.shape[1]
    rows = k_cache.shape[0]
    dev = q.device
    if idx_out is None:
        idx_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty((dsa_decode_workspace_size(B, rows, H_I, d_I, H, k),), dtype=torch.uint8, device=dev)
    _check("dsa_forward_decode", _lib.dsa_forward_decode(
        B, _ptr(cache_off), _ptr(ctx_len), _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(q), _ptr(k_new),
        _ptr(k_scale_new), _ptr(c_new), _ptr(k_cache), _ptr(k_scale_cache), _ptr(c_cache), rows, H_I, d_I, H, k,
        float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out, lse


def dsa_decode_paged_workspace_size(B: int, max_pages: int, page_rows: int, H_I: int, d_I: int, H: int,
                                    k: int) -> int:
    return int(_lib.dsa_decode_paged_workspace_size(B, max_pages, page_rows, H_I, d_I, H, k))


def dsa_forward_decode_paged(page_table, page_rows: int, ctx_len, q_idx, q_scale, w, q, k_new, k_scale_new, c_new,
                             k_cache, k_scale_cache, c_cache, k: int, scale: float, idx_out=None, out=None, lse=None,
                             ws=None, stream=None):
    """One decode step over paged caches (page_table [B, max_pages] int32; pools of page_rows-row pages)
    -> (idx, out, lse)."""
    B, H_I, d_I = q_idx.shape
    H = q.shape[1]
    max_pages = page_table.shape[1]
    num_pages = k_cache.shape[0] // page_rows
    dev = q.device
    if idx_out is None:
        idx_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty((dsa_decode_paged_workspace_size(B, max_pages, page_rows, H_I, d_I, H, k),),
                         dtype=torch.uint8, device=dev)
    _check("dsa_forward_decode_paged", _lib.dsa_forward_decode_paged(
        B, _ptr(page_table), max_pages, page_rows, _ptr(ctx_len), _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(q),
        _ptr(k_new), _ptr(k_scale_new), _ptr(c_new), _ptr(k_cache), _ptr(k_scale_cache), _ptr(c_cache), num_pages,
        H_I, d_I, H, k, float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, out, lse


def dsa_decode_noalloc_scratch_bytes() -> int:
    return int(_lib.dsa_decode_noalloc_scratch_bytes())


def dsa_forward_decode_noalloc(cache_off, ctx_len, q_idx, q_scale, w, q, k_new, k_scale_new, c_new, k_cache,
                               k_scale_cache, c_cache, k: int, scale: float, idx_out=None, out=None, lse=None,
                               stream=None):
    """dsa_forward_decode with the library's fixed scratch array instead of a workspace (allocates nothing
    on the device beyond the outputs this wrapper creates when none are passed)."""
    B, H_I, d_I = q_idx.shape
    H = q.shape[1]
    rows = k_cache.shape[0]
    dev = q.device
    if idx_out is None:
        idx_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    _check("dsa_forward_decode_noalloc", _lib.dsa_forward_decode_noalloc(
        B, _ptr(cache_off), _ptr(ctx_len), _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(q), _ptr(k_new),
        _ptr(k_scale_new), _ptr(c_new), _ptr(k_cache), _ptr(k_scale_cache), _ptr(c_cache), rows, H_I, d_I, H, k,
        float(scale), _ptr(idx_out), _ptr(out), _ptr(lse), _stream(stream)))
    return idx_out, out, lse
