"""Thin Python binding of the DSA C ABI (``include/dsa.h``).

Argument marshalling only: every function passes torch CUDA tensors' device
pointers and the current CUDA stream to the entry point of the same name in
``libdsa_b200.so``; every step of the computation runs in that library's
kernels.  There is no fallback: if the library is missing, or a call returns
an error status, a ``DSAError`` is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa_b200.so")

DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2
STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
          4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT"}

# Every symbol include/dsa.h declares.
EXPORTS = ("dsa_status_string", "dsa_version", "dsa_index_scores", "dsa_topk_workspace_size",
           "dsa_topk", "dsa_topk_window", "dsa_sparse_attn", "dsa_prefill_workspace_size",
           "dsa_prefill", "dsa_prefill_window", "dsa_prefill_host_workspace_size", "dsa_prefill_host",
           "dsa_decode_workspace_size", "dsa_decode", "dsa_decode_window", "dsa_decode_kv8",
           "dsa_quantize_e4m3", "dsa_cache_append", "dsa_cache_append_kv8", "dsa_decode_noalloc",
           "dsa_split_workspace_size", "dsa_decode_select", "dsa_merge_selections", "dsa_decode_attend",
           "dsa_merge_partials", "dsa_stream_status", "dsa_profile_enable", "dsa_profile_read",
           "dsa_prefill_rows_workspace_size", "dsa_prefill_rows", "dsa_test_stall_next")


class DSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"DSA CUDA library not found at {path}; build it with "
            "`python -m long_context_fp8_b200.build`")
    lib = ctypes.CDLL(path)
    P, I64, I32, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "dsa_status_string": ([I32], ctypes.c_char_p),
        "dsa_version": ([], I32),
        "dsa_index_scores": ([P, P, P, P, P, I64, I32, I32, I64, I64, P, I64, I32, I32, P], I32),
        "dsa_topk_workspace_size": ([I64, I64, I32], SZ),
        "dsa_topk": ([P, I64, I64, I64, I64, I32, P, P, SZ, P], I32),
        "dsa_sparse_attn": ([P, P, P, P, I64, I32, I32, I32, F, P, P, I32, P], I32),
        "dsa_prefill_workspace_size": ([I64, I32, I32, I32, I32, I32, I32], SZ),
        "dsa_prefill": ([P, P, P, P, P, P, P, P, I64, I32, I32, I32, I32, I32, F, P, P, P, I32, P,
                         SZ, P], I32),
        "dsa_prefill_host_workspace_size": ([I64, I32, I32, I32, I32, I32, I32], SZ),
        "dsa_prefill_host": ([P, P, P, P, P, P, P, P, I64, I32, I32, I32, I32, I32, F, P, P, P, I32, P,
                              SZ, P], I32),
        "dsa_decode_workspace_size": ([I32, I64, I32, I32, I32], SZ),
        "dsa_decode": ([P, P, P, P, P, P, P, P, P, P, I64, I32, I32, I32, I64, I32, I32, I32, I32,
                        I32, F, P, P, P, P, SZ, P], I32),
        "dsa_decode_noalloc": ([P, P, P, P, P, P, P, P, P, P, I64, I32, I32, I32, I64, I32, I32, I32,
                                I32, I32, F, P, P, P, P, P], I32),
        "dsa_topk_window": ([P, I64, I64, I64, I64, I32, I32, P, P, SZ, P], I32),
        "dsa_prefill_window": ([P, P, P, P, P, P, P, P, I64, I32, I32, I32, I32, I32, I32, F, P, P, P,
                                I32, P, SZ, P], I32),
        "dsa_decode_window": ([P, P, P, P, P, P, P, P, P, P, I64, I32, I32, I32, I64, I32, I32, I32, I32,
                               I32, I32, F, P, P, P, P, SZ, P], I32),
        "dsa_quantize_e4m3": ([P, I32, I64, I64, P, P, P], I32),
        "dsa_decode_kv8": ([P, P, P, P, P, P, P, P, P, P, P, P, I64, I32, I32, I32, I64, I32, I32, I32, I32,
                            I32, I32, F, P, P, P, P, SZ, P], I32),
        "dsa_cache_append_kv8": ([P, I32, P, P, P, P, I64, I32, P, I32, I64, I32, I32, I32, P, P, P, P, P, P,
                                  P, P], I32),
        "dsa_cache_append": ([P, I32, P, P, P, P, I64, I32, P, I32, I64, I32, I32, I32, P, P, P, P, P, P],
                             I32),
        "dsa_split_workspace_size": ([I32, I32, I64, I32, I32, I32], SZ),
        "dsa_decode_select": ([P, P, P, P, P, P, P, P, I64, I32, I32, I32, I64, I32, I32, I32, P, P, P, SZ, P],
                              I32),
        "dsa_merge_selections": ([P, P, I64, I32, I32, I32, P, P, SZ, P], I32),
        "dsa_decode_attend": ([P, P, P, P, P, P, P, P, I64, I32, I32, I32, I32, I32, I32, P, F, P, P, P, SZ, P],
                              I32),
        "dsa_merge_partials": ([P, I64, P, I64, I32, I32, I32, I32, P, P, P], I32),
        "dsa_stream_status": ([P, P], I32),
        "dsa_profile_enable": ([I32], I32),
        "dsa_test_stall_next": ([I32], I32),
        "dsa_prefill_rows_workspace_size": ([I64, I64, I32, I32, I32, I32, I32, I32], SZ),
        "dsa_prefill_rows": ([P, P, P, P, P, P, P, P, I64, I64, I64, I32, I32, I32, I32, I32, F, P, P, P, I32, P,
                              SZ, P], I32),
        "dsa_profile_read": ([P, P], I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path == LIB_PATH:
        _lib = lib
    return lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("DSA entry points take CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("DSA entry points take contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, st: int):
    if st != 0:
        raise DSAError(fn, st)


def _idx_dtype(q_idx: torch.Tensor) -> int:
    if q_idx.dtype == torch.uint8:
        return DSA_E4M3
    if q_idx.dtype == torch.float32:
        return DSA_F32
    raise ValueError(f"unsupported index dtype {q_idx.dtype}")


def _val_dtype(q: torch.Tensor) -> int:
    return {torch.bfloat16: DSA_BF16, torch.float32: DSA_F32}[q.dtype]


def workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned workspace (256-byte aligned by the torch allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def dsa_version() -> int:
    return load().dsa_version()


def dsa_status_string(s: int) -> str:
    return load().dsa_status_string(s).decode()


def dsa_index_scores(q_idx, q_scale, k_idx, k_scale, w, row_begin=0, row_count=None, out=None,
                     ld=None, fill_upper=True, stream=None):
    """Indexer scores of query rows [row_begin, row_begin+row_count) -> f32 [rows, ld]
    (-inf above the diagonal when fill_upper, else those entries untouched)."""
    T, H, D = q_idx.shape
    row_count = T - row_begin if row_count is None else row_count
    ld = T if ld is None else ld
    if out is None:
        out = torch.empty((max(row_count, 0), ld), dtype=torch.float32, device=q_idx.device)
    st = load().dsa_index_scores(_p(q_idx), _p(q_scale), _p(k_idx), _p(k_scale), _p(w), T, H, D,
                                 row_begin, row_count, _p(out), ld, int(bool(fill_upper)),
                                 _idx_dtype(q_idx), _stream(stream))
    _check("dsa_index_scores", st)
    return out


def dsa_topk(scores, k, row_begin=0, T=None, out=None, stream=None):
    """Top-k of score rows (row r = query position row_begin + r) -> int32 [rows, k]."""
    rows, ld = scores.shape
    T = ld if T is None else T
    if out is None:
        out = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    lib = load()
    wsb = lib.dsa_topk_workspace_size(rows, T, k)
    ws = workspace(wsb, scores.device) if wsb else None
    st = lib.dsa_topk(_p(scores), ld, row_begin, rows, T, k, _p(out), _p(ws), wsb, _stream(stream))
    _check("dsa_topk", st)
    return out


def dsa_topk_window(scores, k, window, row_begin=0, T=None, out=None, stream=None):
    """Sliding window plus top-k of score rows -> int32 [rows, k + window]."""
    rows, ld = scores.shape
    T = ld if T is None else T
    if out is None:
        out = torch.empty((rows, k + window), dtype=torch.int32, device=scores.device)
    st = load().dsa_topk_window(_p(scores), ld, row_begin, rows, T, k, window, _p(out), None, 0,
                                _stream(stream))
    _check("dsa_topk_window", st)
    return out


def dsa_quantize_e4m3(x, codes=None, scale=None, stream=None):
    """Per-row FP8 E4M3 quantisation of bf16/fp32 ``x[rows, ...]`` ->
    (uint8 codes of x's shape, fp32 scale[rows])."""
    rows = x.shape[0]
    cols = x.numel() // max(rows, 1) if rows else (x[0].numel() if x.dim() > 1 else 1)
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((rows,), dtype=torch.float32, device=x.device)
    st = load().dsa_quantize_e4m3(_p(x), _val_dtype(x), rows, cols, _p(codes), _p(scale), _stream(stream))
    _check("dsa_quantize_e4m3", st)
    return codes, scale


def dsa_cache_append(caches: dict, kidx_new, k_new, v_new, seq_ids, positions, block_table,
                     status=None, stream=None):
    """Quantise and write N new tokens' index keys and copy their K/V rows into
    the paged caches (``caches``: kidx_cache, kscale_cache, k_cache, v_cache,
    updated in place).  ``status``: optional int32 [1] device tensor that
    receives DSA_ERR_INVALID_ARG for an out-of-range token."""
    N, d_I = kidx_new.shape
    d = k_new.shape[1]
    P, ps, _ = caches["kidx_cache"].shape
    B, max_pages = block_table.shape
    st = load().dsa_cache_append(_p(kidx_new), _val_dtype(kidx_new), _p(k_new), _p(v_new), _p(seq_ids),
                                 _p(positions), N, B, _p(block_table), max_pages, P, ps, d_I, d,
                                 _p(caches["kidx_cache"]), _p(caches["kscale_cache"]), _p(caches["k_cache"]),
                                 _p(caches["v_cache"]), _p(status), _stream(stream))
    _check("dsa_cache_append", st)


def dsa_sparse_attn(q, k, v, idx, sm_scale=None, out=None, lse=None, stream=None):
    """Attention of each query row over its selected K/V rows -> (out, lse)."""
    T, H, D = q.shape
    ksel = idx.shape[1]
    sm_scale = 1.0 / math.sqrt(D) if sm_scale is None else sm_scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    st = load().dsa_sparse_attn(_p(q), _p(k), _p(v), _p(idx), T, H, D, ksel, sm_scale, _p(out),
                                _p(lse), _val_dtype(q), _stream(stream))
    _check("dsa_sparse_attn", st)
    return out, lse


def prefill_workspace_size(T, H_I, d_I, H_q, d, k_sel, dtype=DSA_E4M3) -> int:
    return load().dsa_prefill_workspace_size(T, H_I, d_I, H_q, d, k_sel, dtype)


def dsa_prefill(inp: dict, k_sel: int, sm_scale=None, out=None, lse=None, idx_out=None, ws=None,
                want_idx=True, stream=None):
    """Fused prefill (indexer -> top-k -> sparse attention) of one sequence."""
    q_idx, q = inp["q_idx"], inp["q"]
    T, H_I, d_I = q_idx.shape
    _, H_q, d = q.shape
    dt = _idx_dtype(q_idx)
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_prefill_workspace_size(T, H_I, d_I, H_q, d, k_sel, dt), q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, H_q), dtype=torch.float32, device=q.device)
    if idx_out is None and want_idx:
        idx_out = torch.empty((T, k_sel), dtype=torch.int32, device=q.device)
    st = lib.dsa_prefill(_p(q_idx), _p(inp["q_scale"]), _p(inp["k_idx"]), _p(inp["k_scale"]),
                         _p(inp["w"]), _p(q), _p(inp["k"]), _p(inp["v"]), T, H_I, d_I, H_q, d,
                         k_sel, sm_scale, _p(out), _p(lse), _p(idx_out), dt, _p(ws), ws.numel(),
                         _stream(stream))
    _check("dsa_prefill", st)
    return out, lse, idx_out


def dsa_prefill_window(inp: dict, k_sel: int, window: int, sm_scale=None, out=None, lse=None,
                       idx_out=None, ws=None, want_idx=True, stream=None):
    """dsa_prefill with a sliding window: the last `window` positions of every
    query are always attended, top-k over the older ones; idx [T, k_sel + window]."""
    q_idx, q = inp["q_idx"], inp["q"]
    T, H_I, d_I = q_idx.shape
    _, H_q, d = q.shape
    dt = _idx_dtype(q_idx)
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_prefill_workspace_size(T, H_I, d_I, H_q, d, k_sel + window, dt), q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, H_q), dtype=torch.float32, device=q.device)
    if idx_out is None and want_idx:
        idx_out = torch.empty((T, k_sel + window), dtype=torch.int32, device=q.device)
    st = lib.dsa_prefill_window(_p(q_idx), _p(inp["q_scale"]), _p(inp["k_idx"]), _p(inp["k_scale"]),
                                _p(inp["w"]), _p(q), _p(inp["k"]), _p(inp["v"]), T, H_I, d_I, H_q, d,
                                k_sel, window, sm_scale, _p(out), _p(lse), _p(idx_out), dt, _p(ws),
                                ws.numel(), _stream(stream))
    _check("dsa_prefill_window", st)
    return out, lse, idx_out


def prefill_rows_workspace_size(T, row_count, H_I, d_I, H_q, d, k_sel) -> int:
    return load().dsa_prefill_rows_workspace_size(T, row_count, H_I, d_I, H_q, d, k_sel, DSA_E4M3)


def dsa_prefill_rows(rows: dict, keys: dict, row_begin: int, k_sel: int, sm_scale=None, out=None, lse=None,
                     idx_out=None, ws=None, stream=None):
    """The fused prefill of query rows [row_begin, row_begin + n) of a sequence:
    ``rows`` holds those rows' q_idx [n, H_I, d_I], q_scale [n], w [n, H_I] and
    q [n, H_q, d]; ``keys`` the k_idx [T, d_I], k_scale [T], k and v [T, d] of
    every position.  Returns (out, lse, idx) of the n rows."""
    q_idx, q = rows["q_idx"], rows["q"]
    n, H_I, d_I = q_idx.shape
    _, H_q, d = q.shape
    T = keys["k_idx"].shape[0]
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    if ws is None:
        ws = workspace(max(1, lib.dsa_prefill_rows_workspace_size(T, n, H_I, d_I, H_q, d, k_sel, DSA_E4M3)),
                       q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((n, H_q), dtype=torch.float32, device=q.device)
    if idx_out is None:
        idx_out = torch.empty((n, k_sel), dtype=torch.int32, device=q.device)
    st = lib.dsa_prefill_rows(_p(q_idx), _p(rows["q_scale"]), _p(keys["k_idx"]), _p(keys["k_scale"]),
                              _p(rows["w"]), _p(q), _p(keys["k"]), _p(keys["v"]), T, row_begin, n, H_I, d_I,
                              H_q, d, k_sel, sm_scale, _p(out), _p(lse), _p(idx_out), DSA_E4M3, _p(ws),
                              ws.numel(), _stream(stream))
    _check("dsa_prefill_rows", st)
    return out, lse, idx_out


def _h(t: Optional[torch.Tensor]):
    """Host tensor pointer (contiguous, CPU; page-locked for overlapped copies)."""
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("dsa_prefill_host takes host (CPU) tensors")
    if not t.is_contiguous():
        raise ValueError("DSA entry points take contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def prefill_host_workspace_size(T, H_I, d_I, H_q, d, k_sel) -> int:
    return load().dsa_prefill_host_workspace_size(T, H_I, d_I, H_q, d, k_sel, DSA_E4M3)


def dsa_prefill_host(inp: dict, k_sel: int, out, sm_scale=None, lse=None, idx_out=None, ws=None,
                     stream=None):
    """dsa_prefill with host (CPU) inputs and outputs: the library moves the query
    rows in and the outputs back pass by pass, overlapped with the computation.
    Asynchronous on `stream`; `out` (and lse / idx_out) hold the results once the
    stream has reached this point."""
    q_idx, q = inp["q_idx"], inp["q"]
    T, H_I, d_I = q_idx.shape
    _, H_q, d = q.shape
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_prefill_host_workspace_size(T, H_I, d_I, H_q, d, k_sel, _idx_dtype(q_idx)),
                       torch.device("cuda"))
    st = lib.dsa_prefill_host(_h(q_idx), _h(inp["q_scale"]), _h(inp["k_idx"]), _h(inp["k_scale"]),
                              _h(inp["w"]), _h(q), _h(inp["k"]), _h(inp["v"]), T, H_I, d_I, H_q, d, k_sel,
                              sm_scale, _h(out), _h(lse), _h(idx_out), _idx_dtype(q_idx), _p(ws), ws.numel(),
                              _stream(stream))
    _check("dsa_prefill_host", st)
    return out, lse, idx_out


def decode_workspace_size(B, max_context, H_q, d, k_sel) -> int:
    return load().dsa_decode_workspace_size(B, max_context, H_q, d, k_sel)


def dsa_decode(inp: dict, k_sel: int, max_context: int, sm_scale=None, out=None, lse=None,
               idx_out=None, ws=None, want_idx=True, stream=None):
    """One decode step of B sequences over paged caches -> (out, lse, idx)."""
    B, H_I, d_I = inp["q_idx"].shape
    _, H_q, d = inp["q"].shape
    P, ps, _ = inp["kidx_cache"].shape
    max_pages = inp["block_table"].shape[1]
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_decode_workspace_size(B, max_context, H_q, d, k_sel), inp["q"].device)
    if out is None:
        out = torch.empty_like(inp["q"])
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=inp["q"].device)
    if idx_out is None and want_idx:
        idx_out = torch.empty((B, k_sel), dtype=torch.int32, device=inp["q"].device)
    st = lib.dsa_decode(_p(inp["q_idx"]), _p(inp["q_scale"]), _p(inp["w"]), _p(inp["q"]),
                        _p(inp["kidx_cache"]), _p(inp["kscale_cache"]), _p(inp["k_cache"]),
                        _p(inp["v_cache"]), _p(inp["block_table"]), _p(inp["context_lens"]),
                        P, max_pages, ps, B, max_context, H_I, d_I, H_q, d, k_sel, sm_scale,
                        _p(out), _p(lse), _p(idx_out), _p(ws), ws.numel(), _stream(stream))
    _check("dsa_decode", st)
    return out, lse, idx_out


def dsa_decode_window(inp: dict, k_sel: int, window: int, max_context: int, sm_scale=None, out=None,
                      lse=None, idx_out=None, ws=None, want_idx=True, stream=None):
    """dsa_decode with a sliding window (the last `window` cached positions of
    each sequence always attended) -> (out, lse, idx [B, k_sel + window])."""
    B, H_I, d_I = inp["q_idx"].shape
    _, H_q, d = inp["q"].shape
    P, ps, _ = inp["kidx_cache"].shape
    max_pages = inp["block_table"].shape[1]
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    kw = k_sel + window
    if ws is None:
        ws = workspace(lib.dsa_decode_workspace_size(B, max_context, H_q, d, kw), inp["q"].device)
    if out is None:
        out = torch.empty_like(inp["q"])
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=inp["q"].device)
    if idx_out is None and want_idx:
        idx_out = torch.empty((B, kw), dtype=torch.int32, device=inp["q"].device)
    st = lib.dsa_decode_window(_p(inp["q_idx"]), _p(inp["q_scale"]), _p(inp["w"]), _p(inp["q"]),
                               _p(inp["kidx_cache"]), _p(inp["kscale_cache"]), _p(inp["k_cache"]),
                               _p(inp["v_cache"]), _p(inp["block_table"]), _p(inp["context_lens"]),
                               P, max_pages, ps, B, max_context, H_I, d_I, H_q, d, k_sel, window,
                               sm_scale, _p(out), _p(lse), _p(idx_out), _p(ws), ws.numel(),
                               _stream(stream))
    _check("dsa_decode_window", st)
    return out, lse, idx_out


def dsa_decode_kv8(inp: dict, k_sel: int, max_context: int, window: int = 0, sm_scale=None, out=None,
                   lse=None, idx_out=None, ws=None, want_idx=True, stream=None):
    """Decode over FP8 K/V caches (``inp`` holds uint8 k_cache/v_cache and f32
    k_cache_scale/v_cache_scale) -> (out, lse, idx [B, k_sel + window])."""
    B, H_I, d_I = inp["q_idx"].shape
    _, H_q, d = inp["q"].shape
    P, ps, _ = inp["kidx_cache"].shape
    max_pages = inp["block_table"].shape[1]
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    kw = k_sel + window
    if ws is None:
        ws = workspace(lib.dsa_decode_workspace_size(B, max_context, H_q, d, kw), inp["q"].device)
    if out is None:
        out = torch.empty_like(inp["q"])
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=inp["q"].device)
    if idx_out is None and want_idx:
        idx_out = torch.empty((B, kw), dtype=torch.int32, device=inp["q"].device)
    st = lib.dsa_decode_kv8(_p(inp["q_idx"]), _p(inp["q_scale"]), _p(inp["w"]), _p(inp["q"]),
                            _p(inp["kidx_cache"]), _p(inp["kscale_cache"]), _p(inp["k_cache"]),
                            _p(inp["k_cache_scale"]), _p(inp["v_cache"]), _p(inp["v_cache_scale"]),
                            _p(inp["block_table"]), _p(inp["context_lens"]), P, max_pages, ps, B, max_context,
                            H_I, d_I, H_q, d, k_sel, window, sm_scale, _p(out), _p(lse), _p(idx_out), _p(ws),
                            ws.numel(), _stream(stream))
    _check("dsa_decode_kv8", st)
    return out, lse, idx_out


def dsa_cache_append_kv8(caches: dict, kidx_new, k_new, v_new, seq_ids, positions, block_table,
                         status=None, stream=None):
    """dsa_cache_append for FP8 K/V caches (``caches`` also holds
    k_cache_scale/v_cache_scale): index key, K and V rows all quantised."""
    N, d_I = kidx_new.shape
    d = k_new.shape[1]
    P, ps, _ = caches["kidx_cache"].shape
    B, max_pages = block_table.shape
    st = load().dsa_cache_append_kv8(_p(kidx_new), _val_dtype(kidx_new), _p(k_new), _p(v_new), _p(seq_ids),
                                     _p(positions), N, B, _p(block_table), max_pages, P, ps, d_I, d,
                                     _p(caches["kidx_cache"]), _p(caches["kscale_cache"]), _p(caches["k_cache"]),
                                     _p(caches["k_cache_scale"]), _p(caches["v_cache"]),
                                     _p(caches["v_cache_scale"]), _p(status), _stream(stream))
    _check("dsa_cache_append_kv8", st)


NOALLOC_SCRATCH_BYTES = 64 << 20


def dsa_decode_noalloc(inp: dict, k_sel: int, max_context: int, sm_scale=None, out=None, lse=None,
                       idx_out=None, status_out=None, stream=None):
    """dsa_decode with the library's fixed internal scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    B, H_I, d_I = inp["q_idx"].shape
    _, H_q, d = inp["q"].shape
    P, ps, _ = inp["kidx_cache"].shape
    max_pages = inp["block_table"].shape[1]
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    if out is None:
        out = torch.empty_like(inp["q"])
    st = load().dsa_decode_noalloc(_p(inp["q_idx"]), _p(inp["q_scale"]), _p(inp["w"]), _p(inp["q"]),
                                   _p(inp["kidx_cache"]), _p(inp["kscale_cache"]), _p(inp["k_cache"]),
                                   _p(inp["v_cache"]), _p(inp["block_table"]), _p(inp["context_lens"]),
                                   P, max_pages, ps, B, max_context, H_I, d_I, H_q, d, k_sel, sm_scale,
                                   _p(out), _p(lse), _p(idx_out), _p(status_out), _stream(stream))
    _check("dsa_decode_noalloc", st)
    return out, lse, idx_out


def _p_lists(t: torch.Tensor):
    """Pointer and dim-0 stride (elements) of G lists whose inner dims are
    dense (a [G, ...] view that may be a slice of a larger message)."""
    if not t.is_cuda:
        raise ValueError("DSA entry points take CUDA tensors")
    if not t[0].is_contiguous():
        raise ValueError("each list must be dense")
    return ctypes.c_void_p(t.data_ptr()), int(t.stride(0))


def split_workspace_size(G, B, max_context, H_q, d, k_sel) -> int:
    return load().dsa_split_workspace_size(G, B, max_context, H_q, d, k_sel)


def dsa_decode_select(shard: dict, pos_base, k_sel: int, max_context: int, cand_pos=None, cand_score=None,
                      ws=None, stream=None):
    """This shard's indexer scores and top-k as global positions (+ pos_base)
    with their scores -> (cand_pos [B, k_sel], cand_score [B, k_sel])."""
    B, H_I, d_I = shard["q_idx"].shape
    P, ps, _ = shard["kidx_cache"].shape
    max_pages = shard["block_table"].shape[1]
    dev = shard["q_idx"].device
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_split_workspace_size(1, B, max_context, 128, 128, k_sel), dev)
    if cand_pos is None:
        cand_pos = torch.empty((B, k_sel), dtype=torch.int32, device=dev)
    if cand_score is None:
        cand_score = torch.empty((B, k_sel), dtype=torch.float32, device=dev)
    st = lib.dsa_decode_select(_p(shard["q_idx"]), _p(shard["q_scale"]), _p(shard["w"]), _p(shard["kidx_cache"]),
                               _p(shard["kscale_cache"]), _p(shard["block_table"]), _p(shard["context_lens"]),
                               _p(pos_base), P, max_pages, ps, B, max_context, H_I, d_I, k_sel, _p(cand_pos),
                               _p(cand_score), _p(ws), ws.numel(), _stream(stream))
    _check("dsa_decode_select", st)
    return cand_pos, cand_score


def dsa_merge_selections(cand_pos, cand_score, idx_out=None, ws=None, stream=None):
    """Exact top-k of the union of G candidate lists (cand_pos/cand_score
    [G, B, k_sel] views with a common dim-0 stride) -> idx [B, k_sel]."""
    G, B, k_sel = cand_pos.shape
    pp, sp = _p_lists(cand_pos)
    ps_, ss = _p_lists(cand_score)
    if sp != ss or cand_score.shape != cand_pos.shape:
        raise ValueError("positions and scores must share shape and list stride")
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_split_workspace_size(G, B, 1, 128, 128, k_sel), cand_pos.device)
    if idx_out is None:
        idx_out = torch.empty((B, k_sel), dtype=torch.int32, device=cand_pos.device)
    st = lib.dsa_merge_selections(pp, ps_, sp, G, B, k_sel, _p(idx_out), _p(ws), ws.numel(), _stream(stream))
    _check("dsa_merge_selections", st)
    return idx_out


def dsa_decode_attend(shard: dict, pos_base, idx, sm_scale=None, out=None, lse=None, ws=None, stream=None):
    """Attention of each sequence's query over the selected positions this
    shard holds -> partial (out [B, H_q, d], lse [B, H_q]).  FP8 K/V when
    ``shard`` holds k_cache_scale/v_cache_scale."""
    B, H_q, d = shard["q"].shape
    P, ps, _ = shard["k_cache"].shape
    max_pages = shard["block_table"].shape[1]
    k_sel = idx.shape[1]
    dev = shard["q"].device
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    lib = load()
    if ws is None:
        ws = workspace(lib.dsa_split_workspace_size(1, B, 1, H_q, d, k_sel), dev)
    if out is None:
        out = torch.empty_like(shard["q"])
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=dev)
    st = lib.dsa_decode_attend(_p(shard["q"]), _p(shard["k_cache"]), _p(shard.get("k_cache_scale")),
                               _p(shard["v_cache"]), _p(shard.get("v_cache_scale")), _p(shard["block_table"]),
                               _p(shard["context_lens"]), _p(pos_base), P, max_pages, ps, B, H_q, d, k_sel, _p(idx),
                               sm_scale, _p(out), _p(lse), _p(ws), ws.numel(), _stream(stream))
    _check("dsa_decode_attend", st)
    return out, lse


def dsa_merge_partials(part_out, part_lse, out=None, lse=None, stream=None):
    """Log-sum-exp merge of G partial attentions (part_out [G, B, H_q, d]
    bf16, part_lse [G, B, H_q] f32; views with dense inner dims) -> (out, lse)."""
    G, B, H_q, d = part_out.shape
    po, so = _p_lists(part_out)
    pl, sl = _p_lists(part_lse)
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.bfloat16, device=part_out.device)
    if lse is None:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=part_out.device)
    st = load().dsa_merge_partials(po, so, pl, sl, G, B, H_q, d, _p(out), _p(lse), _stream(stream))
    _check("dsa_merge_partials", st)
    return out, lse


def dsa_stream_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return (and clear) the workspace's device status."""
    return load().dsa_stream_status(_p(ws), _stream(stream))


# Stage names of dsa_profile_read, in dsa_stage order.
STAGES = ("sample", "tau", "select", "finish", "repair", "scores", "topk", "attention")


def profile_enable(on: bool = True):
    """Turn the library's per-stage CUDA-event timing on or off (process-wide)."""
    _check("dsa_profile_enable", load().dsa_profile_enable(1 if on else 0))


def profile_read():
    """Device milliseconds and run counts per stage recorded since the last
    read (waits for the recorded events): {stage: (ms, runs)}."""
    ms = (ctypes.c_double * len(STAGES))()
    n = (ctypes.c_int64 * len(STAGES))()
    _check("dsa_profile_read", load().dsa_profile_read(ctypes.cast(ms, ctypes.c_void_p),
                                                       ctypes.cast(n, ctypes.c_void_p)))
    return {name: (ms[i], n[i]) for i, name in enumerate(STAGES)}


STALL_NONE, STALL_PREFILL_INDEXER, STALL_DECODE_INDEXER = 0, 1, 2


def test_stall_next(target: int):
    """Arm the library's one-shot test hook: the next launch of the named
    indexer leaves one copy unissued, so that its bounded wait runs out."""
    _check("dsa_test_stall_next", load().dsa_test_stall_next(int(target)))
