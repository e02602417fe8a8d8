"""Python face of the fp64 CPU oracle (``dsa_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product library.  It
marshals numpy/torch CPU arrays into the C oracle and back; all arithmetic
lives in the C file.  Each function cites the passage it follows in
``dsa_oracle.c``'s header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")

OR_F32, OR_BF16, OR_E4M3 = 0, 1, 2

_lib = None


def build(out: str = _LIB, extra_flags=()) -> str:
    """Compile the oracle with gcc (plain -O2, OpenMP, no fast-math)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", *extra_flags,
           _SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is None:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        path = _LIB
    lib = ctypes.CDLL(path)
    P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.dsa_or_e4m3.argtypes = [ctypes.c_uint8]
    lib.dsa_or_e4m3.restype = D
    lib.dsa_or_bf16.argtypes = [ctypes.c_uint16]
    lib.dsa_or_bf16.restype = D
    lib.dsa_or_index_scores.argtypes = [P, P, P, P, P, I32, I32, I64, I32, I32, P, I64, P]
    lib.dsa_or_index_scores.restype = I32
    lib.dsa_or_topk.argtypes = [P, I64, P, I64, I32, P]
    lib.dsa_or_topk.restype = I32
    lib.dsa_or_sparse_attn.argtypes = [P, P, P, I32, P, I64, I32, I32, I32, D, P, P]
    lib.dsa_or_sparse_attn.restype = I32
    lib.dsa_or_decode.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, I32, I32, I32, I32, I32,
                                  I32, I32, I32, I32, D, P, I64, P, P, P]
    lib.dsa_or_decode.restype = I32
    lib.dsa_or_topk_window.argtypes = [P, I64, P, I64, I32, I32, P]
    lib.dsa_or_topk_window.restype = I32
    lib.dsa_or_e4m3_encode.argtypes = [ctypes.c_float]
    lib.dsa_or_e4m3_encode.restype = ctypes.c_uint8
    lib.dsa_or_quantize_e4m3.argtypes = [P, I32, I64, I64, P, P]
    lib.dsa_or_quantize_e4m3.restype = I32
    lib.dsa_or_cache_append.argtypes = [P, I32, P, P, P, P, I64, I32, P, I32, I64, I32, I32, I32,
                                        P, P, P, P, P, P]
    lib.dsa_or_cache_append.restype = I32
    if path == _LIB:
        _lib = lib
    return lib


def _np(x, dtype=None):
    """CPU contiguous numpy view of a torch tensor / numpy array (bf16 -> uint16 bits)."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16)
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    if dtype is not None:
        a = np.ascontiguousarray(a.astype(dtype, copy=False))
    return a


def _is_torch(x) -> bool:
    try:
        import torch
        return isinstance(x, torch.Tensor)
    except ImportError:  # pragma: no cover
        return False


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _idx_dtype(q_idx) -> int:
    a = _np(q_idx)
    return OR_E4M3 if a.dtype == np.uint8 else OR_F32


def _val_dtype(x) -> int:
    try:
        import torch
        if isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16:
            return OR_BF16
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(x)
    return OR_BF16 if a.dtype in (np.uint16, np.int16) else OR_F32


def e4m3(code: int) -> float:
    return load().dsa_or_e4m3(code)


def bf16(bits: int) -> float:
    return load().dsa_or_bf16(bits)


def index_scores(q_idx, q_scale, k_idx, k_scale, w, rows, lib=None, compact=False) -> np.ndarray:
    """Indexer scores I[rows[r], s] for all s (-inf for s > rows[r]); fp64 [nrows, T].

    Follows stage 1 of the oracle header (lightning indexer, DSA section 1).
    q_idx/q_scale/w hold every query row, or (compact=True) only the listed rows.
    """
    lib = lib or load()
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if not compact:
        # keep only the listed query rows (the oracle reads query data per listed row)
        sel = torch.from_numpy(rows) if _is_torch(q_idx) else rows
        q_idx, w = q_idx[sel], w[sel]
        q_scale = q_scale[sel] if q_scale is not None else None
    qa, ka, wa = _np(q_idx), _np(k_idx), _np(w)
    T, D = ka.shape
    H = qa.shape[1]
    dt = OR_E4M3 if qa.dtype == np.uint8 else OR_F32
    if dt == OR_F32:
        qa, ka = qa.astype(np.float32), ka.astype(np.float32)
    wdt = _val_dtype(w)
    qs = _np(q_scale, np.float32) if q_scale is not None else None
    ks = _np(k_scale, np.float32) if k_scale is not None else None
    out = np.empty((rows.size, T), dtype=np.float64)
    rc = lib.dsa_or_index_scores(_ptr(qa), _ptr(qs), _ptr(ka), _ptr(ks), _ptr(wa), dt, wdt,
                                 T, H, D, _ptr(rows), rows.size, _ptr(out))
    assert rc == 0, "oracle allocation failure"
    return out


def topk(scores, rows, k, lib=None) -> np.ndarray:
    """Top-k selection of each row (stage 2 of the oracle header); int32 [nrows, k].

    ``scores`` is [nrows, ld] of any float dtype (widened exactly to fp64);
    row r's candidates are entries 0..rows[r].
    """
    lib = lib or load()
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((rows.size, k), dtype=np.int32)
    rc = lib.dsa_or_topk(_ptr(s), s.shape[1], _ptr(rows), rows.size, k, _ptr(out))
    assert rc == 0
    return out


def topk_window(scores, rows, k, window, lib=None) -> np.ndarray:
    """Sliding window plus top-k of each row (stage 5 of the oracle header);
    int32 [nrows, k + window]: the top-k of positions 0..rows[r]-window
    ascending, then the window positions, then -1."""
    lib = lib or load()
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((rows.size, k + window), dtype=np.int32)
    rc = lib.dsa_or_topk_window(_ptr(s), s.shape[1], _ptr(rows), rows.size, k, window, _ptr(out))
    assert rc == 0
    return out


def e4m3_encode(y: float) -> int:
    """E4M3 code nearest to the fp32 value y (stage 6: ties to even, saturating)."""
    return int(load().dsa_or_e4m3_encode(float(y)))


def quantize_e4m3(x, lib=None):
    """Per-row FP8 quantisation (stage 6) of fp32 or bf16 ``x[rows, ...]``:
    (uint8 codes of x's shape, fp32 scale[rows])."""
    lib = lib or load()
    dt = _val_dtype(x)
    a = _np(x)
    if dt == OR_F32:
        a = np.ascontiguousarray(a.astype(np.float32))
    rows = a.shape[0]
    cols = int(np.prod(a.shape[1:])) if a.ndim > 1 else 1
    codes = np.empty(a.shape, dtype=np.uint8)
    scale = np.empty(rows, dtype=np.float32)
    rc = lib.dsa_or_quantize_e4m3(_ptr(a), dt, rows, cols, _ptr(codes), _ptr(scale))
    assert rc == 0
    return codes, scale


def cache_append(caches: dict, kidx_new, k_new, v_new, seq, pos, block_table, lib=None) -> int:
    """Append tokens to copies of the paged caches (stage 6).  ``caches`` holds
    numpy arrays kidx_cache/kscale_cache/k_cache/v_cache (bf16 as uint16
    bits), updated in place.  Returns the oracle's status (0, or -2 for an
    out-of-range sequence, position or page)."""
    lib = lib or load()
    dt = _val_dtype(kidx_new)
    kn = _np(kidx_new)
    if dt == OR_F32:
        kn = np.ascontiguousarray(kn.astype(np.float32))
    kk, vv = _np(k_new), _np(v_new)
    sq, ps_ = _np(seq, np.int32), _np(pos, np.int32)
    bt = _np(block_table, np.int32)
    kic, ksc, kc, vc = (caches[n] for n in ("kidx_cache", "kscale_cache", "k_cache", "v_cache"))
    kcs, vcs = caches.get("k_cache_scale"), caches.get("v_cache_scale")   # FP8 K/V (stage 7)
    for a in (kic, ksc, kc, vc) + ((kcs, vcs) if kcs is not None else ()):
        assert a.flags.c_contiguous
    P, ps, D_I = kic.shape
    D = kc.shape[2]
    return lib.dsa_or_cache_append(_ptr(kn), dt, _ptr(kk), _ptr(vv), _ptr(sq), _ptr(ps_), sq.size,
                                   bt.shape[0], _ptr(bt), bt.shape[1], P, ps, D_I, D, _ptr(kic),
                                   _ptr(ksc), _ptr(kc), _ptr(vc), _ptr(kcs), _ptr(vcs))


def sparse_attn(q, K, V, idx, rows, sm_scale, lib=None, compact=False):
    """Attention of query rows over their selected K/V rows (stage 3); (out, lse) fp64.

    idx row r holds the selection of query position rows[r]; q holds every
    query row, or (compact=True) only the listed rows.
    """
    lib = lib or load()
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    if not compact:
        q = q[torch.from_numpy(rows)] if _is_torch(q) else q[rows]
    dt = _val_dtype(q)
    qa, ka, va = _np(q), _np(K), _np(V)
    if dt == OR_F32:
        qa, ka, va = qa.astype(np.float32), ka.astype(np.float32), va.astype(np.float32)
    n, H, D = qa.shape
    ia = _np(idx, np.int32)
    k = ia.shape[1]
    assert ia.shape[0] == n == rows.size
    out = np.empty((n, H, D), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    rc = lib.dsa_or_sparse_attn(_ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(ia), n, k, H, D,
                                float(sm_scale), _ptr(out), _ptr(lse))
    assert rc == 0
    return out, lse


def decode(inp: dict, k: int, sm_scale: float, want_scores: bool = False, lib=None, window: int = 0):
    """One decode step over paged caches (stage 4; with window > 0, stage 5's
    selection; with FP8 K/V caches -- uint8 k_cache/v_cache plus
    k_cache_scale/v_cache_scale -- stage 7's attention); returns dict
    idx [B, k+window]/out/lse[/scores]."""
    lib = lib or load()
    q_idx, q_scale, w, q = _np(inp["q_idx"]), _np(inp["q_scale"], np.float32), _np(inp["w"]), _np(inp["q"])
    kidx, ksc = _np(inp["kidx_cache"]), _np(inp["kscale_cache"], np.float32)
    kc, vc = _np(inp["k_cache"]), _np(inp["v_cache"])
    kv8 = kc.dtype == np.uint8
    kcs = _np(inp["k_cache_scale"], np.float32) if kv8 else None
    vcs = _np(inp["v_cache_scale"], np.float32) if kv8 else None
    bt, ctx = _np(inp["block_table"], np.int32), _np(inp["context_lens"], np.int32)
    B, H_I, D_I = q_idx.shape
    H_q, D = q.shape[1], q.shape[2]
    ps = kidx.shape[1]
    ld = int(ctx.max()) if want_scores else 0
    scores = np.full((B, ld), np.nan) if want_scores else None
    idx = np.empty((B, k + window), dtype=np.int32)
    out = np.empty((B, H_q, D), dtype=np.float64)
    lse = np.empty((B, H_q), dtype=np.float64)
    rc = lib.dsa_or_decode(_ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(q), _ptr(kidx), _ptr(ksc),
                           _ptr(kc), _ptr(vc), _ptr(kcs), _ptr(vcs), _ptr(bt), _ptr(ctx), B, bt.shape[1], ps, H_I,
                           D_I, H_q, D, k, window, float(sm_scale), _ptr(scores), ld, _ptr(idx),
                           _ptr(out), _ptr(lse))
    assert rc == 0
    res = dict(idx=idx, out=out, lse=lse)
    if want_scores:
        res["scores"] = scores
    return res


def prefill(inp: dict, k: int, sm_scale: float, rows, lib=None, window: int = 0):
    """Stages 1-3 (with window > 0, stage 5's selection) for the listed query
    rows: dict scores/idx/out/lse."""
    rows = np.asarray(rows, dtype=np.int64)
    sc = index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"], rows, lib)
    idx = topk_window(sc, rows, k, window, lib) if window > 0 else topk(sc, rows, k, lib)
    out, lse = sparse_attn(inp["q"], inp["k"], inp["v"], idx, rows, sm_scale, lib)
    return dict(scores=sc, idx=idx, out=out, lse=lse)
