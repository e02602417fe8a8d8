"""Brute-force dense-mask DSA in numpy ("Mask MHA" emulation).

TEST INFRASTRUCTURE ONLY.  A second, independent restatement of the method
used to cross-check the C oracle on tiny inputs: it builds the whole dense
score matrix, the whole selection mask and a dense masked softmax, the way the
pages say short sequences emulate DSA with a masked MHA ("DeepSeek-V3.2-Exp
DSA 技术深度解析", section 1).  FP8 and bf16 storage is decoded through the
library conversions of torch (not through the C oracle's decoders).
"""
from __future__ import annotations

import numpy as np
import torch


def decode_storage(x) -> np.ndarray:
    """fp64 values of a stored tensor: uint8 = E4M3 bytes, bf16, fp32."""
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(x)
    x = x.detach().cpu()
    if x.dtype == torch.uint8:
        x = x.view(torch.float8_e4m3fn)
    return x.to(torch.float64).numpy()


def dense_scores(q_idx, q_scale, k_idx, k_scale, w) -> np.ndarray:
    """[T, T] matrix I with -inf above the diagonal."""
    q = decode_storage(q_idx)                       # [T,H,D]
    kk = decode_storage(k_idx)                      # [T,D]
    if q_scale is not None:
        q = q * decode_storage(q_scale)[:, None, None]
        kk = kk * decode_storage(k_scale)[:, None]
    ww = decode_storage(w)                          # [T,H]
    dots = np.einsum("thd,sd->ths", q, kk)          # [T,H,T]
    scores = np.einsum("th,ths->ts", ww, np.maximum(dots, 0.0))
    T = scores.shape[0]
    scores[np.triu_indices(T, 1)] = -np.inf
    return scores


def dense_topk_mask(scores: np.ndarray, k: int) -> np.ndarray:
    """Boolean [T, T] selection mask: per row t, the min(k, t+1) best s <= t,
    ties to the lower s (a stable sort on -score)."""
    T = scores.shape[0]
    mask = np.zeros((T, T), dtype=bool)
    for t in range(T):
        order = np.argsort(-scores[t, : t + 1], kind="stable")
        mask[t, order[: min(k, t + 1)]] = True
    return mask


def mask_to_idx(mask: np.ndarray, k: int) -> np.ndarray:
    T = mask.shape[0]
    out = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        sel = np.nonzero(mask[t])[0]
        out[t, : sel.size] = sel
    return out


def dense_masked_attention(q, K, V, mask: np.ndarray, sm_scale: float):
    """Dense MHA with a selection mask: softmax over the selected keys only.
    Returns (out [T,H,D], lse [T,H])."""
    qq, kk, vv = decode_storage(q), decode_storage(K), decode_storage(V)
    logits = sm_scale * np.einsum("thd,sd->hts", qq, kk)          # [H,T,T]
    logits = np.where(mask[None], logits, -np.inf)
    m = logits.max(axis=2, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=2, keepdims=True)
    out = np.einsum("hts,sd->thd", p / l, vv)
    lse = (m + np.log(l))[..., 0].T
    return out, lse
