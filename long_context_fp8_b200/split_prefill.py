"""Prefill of one long sequence split over the ranks of a process group.

Query row t of a causal prefill scores t + 1 keys, so its cost grows with t.
The rows are therefore dealt in a zigzag: the T rows are cut into 2G
near-equal chunks in position order, and rank g takes chunks g and
2G - 1 - g, which pairs a cheap chunk with an expensive one.  Each rank holds
the per-token inputs of its own rows: the query side (q_idx, q_scale, w, q)
and the key side (k_idx, k_scale, k, v).  A prefill then takes one exchange:
an all-gather of the key side, since every row needs the index keys, keys and
values of all earlier positions.  After it each rank runs the unchanged
single-device prefill on its two chunks (``dsa_prefill_rows``); the outputs
stay sharded.  None of the pages describes a multi-device prefill; the
hotdry page's million-token setting motivates it.

The arithmetic runs in the library's kernels (``CudaOps``); this module only
lays out the message, issues the collective and copies the gathered chunks
into place.  Every rank makes the same collective call.  No copy here uses
TMA multicast: the gathered key side is in this rank's own memory before any
kernel reads it.
"""
from __future__ import annotations

import math
from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import dsa

KEY_FIELDS = ("k_idx", "k_scale", "k", "v")
QUERY_FIELDS = ("q_idx", "q_scale", "w", "q")


def chunk_bounds(T: int, G: int) -> List[Tuple[int, int]]:
    """The 2G chunks [floor(j T / 2G), floor((j + 1) T / 2G)) in position order."""
    n = 2 * G
    return [(j * T // n, (j + 1) * T // n) for j in range(n)]


def rank_chunks(g: int, G: int) -> Tuple[int, int]:
    """Chunk indices of rank g: g and 2G - 1 - g."""
    return g, 2 * G - 1 - g


def rank_rows(T: int, G: int, g: int) -> List[Tuple[int, int]]:
    """Row ranges [begin, end) of rank g, in chunk order (g, then 2G - 1 - g)."""
    b = chunk_bounds(T, G)
    return [b[j] for j in rank_chunks(g, G)]


def _align16(n: int) -> int:
    return (n + 15) // 16 * 16


def key_layout(c_max: int, d_I: int, d: int):
    """Byte offsets of one chunk's key side inside a message slot of c_max rows:
    k_idx u8 [c_max, d_I], k_scale f32 [c_max], k and v bf16 [c_max, d], each
    part starting 16-byte aligned.  Returns ({field: offset}, slot bytes)."""
    sizes = {"k_idx": c_max * d_I, "k_scale": 4 * c_max, "k": 2 * c_max * d, "v": 2 * c_max * d}
    off, pos = {}, 0
    for f in KEY_FIELDS:
        off[f] = pos
        pos += _align16(sizes[f])
    return off, pos


_DT = {"k_idx": torch.uint8, "k_scale": torch.float32, "k": torch.bfloat16, "v": torch.bfloat16}


def _field_view(slot: torch.Tensor, off: dict, field: str, rows: int, width: int):
    """View of `rows` rows of a field inside a uint8 message slot."""
    esz = torch.empty((), dtype=_DT[field]).element_size()
    n = rows * width
    v = slot[off[field]:off[field] + n * esz].view(_DT[field])
    return v.view(rows, width) if width > 1 else v


def all_gather(recv: torch.Tensor, send: torch.Tensor, group=None):
    """recv[g] = rank g's send (recv [G, *send.shape], contiguous)."""
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(recv, send, group=group)
    else:
        dist.all_gather(list(recv.unbind(0)), send, group=group)


def gather_keys(chunks: List[dict], T: int, group=None) -> dict:
    """The key side of all T positions on every rank, from each rank's two
    chunks (``chunks[i]`` holds the key fields of this rank's i-th chunk in
    rank_rows order): one all-gather of a [2, slot] byte message per rank."""
    G = dist.get_world_size(group)
    d_I = chunks[0]["k_idx"].shape[1]
    d = chunks[0]["k"].shape[1]
    dev = chunks[0]["k_idx"].device
    c_max = max(e - b for b, e in chunk_bounds(T, G))
    off, slot = key_layout(c_max, d_I, d)
    send = torch.zeros((2, slot), dtype=torch.uint8, device=dev)
    width = {"k_idx": d_I, "k_scale": 1, "k": d, "v": d}
    for i, ch in enumerate(chunks):
        rows = ch["k_idx"].shape[0]
        for f in KEY_FIELDS:
            _field_view(send[i], off, f, rows, width[f]).copy_(ch[f].reshape(rows, width[f]) if width[f] > 1
                                                                else ch[f].reshape(rows))
    recv = torch.empty((G,) + tuple(send.shape), dtype=torch.uint8, device=dev)
    all_gather(recv, send, group)
    keys = {"k_idx": torch.empty((T, d_I), dtype=torch.uint8, device=dev),
            "k_scale": torch.empty((T,), dtype=torch.float32, device=dev),
            "k": torch.empty((T, d), dtype=torch.bfloat16, device=dev),
            "v": torch.empty((T, d), dtype=torch.bfloat16, device=dev)}
    for g in range(G):
        for i, (b, e) in enumerate(rank_rows(T, G, g)):
            for f in KEY_FIELDS:
                keys[f][b:e].copy_(_field_view(recv[g, i], off, f, e - b, width[f]))
    return keys


class CudaOps:
    """The per-rank prefill of a row range on this rank's GPU, through the C
    ABI, with one workspace reused across calls."""

    def __init__(self):
        self._ws: Optional[torch.Tensor] = None

    def prefill_rows(self, rows: dict, keys: dict, row_begin: int, k_sel: int, sm_scale: float):
        n, H_I, d_I = rows["q_idx"].shape
        _, H_q, d = rows["q"].shape
        T = keys["k_idx"].shape[0]
        need = dsa.prefill_rows_workspace_size(T, n, H_I, d_I, H_q, d, k_sel)
        if self._ws is None or self._ws.numel() < need or self._ws.device != rows["q"].device:
            self._ws = dsa.workspace(need, rows["q"].device)
        return dsa.dsa_prefill_rows(rows, keys, row_begin, k_sel, sm_scale, ws=self._ws)


_default_ops: Optional[CudaOps] = None


def split_prefill(chunks: List[dict], T: int, k_sel: int, group=None, sm_scale: Optional[float] = None,
                  ops=None):
    """The prefill of this rank's two zigzag chunks of a T-token sequence.
    ``chunks[i]`` holds the query and key fields of the rows rank_rows(T, G,
    rank)[i].  Returns [(out, lse, idx)] per chunk, each equal to those rows
    of a single-device prefill of the whole sequence."""
    global _default_ops
    if ops is None:
        if _default_ops is None:
            _default_ops = CudaOps()
        ops = _default_ops
    G, g = dist.get_world_size(group), dist.get_rank(group)
    d = chunks[0]["q"].shape[2]
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    keys = gather_keys(chunks, T, group)
    return [ops.prefill_rows({f: ch[f] for f in QUERY_FIELDS}, keys, b, k_sel, sm_scale)
            for ch, (b, _) in zip(chunks, rank_rows(T, G, g))]
