"""Decode of one context split over the ranks of a process group.

Each sequence's cached positions are cut into G contiguous shards, one per
rank in rank order; rank g holds shard g in its own paged caches (local
positions 0..n_g-1, global position = pos_base[b] + local).  A decode step
then takes two small all-gathers and reproduces the single-device decode:

1. every rank scores its keys and selects its own top-k, as global positions
   with their indexer scores (``dsa_decode_select``);
2. all-gather of the candidates, one message of [positions | scores];
3. every rank takes the exact top-k of the union (``dsa_merge_selections``):
   each member of the global top-k is in its shard's top-k, and with the
   shards in position order the lower column of a tie is the lower position,
   so the result equals the whole-context selection;
4. every rank attends the selected positions it holds (``dsa_decode_attend``),
   a partial output with its log-sum-exp;
5. all-gather of the partials, one message of [out | lse], and the
   log-sum-exp merge (``dsa_merge_partials``).

The step's arithmetic runs in the library's kernels (``CudaOps``); this module
only lays out the two messages and issues the collectives.  Every rank makes
the same collective calls in the same order.
"""
from __future__ import annotations

import math
from typing import Optional

import torch
import torch.distributed as dist

from . import dsa


def shard_bounds(context_lens, G: int):
    """Contiguous near-equal shards: shard g of a context of n positions is
    [floor(g n / G), floor((g + 1) n / G)).  Returns (base [G, B], lens [G, B])
    as int64 tensors; every shard is non-empty when n >= G."""
    n = torch.as_tensor(context_lens, dtype=torch.int64)
    g = torch.arange(G + 1, dtype=torch.int64)[:, None]
    edges = (g * n[None, :]) // G
    return edges[:-1], edges[1:] - edges[:-1]


def candidate_message(B: int, k_sel: int, G: int, device):
    """Send buffer [2, B, k_sel] int32 (positions, score bits) and receive
    buffer [G, 2, B, k_sel], with the typed views each step uses."""
    send = torch.empty((2, B, k_sel), dtype=torch.int32, device=device)
    recv = torch.empty((G, 2, B, k_sel), dtype=torch.int32, device=device)
    return send, recv


def candidate_views(buf: torch.Tensor):
    """(positions int32, scores f32) views of a [..., 2, B, k] message."""
    return buf.select(-3, 0), buf.select(-3, 1).view(torch.float32)


def partial_words(B: int, H_q: int, d: int) -> int:
    """int32 words of one partial message: bf16 out [B, H_q, d] then f32 lse
    [B, H_q], padded to 16 bytes."""
    w = B * H_q * d // 2 + B * H_q
    return (w + 3) // 4 * 4


def partial_message(B: int, H_q: int, d: int, G: int, device):
    W = partial_words(B, H_q, d)
    return (torch.empty((W,), dtype=torch.int32, device=device),
            torch.empty((G, W), dtype=torch.int32, device=device))


def partial_views(buf: torch.Tensor, B: int, H_q: int, d: int):
    """(out bf16 [..., B, H_q, d], lse f32 [..., B, H_q]) views of partial
    messages ([W] or [G, W] int32)."""
    lead = buf.shape[:-1]
    n_out = B * H_q * d // 2
    out = buf[..., :n_out].view(torch.bfloat16).view(*lead, B, H_q, d)
    lse = buf[..., n_out:n_out + B * H_q].view(torch.float32).view(*lead, B, H_q)
    return out, lse


def all_gather(recv: torch.Tensor, send: torch.Tensor, group=None):
    """recv[g] = rank g's send (recv [G, *send.shape], contiguous)."""
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(recv, send, group=group)
    else:
        dist.all_gather(list(recv.unbind(0)), send, group=group)


class CudaOps:
    """The four per-rank steps on this rank's GPU, through the C ABI, with
    one workspace reused across calls."""

    def __init__(self):
        self._ws: Optional[torch.Tensor] = None

    def workspace(self, G, B, max_context, H_q, d, k_sel, device):
        need = dsa.split_workspace_size(G, B, max_context, H_q, d, k_sel)
        if self._ws is None or self._ws.numel() < need or self._ws.device != device:
            self._ws = dsa.workspace(need, device)
        return self._ws

    def select(self, shard, pos_base, k_sel, max_context, cand_pos, cand_score, ws):
        dsa.dsa_decode_select(shard, pos_base, k_sel, max_context, cand_pos=cand_pos, cand_score=cand_score, ws=ws)

    def merge_selections(self, cand_pos, cand_score, idx_out, ws):
        dsa.dsa_merge_selections(cand_pos, cand_score, idx_out=idx_out, ws=ws)

    def attend(self, shard, pos_base, idx, sm_scale, out, lse, ws):
        dsa.dsa_decode_attend(shard, pos_base, idx, sm_scale, out=out, lse=lse, ws=ws)

    def merge_partials(self, part_out, part_lse, out, lse):
        dsa.dsa_merge_partials(part_out, part_lse, out=out, lse=lse)


_default_ops: Optional[CudaOps] = None


def split_decode_step(shard: dict, pos_base: torch.Tensor, k_sel: int, max_context: int, group=None,
                      sm_scale: Optional[float] = None, ops=None):
    """One decode step of B sequences whose contexts are split over the ranks
    of ``group``.  ``shard`` holds this rank's inputs as for ``dsa_decode``
    (queries replicated, caches and context_lens of this shard only);
    pos_base int32 [B] is the global position of this shard's first cached
    position of each sequence; max_context is the largest shard length on
    any rank.  Returns (out [B, H_q, d] bf16, lse [B, H_q], idx [B, k_sel]),
    identical on every rank."""
    global _default_ops
    if ops is None:
        if _default_ops is None:
            _default_ops = CudaOps()              # one workspace, grown on demand, reused by every step
        ops = _default_ops
    G = dist.get_world_size(group)
    B, H_q, d = shard["q"].shape
    dev = shard["q"].device
    sm_scale = 1.0 / math.sqrt(d) if sm_scale is None else sm_scale
    ws = ops.workspace(G, B, max_context, H_q, d, k_sel, dev) if hasattr(ops, "workspace") else None

    send, recv = candidate_message(B, k_sel, G, dev)
    pos, score = candidate_views(send)
    ops.select(shard, pos_base, k_sel, max_context, pos, score, ws)
    all_gather(recv, send, group)
    idx = torch.empty((B, k_sel), dtype=torch.int32, device=dev)
    ops.merge_selections(*candidate_views(recv), idx, ws)

    psend, precv = partial_message(B, H_q, d, G, dev)
    ops.attend(shard, pos_base, idx, sm_scale, *partial_views(psend, B, H_q, d), ws)
    all_gather(precv, psend, group)
    out = torch.empty((B, H_q, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H_q), dtype=torch.float32, device=dev)
    ops.merge_partials(*partial_views(precv, B, H_q, d), out, lse)
    return out, lse, idx
