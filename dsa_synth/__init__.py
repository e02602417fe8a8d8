"""Seeded synthetic inputs for DeepSeek Sparse Attention (DSA) workloads.

This module is the one piece shared by the CPU oracle's tests and the CUDA
path.  It only draws random numbers and packs them into the storage formats
the library consumes (FP8 E4M3 bytes with a per-token fp32 scale, bf16, fp32,
paged caches).  It contains none of the method's arithmetic: no indexer
score, no selection, no attention.

Workload shapes follow the pages' workloads:
  * the lightning indexer uses few heads, low-dimensional FP8 query/key
    (index_head_dim 128) -- "DeepSeek-V3.2-Exp DSA 技术深度解析", section 1;
  * k = 2048 in the training configuration (~1.6 % of a 128K context),
    same section; 256-512 suggested for deployment -- "DeepSeek V4 ... 稀疏
    注意力" (hotdry), section on the fine-grained selector;
  * needle-in-a-haystack style recall is stood in for by planted "needle"
    keys that are noisy copies of a chosen query, so that the selection is
    non-trivial (the pages' needle tests at several depths).

All draws come from one ``torch.Generator`` seeded per workload, in a fixed
order, so a (spec, device) pair always yields the same bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class PrefillSpec:
    """One causal prefill of a single sequence of L tokens."""
    name: str
    L: int
    H_I: int          # indexer heads
    d_I: int          # indexer head dim
    k: int            # top-k budget
    H_q: int          # main-attention query heads (one shared KV head)
    d: int            # main-attention head dim
    fp8: bool         # True: e4m3 index Q/K + fp32 scales, bf16 w/Q/K/V; False: all fp32
    n_needles: int
    seed: int
    idx_std: float = 1.0   # std of the source index Q/K values


@dataclass(frozen=True)
class DecodeSpec:
    """One decode step of B sequences against paged caches."""
    name: str
    context_lens: Tuple[int, ...]   # includes the current (already appended) token
    H_I: int
    d_I: int
    k: int
    H_q: int
    d: int
    page_size: int
    needle_frac: float
    needle_min_age: int   # needles sit at positions p <= n - 1 - needle_min_age
    seed: int

    @property
    def B(self) -> int:
        return len(self.context_lens)


PRESETS: Dict[str, object] = {
    # L=1024 fp32 workload with 16 needles, seed 0
    "tiny": PrefillSpec("tiny", L=1024, H_I=4, d_I=64, k=64, H_q=4, d=64,
                        fp8=False, n_needles=16, seed=0, idx_std=1.0 / 8.0),
    # 16K prefill: 1 % needles
    "p16k": PrefillSpec("p16k", L=16384, H_I=64, d_I=128, k=2048, H_q=16, d=128,
                        fp8=True, n_needles=164, seed=1),
    # 16K prefill with the 128K workload's 128 query heads: a small case of the
    # tensor-core attention path for profiling (inputs a few GB, still above L2)
    "p16k_hq128": PrefillSpec("p16k_hq128", L=16384, H_I=64, d_I=128, k=2048, H_q=128, d=128,
                              fp8=True, n_needles=164, seed=1),
    # 128K prefill: 0.5 % needles
    "p128k": PrefillSpec("p128k", L=131072, H_I=64, d_I=128, k=2048, H_q=128, d=128,
                         fp8=True, n_needles=655, seed=2),
    # decode: 64 sequences x 64K cached tokens
    "dec64x64k": DecodeSpec("dec64x64k", context_lens=(65536,) * 64, H_I=64, d_I=128,
                            k=2048, H_q=128, d=128, page_size=64, needle_frac=0.005,
                            needle_min_age=0, seed=3),
    # ragged long-context decode, needles beyond the most recent 16K positions
    "dec_ragged": DecodeSpec("dec_ragged", context_lens=(1048576, 786432, 524288, 262144),
                             H_I=64, d_I=128, k=512, H_q=128, d=128, page_size=64,
                             needle_frac=0.001, needle_min_age=16384, seed=4),
}


def prefill_spec(name: str, **overrides) -> PrefillSpec:
    spec = PRESETS[name]
    assert isinstance(spec, PrefillSpec)
    return replace(spec, **overrides) if overrides else spec


def decode_spec(name: str, **overrides) -> DecodeSpec:
    spec = PRESETS[name]
    assert isinstance(spec, DecodeSpec)
    return replace(spec, **overrides) if overrides else spec


# --------------------------------------------------------------------------
# storage packing (format conversion only)
# --------------------------------------------------------------------------

def quantize_e4m3_per_token(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Pack fp32 ``x[n, ...]`` as E4M3 bytes with one fp32 scale per leading row.

    scale = amax / 448 (1 for an all-zero row); bytes = round-to-nearest-even
    of x / scale, clamped to the finite E4M3 range.  Returns (uint8 bytes of
    x's shape, fp32 scale[n]).  Consumers decode the stored bytes, so the
    rounding here never enters a parity comparison.
    """
    n = x.shape[0]
    flat = x.reshape(n, -1).float()
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    q8 = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return q8.contiguous(), scale.float().contiguous()


def _randn(shape, g, device, std=1.0, dtype=torch.float32):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype) if dtype != torch.float32 else t


def _rand(shape, g, device):
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32)


# --------------------------------------------------------------------------
# prefill
# --------------------------------------------------------------------------

def make_prefill(spec: PrefillSpec, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of one causal prefill.

    Keys: q_idx [L,H_I,d_I], q_scale [L] (None for fp32), k_idx [L,d_I],
    k_scale [L] (None for fp32), w [L,H_I], q [L,H_q,d], k [L,d], v [L,d],
    needle_pos [n], needle_src [n] (the query position each needle copies).
    fp8 specs: q_idx/k_idx uint8 (E4M3 bytes), w/q/k/v bfloat16.
    fp32 specs: everything float32.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed)
    L, H_I, d_I, H_q, d = spec.L, spec.H_I, spec.d_I, spec.H_q, spec.d

    q_src = _randn((L, H_I, d_I), g, device, spec.idx_std)
    k_src = _randn((L, d_I), g, device, spec.idx_std)
    if spec.fp8:
        w = (_rand((L, H_I), g, device) / math.sqrt(H_I)).to(torch.bfloat16)
    else:
        w = _rand((L, H_I), g, device)
    vdt = torch.bfloat16 if spec.fp8 else torch.float32
    q = _randn((L, H_q, d), g, device, dtype=vdt)
    k = _randn((L, d), g, device, dtype=vdt)
    v = _randn((L, d), g, device, dtype=vdt)

    # needles: key position p is a noisy copy of a later query t (p < t < L)
    n = min(spec.n_needles, max(L - 1, 0))
    if n > 0:
        pos = torch.randperm(L - 1, generator=g, device=device)[:n].sort().values
        u = _rand((n,), g, device)
        src = pos + 1 + (u * (L - 1 - pos).float()).long().clamp_max(L - 1 - pos - 1)
        hs = (_rand((n,), g, device) * H_I).long().clamp_max(H_I - 1)
        hq = (_rand((n,), g, device) * H_q).long().clamp_max(H_q - 1)
        eps_i = _randn((n, d_I), g, device, spec.idx_std)
        eps_q = _randn((n, d), g, device)
        k_src[pos] = q_src[src, hs] + 0.1 * eps_i
        k[pos] = (q[src, hq].float() + 0.1 * eps_q).to(vdt)
    else:
        pos = torch.zeros(0, dtype=torch.long, device=device)
        src = pos.clone()

    if spec.fp8:
        q_idx, q_scale = quantize_e4m3_per_token(q_src)
        k_idx, k_scale = quantize_e4m3_per_token(k_src)
    else:
        q_idx, q_scale, k_idx, k_scale = q_src.contiguous(), None, k_src.contiguous(), None
    del q_src, k_src
    return dict(q_idx=q_idx, q_scale=q_scale, k_idx=k_idx, k_scale=k_scale,
                w=w.contiguous(), q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                needle_pos=pos, needle_src=src)


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

def make_decode(spec: DecodeSpec, device="cpu") -> Dict[str, torch.Tensor]:
    """Inputs of one decode step over paged caches.

    Keys: q_idx uint8 [B,H_I,d_I], q_scale f32 [B], w bf16 [B,H_I],
    q bf16 [B,H_q,d], kidx_cache uint8 [P,ps,d_I], kscale_cache f32 [P,ps],
    k_cache/v_cache bf16 [P,ps,d], block_table int32 [B,max_pages] (-1 past
    the end), context_lens int32 [B], needle_pos list of int64 tensors.
    Logical page i of sequence b lives in physical page block_table[b,i]; the
    physical pages are a seeded permutation so that paging is exercised.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed)
    B, H_I, d_I, H_q, d, ps = spec.B, spec.H_I, spec.d_I, spec.H_q, spec.d, spec.page_size
    lens = list(spec.context_lens)
    pages = [(n + ps - 1) // ps for n in lens]
    P = sum(pages)
    max_pages = max(pages)

    perm = torch.randperm(P, generator=g, device=device)
    block_table = torch.full((B, max_pages), -1, dtype=torch.int32, device=device)
    off = 0
    for b in range(B):
        block_table[b, :pages[b]] = perm[off:off + pages[b]].int()
        off += pages[b]

    q_src = _randn((B, H_I, d_I), g, device)
    w = (_rand((B, H_I), g, device) / math.sqrt(H_I)).to(torch.bfloat16)
    q = _randn((B, H_q, d), g, device, dtype=torch.bfloat16)

    kidx_cache = torch.zeros((P, ps, d_I), dtype=torch.uint8, device=device)
    kscale_cache = torch.ones((P, ps), dtype=torch.float32, device=device)
    k_cache = torch.zeros((P, ps, d), dtype=torch.bfloat16, device=device)
    v_cache = torch.zeros((P, ps, d), dtype=torch.bfloat16, device=device)
    needle_pos = []
    for b in range(B):
        n = lens[b]
        k_src = _randn((n, d_I), g, device)
        kb = _randn((n, d), g, device, dtype=torch.bfloat16)
        vb = _randn((n, d), g, device, dtype=torch.bfloat16)
        span = max(n - 1 - spec.needle_min_age, 0)   # candidates p in [0, span)
        nn = min(int(round(spec.needle_frac * n)), span)
        if nn > 0:
            pos = torch.randperm(span, generator=g, device=device)[:nn].sort().values
            hs = (_rand((nn,), g, device) * H_I).long().clamp_max(H_I - 1)
            hq = (_rand((nn,), g, device) * H_q).long().clamp_max(H_q - 1)
            eps_i = _randn((nn, d_I), g, device)
            eps_q = _randn((nn, d), g, device)
            k_src[pos] = q_src[b][hs] + 0.1 * eps_i
            kb[pos] = (q[b][hq].float() + 0.1 * eps_q).to(torch.bfloat16)
        else:
            pos = torch.zeros(0, dtype=torch.long, device=device)
        needle_pos.append(pos)
        k8, ks = quantize_e4m3_per_token(k_src)
        del k_src
        npg = pages[b]
        phys = block_table[b, :npg].long()
        padded = npg * ps
        def scatter(dst, src, fill=0):
            buf = torch.full((padded,) + tuple(src.shape[1:]), fill, dtype=src.dtype, device=device)
            buf[:n] = src
            dst[phys] = buf.view((npg, ps) + tuple(src.shape[1:]))
        scatter(kidx_cache, k8)
        scatter(kscale_cache, ks, 1)
        scatter(k_cache, kb)
        scatter(v_cache, vb)
        del k8, ks, kb, vb

    q_idx, q_scale = quantize_e4m3_per_token(q_src)
    return dict(q_idx=q_idx, q_scale=q_scale, w=w.contiguous(), q=q.contiguous(),
                kidx_cache=kidx_cache, kscale_cache=kscale_cache,
                k_cache=k_cache, v_cache=v_cache, block_table=block_table,
                context_lens=torch.tensor(lens, dtype=torch.int32, device=device),
                needle_pos=needle_pos)


def prefill_flops(spec: PrefillSpec) -> Dict[str, float]:
    """Algorithmic work of one prefill (what the method must compute)."""
    L, k = spec.L, spec.k
    pairs = L * (L + 1) / 2
    sel = sum(min(k, t + 1) for t in range(L)) if L <= 1 << 16 else (
        k * (k + 1) / 2 + (L - k) * k)
    return dict(pairs=pairs, selected=sel,
                indexer_flop=2.0 * spec.H_I * spec.d_I * pairs,
                attn_flop=4.0 * spec.H_q * spec.d * sel)


def decode_kv_to_fp8(inp: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Copy of a decode input whose K/V caches are stored as FP8 E4M3 codes with
    one fp32 scale per cached token (storage packing only: the bf16 cache rows
    are packed by quantize_e4m3_per_token).  k_cache/v_cache become uint8
    [P, ps, d]; k_cache_scale/v_cache_scale are added as f32 [P, ps]."""
    out = dict(inp)
    for name in ("k", "v"):
        c = inp[name + "_cache"]
        P, ps, d = c.shape
        codes, scale = quantize_e4m3_per_token(c.reshape(P * ps, d).float())
        out[name + "_cache"] = codes.reshape(P, ps, d).contiguous()
        out[name + "_cache_scale"] = scale.reshape(P, ps).contiguous()
    return out


def split_decode_input(inp: Dict[str, torch.Tensor], G: int):
    """Cut a decode input's caches into G contiguous shards of every sequence's
    positions (shard g of a context of n positions: [floor(g n / G),
    floor((g + 1) n / G))), each shard in paged caches of its own, the pages
    in reverse order so that paging is exercised.  Returns a list of
    (shard dict, pos_base int32 [B]); queries are shared.  Only re-packs
    cache rows."""
    dev = inp["q"].device
    ps = inp["kidx_cache"].shape[1]
    lens = inp["context_lens"].cpu().long()
    B = lens.numel()
    bt = inp["block_table"].cpu().long()
    g_ = torch.arange(G + 1, dtype=torch.int64)[:, None]
    edges = (g_ * lens[None, :]) // G
    cache_keys = [k for k in ("kidx_cache", "kscale_cache", "k_cache", "v_cache", "k_cache_scale",
                              "v_cache_scale") if k in inp]
    flat = {k: inp[k].reshape((-1,) + tuple(inp[k].shape[2:])) for k in cache_keys}
    shards = []
    for g in range(G):
        base, n = edges[g], edges[g + 1] - edges[g]
        pages = [(int(x) + ps - 1) // ps for x in n]
        P = max(sum(pages), 1)
        order = torch.arange(P - 1, -1, -1, dtype=torch.int64)
        table = torch.full((B, max(max(pages), 1)), -1, dtype=torch.int32)
        sh = {k: inp[k] for k in ("q_idx", "q_scale", "w", "q")}
        for k in cache_keys:
            fill = 1 if "scale" in k else 0
            sh[k] = torch.full((P * ps,) + tuple(inp[k].shape[2:]), fill, dtype=inp[k].dtype, device=dev)
        off = 0
        for b in range(B):
            table[b, :pages[b]] = order[off:off + pages[b]].int()
            p = torch.arange(int(base[b]), int(base[b] + n[b]), dtype=torch.int64)
            src = bt[b, p // ps] * ps + p % ps
            local = torch.arange(int(n[b]), dtype=torch.int64)
            dst = table[b].long()[local // ps] * ps + local % ps
            for k in cache_keys:
                sh[k][dst.to(dev)] = flat[k][src.to(dev)]
            off += pages[b]
        for k in cache_keys:
            sh[k] = sh[k].view((P, ps) + tuple(inp[k].shape[2:]))
        sh["block_table"] = table.to(dev)
        sh["context_lens"] = n.to(torch.int32).to(dev)
        shards.append((sh, base.to(torch.int32).to(dev)))
    return shards
