"""The rank orchestration of the split-context decode (split_decode_step: the
two messages, their layout and the collectives), run as gloo ranks on the
host.  Each rank holds one contiguous shard of every sequence's cache; the
per-rank steps are played by CPU stand-ins built on the oracle (its decode's
scores and selection on the shard, its sparse attention over the shard's
selected rows) and on the textbook definitions of the two merges.  The step
must reproduce the oracle's whole-context decode on every rank: the same
selection, and the same attention within the bf16 rounding of the messages."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SM = 0.125


class OracleOps:
    """CPU stand-ins for the four per-rank steps."""

    def select(self, shard, pos_base, k, max_context, cand_pos, cand_score, ws):
        from oracle import oracle
        res = oracle.decode(shard, k, SM, want_scores=True)
        li = res["idx"]
        base = pos_base.numpy().astype(np.int64)
        pos = np.where(li >= 0, li + base[:, None], -1).astype(np.int32)
        sc = np.full(li.shape, -np.inf, np.float32)
        for b in range(li.shape[0]):
            m = li[b] >= 0
            sc[b, m] = res["scores"][b, li[b, m]]
        cand_pos.copy_(torch.from_numpy(pos))
        cand_score.copy_(torch.from_numpy(sc))

    def merge_selections(self, cand_pos, cand_score, idx_out, ws):
        G, B, k = cand_pos.shape
        P, S = cand_pos.numpy(), cand_score.numpy()
        idx_out.fill_(-1)
        for b in range(B):
            p, s = P[:, b].reshape(-1), S[:, b].reshape(-1).astype(np.float64)
            m = p >= 0
            p, s = p[m], s[m]
            sel = np.sort(p[np.lexsort((p, -s))[:k]])               # score desc, then lower position
            idx_out[b, :sel.size] = torch.from_numpy(sel)

    def attend(self, shard, pos_base, idx, sm_scale, out, lse, ws):
        from oracle import oracle
        ps = shard["k_cache"].shape[1]
        d = shard["k_cache"].shape[2]
        kc, vc = shard["k_cache"].reshape(-1, d), shard["v_cache"].reshape(-1, d)
        bt = shard["block_table"].numpy().astype(np.int64)
        n = shard["context_lens"].numpy()
        base = pos_base.numpy()
        for b in range(idx.shape[0]):
            g = idx[b].numpy()
            loc = g[(g >= 0) & (g >= base[b]) & (g < base[b] + n[b])] - base[b]
            if loc.size == 0:
                out[b].zero_()
                lse[b].fill_(-float("inf"))
                continue
            slot = torch.from_numpy(bt[b, loc // ps] * ps + loc % ps)
            o, l = oracle.sparse_attn(shard["q"][b:b + 1], kc[slot], vc[slot],
                                      np.arange(loc.size, dtype=np.int32)[None], [0], sm_scale)
            out[b].copy_(torch.from_numpy(o[0]).to(torch.bfloat16))
            lse[b].copy_(torch.from_numpy(l[0]).float())

    def merge_partials(self, part_out, part_lse, out, lse):
        L = part_lse.double()
        tot = torch.logsumexp(L, dim=0)
        w = torch.exp(L - tot[None])
        w = torch.nan_to_num(w, nan=0.0)
        out.copy_((w[..., None] * part_out.double()).sum(0).to(torch.bfloat16))
        lse.copy_(tot.float())


def _rank_main(rank, world, port, root):
    import sys
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch.distributed as dist
    import dsa_synth
    from oracle import oracle
    from long_context_fp8_b200 import split_decode

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        spec = dsa_synth.DecodeSpec("split_cpu", context_lens=(3000, 1000, 150, 2049), H_I=8, d_I=64, k=96,
                                    H_q=8, d=64, page_size=64, needle_frac=0.01, needle_min_age=0, seed=12)
        inp = dsa_synth.make_decode(spec)                 # the same problem on every rank
        shard, base = dsa_synth.split_decode_input(inp, world)[rank]
        max_ctx = int(max(int(s["context_lens"].max()) for s, _ in dsa_synth.split_decode_input(inp, world)))
        out, lse, idx = split_decode.split_decode_step(shard, base, spec.k, max_ctx, sm_scale=SM, ops=OracleOps())
        ref = oracle.decode(inp, spec.k, SM)
        assert np.array_equal(idx.numpy(), ref["idx"]), "split selection differs from the whole-context one"
        from gpu_common import assert_attn_close
        assert_attn_close(out.float().numpy(), ref["out"], lse.numpy(), ref["lse"], f"rank {rank}")
        # every rank holds the same result
        digest = torch.tensor([float(out.double().sum()), float(lse.double().sum()), float(idx.double().sum())],
                              dtype=torch.float64)
        got = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(got, digest)
        assert all(torch.equal(g, digest) for g in got)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_decode_step_gloo(world):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    mp.spawn(_rank_main, args=(world, _free_port(), root), nprocs=world, join=True)


def test_shard_bounds_cover_every_position_once():
    from long_context_fp8_b200 import split_decode
    lens = [1048576, 786432, 524288, 262144, 7, 8]
    for G in (1, 2, 3, 8):
        base, n = split_decode.shard_bounds(lens, G)
        assert torch.equal(n.sum(0), torch.tensor(lens))
        assert torch.equal(base[0], torch.zeros(len(lens), dtype=torch.int64))
        assert torch.equal(base[1:], (base + n)[:-1])                 # contiguous, in order
        assert int((n.max(0).values - n.min(0).values).max()) <= 1    # near-equal


def test_messages_layout():
    from long_context_fp8_b200 import split_decode
    B, H, d, G, k = 3, 8, 64, 4, 16
    send, recv = split_decode.candidate_message(B, k, G, "cpu")
    p, s = split_decode.candidate_views(send)
    p.copy_(torch.arange(B * k, dtype=torch.int32).view(B, k))
    s.copy_(torch.full((B, k), -2.5))
    assert send.numel() * 4 == 8 * B * k                               # 8 bytes per candidate
    assert torch.equal(split_decode.candidate_views(send)[1], torch.full((B, k), -2.5))
    W = split_decode.partial_words(B, H, d)
    assert W % 4 == 0 and W * 4 >= 2 * B * H * d + 4 * B * H
    psend, precv = split_decode.partial_message(B, H, d, G, "cpu")
    o, l = split_decode.partial_views(precv, B, H, d)
    assert o.shape == (G, B, H, d) and l.shape == (G, B, H)
    assert o.stride(0) == 2 * W and l.stride(0) == W
    o[2].fill_(1.5)
    l[2].fill_(-3.0)
    o2, l2 = split_decode.partial_views(precv[2], B, H, d)
    assert bool((o2 == 1.5).all()) and bool((l2 == -3.0).all())


def test_union_of_shard_topk_holds_the_whole_topk():
    """The exactness the split decode rests on, checked on the oracle's own
    selector: the top-k of the union of the shards' top-k lists (score
    descending, ties to the lower position) is the top-k of the whole row.
    Scores are drawn from a few values so that ties are the rule, and shard
    sizes range from below k to several times k."""
    from oracle import oracle
    rng = np.random.default_rng(21)
    for trial in range(40):
        n = int(rng.integers(1, 3000))
        k = int(rng.integers(1, 300))
        G = int(rng.integers(1, 9))
        row = rng.integers(-6, 7, size=n).astype(np.float64) * 0.25
        whole = oracle.topk(row[None], [n - 1], k)[0]
        edges = [(g * n) // G for g in range(G + 1)]
        cand_p, cand_s = [], []
        for g in range(G):
            a, b = edges[g], edges[g + 1]
            if b == a:
                continue
            sel = oracle.topk(row[None, a:b], [b - a - 1], k)[0]
            sel = sel[sel >= 0]
            cand_p.append(sel + a)
            cand_s.append(row[a:b][sel])
        p, s = np.concatenate(cand_p), np.concatenate(cand_s)
        merged = np.sort(p[np.lexsort((p, -s))[:k]])
        want = whole[whole >= 0]
        assert np.array_equal(merged, want), (trial, n, k, G)


def test_partition_merge_equals_whole_attention():
    """The partial-attention merge: the oracle's attention over a selection
    equals the log-sum-exp merge of its attentions over any partition of the
    selection (fp64, to rounding)."""
    from oracle import oracle
    g = torch.Generator().manual_seed(22)
    H, d, n = 8, 64, 300
    q = torch.randn((1, H, d), generator=g).to(torch.bfloat16)
    K = torch.randn((n, d), generator=g).to(torch.bfloat16)
    V = torch.randn((n, d), generator=g).to(torch.bfloat16)
    o_all, l_all = oracle.sparse_attn(q, K, V, np.arange(n, dtype=np.int32)[None], [0], 0.125)
    rng = np.random.default_rng(5)
    for parts in (2, 3, 7):
        cuts = np.sort(rng.choice(np.arange(1, n), size=parts - 1, replace=False))
        bounds = [0, *cuts.tolist(), n]
        outs, lses = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            o, l = oracle.sparse_attn(q, K[a:b], V[a:b], np.arange(b - a, dtype=np.int32)[None], [0], 0.125)
            outs.append(o[0]); lses.append(l[0])
        L = np.stack(lses)                                      # [parts, H]
        tot = np.logaddexp.reduce(L, axis=0)
        merged = (np.exp(L - tot)[..., None] * np.stack(outs)).sum(0)
        assert np.allclose(tot, l_all[0], rtol=0, atol=1e-12)
        assert np.allclose(merged, o_all[0], rtol=0, atol=1e-12)


def test_split_decode_input_repacks_rows_exactly():
    """Every cached row of every sequence lands in exactly one shard, at its
    local position, with the same bytes (index key, its scale, K, V and, for
    FP8 K/V caches, their scales); shard tables point only at the shard's
    own pages; the queries are shared."""
    import dsa_synth
    spec = dsa_synth.DecodeSpec("split_repack", context_lens=(1000, 64, 1, 2049, 130), H_I=8, d_I=64, k=32,
                                H_q=8, d=64, page_size=64, needle_frac=0.0, needle_min_age=0, seed=31)
    for inp in (dsa_synth.make_decode(spec), dsa_synth.decode_kv_to_fp8(dsa_synth.make_decode(spec))):
        ps = spec.page_size
        keys = [k for k in ("kidx_cache", "kscale_cache", "k_cache", "v_cache", "k_cache_scale", "v_cache_scale")
                if k in inp]
        for G in (1, 3, 4):
            shards = dsa_synth.split_decode_input(inp, G)
            seen = [np.zeros(n, dtype=np.int64) for n in spec.context_lens]
            for sh, base in shards:
                for k_ in ("q_idx", "q_scale", "w", "q"):
                    assert sh[k_] is inp[k_]
                P = sh["kidx_cache"].shape[0]
                for b, n_all in enumerate(spec.context_lens):
                    n, pb = int(sh["context_lens"][b]), int(base[b])
                    pages = (n + ps - 1) // ps
                    tab = sh["block_table"][b]
                    assert bool((tab[:pages] >= 0).all()) and bool((tab[:pages] < P).all())
                    assert bool((tab[pages:] == -1).all())
                    for p in range(n):
                        g_slot = int(inp["block_table"][b, (pb + p) // ps]) * ps + (pb + p) % ps
                        l_slot = int(tab[p // ps]) * ps + p % ps
                        for k_ in keys:
                            full = inp[k_].reshape((-1,) + tuple(inp[k_].shape[2:]))
                            part = sh[k_].reshape((-1,) + tuple(sh[k_].shape[2:]))
                            assert torch.equal(full[g_slot], part[l_slot]), (k_, G, b, p)
                        seen[b][pb + p] += 1
            for b in range(len(seen)):
                assert bool((seen[b] == 1).all()), (G, b)
