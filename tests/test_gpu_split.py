"""Decode of contexts split over G devices (dsa_decode_select,
dsa_merge_selections, dsa_decode_attend, dsa_merge_partials through the C
ABI), the G shards run one after another on one GPU, the two all-gathers
played by the shards writing into their slots of the gathered messages.

Bars: the merged selection equals the whole-context dsa_decode selection bit
for bit (the shards' indexer scores are the whole context's, the merge is an
exact top-k) and overlaps the oracle's >= 0.999; the merged attention is within
2e-2 + 1e-2 |o| of the fp64 attention over that selection (the partials are
bf16 like any output, then merged in fp32); the merge kernels equal their
definitions (a sort with ties to the lower position; the log-sum-exp formula)
on hand-made lists."""
import math

import numpy as np
import pytest
import torch

import dsa_synth
from oracle import oracle
from long_context_fp8_b200 import dsa, split_decode

from gpu_common import OVERLAP_MIN, assert_attn_close, overlap, sm_of, to_dev

pytestmark = pytest.mark.gpu


def _spec(lens, k, seed):
    return dsa_synth.DecodeSpec("split", context_lens=tuple(lens), H_I=64, d_I=128, k=k, H_q=128, d=128,
                                page_size=64, needle_frac=0.01, needle_min_age=0, seed=seed)


def _emulated_split(inp, G, k, sm):
    """The split decode step with G shards run in turn on this GPU, through the
    packed messages the ranks exchange.  Returns (out, lse, idx, parts)."""
    shards = dsa_synth.split_decode_input(inp, G)
    B, H_q, d = inp["q"].shape
    max_ctx = max(int(s["context_lens"].max()) for s, _ in shards)
    ws = dsa.workspace(dsa.split_workspace_size(G, B, max_ctx, H_q, d, k), "cuda")
    _, recv = split_decode.candidate_message(B, k, G, "cuda")
    for g, (sh, base) in enumerate(shards):
        pos, score = split_decode.candidate_views(recv[g])
        dsa.dsa_decode_select(sh, base, k, max_ctx, cand_pos=pos, cand_score=score, ws=ws)
        assert dsa.dsa_stream_status(ws) == 0
    idx = dsa.dsa_merge_selections(*split_decode.candidate_views(recv), ws=ws)
    assert dsa.dsa_stream_status(ws) == 0
    _, precv = split_decode.partial_message(B, H_q, d, G, "cuda")
    for g, (sh, base) in enumerate(shards):
        o, l = split_decode.partial_views(precv[g], B, H_q, d)
        dsa.dsa_decode_attend(sh, base, idx, sm, out=o, lse=l, ws=ws)
        assert dsa.dsa_stream_status(ws) == 0
    out, lse = dsa.dsa_merge_partials(*split_decode.partial_views(precv, B, H_q, d))
    torch.cuda.synchronize()
    return out, lse, idx, split_decode.partial_views(precv, B, H_q, d)


def _attention_over(inp, idx, sm, fp8=False):
    """fp64 attention of each sequence's query over the listed positions."""
    bt = inp["block_table"].cpu().numpy()
    ps = inp["kidx_cache"].shape[1]
    d = inp["q"].shape[-1]
    kc, vc = inp["k_cache"].cpu().reshape(-1, d), inp["v_cache"].cpu().reshape(-1, d)
    outs, lses = [], []
    for b in range(idx.shape[0]):
        sel = idx[b][idx[b] >= 0]
        slot = torch.from_numpy(bt[b, sel // ps].astype(np.int64) * ps + sel % ps)
        if fp8:
            ks = inp["k_cache_scale"].cpu().reshape(-1)[slot].double()
            vs = inp["v_cache_scale"].cpu().reshape(-1)[slot].double()
            K = kc[slot].view(torch.float8_e4m3fn).double() * ks[:, None]
            V = vc[slot].view(torch.float8_e4m3fn).double() * vs[:, None]
        else:
            K, V = kc[slot], vc[slot]
        o, l = oracle.sparse_attn(inp["q"][b:b + 1].cpu(), K, V, np.arange(sel.size, dtype=np.int32)[None], [0], sm)
        outs.append(o[0]); lses.append(l[0])
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("lens,k,G", [((5000, 3000, 777, 12000), 512, 2), ((5000, 3000, 777, 12000), 512, 3),
                                      ((20000, 9000, 4100), 2048, 8), ((700, 129, 64), 128, 4)])
def test_split_decode_equals_whole_context(lens, k, G):
    inp = to_dev(dsa_synth.make_decode(_spec(lens, k, seed=80 + G + k)))
    sm = sm_of(128)
    out, lse, idx, _ = _emulated_split(inp, G, k, sm)
    w_out, w_lse, w_idx = dsa.dsa_decode(inp, k, max(lens), sm)
    torch.cuda.synchronize()
    assert torch.equal(idx, w_idx), "merged selection differs from the whole-context selection"
    idx_np = idx.cpu().numpy()
    ref = oracle.decode({k_: (v.cpu() if torch.is_tensor(v) else v) for k_, v in inp.items()}, k, sm)
    mean_ov, min_ov = overlap(idx_np, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    ro, rl = _attention_over(inp, idx_np, sm)
    assert_attn_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, f"split G={G}")


def test_split_decode_kv8():
    lens, k, G = (6000, 2500, 9000), 512, 4
    inp = to_dev(dsa_synth.decode_kv_to_fp8(dsa_synth.make_decode(_spec(lens, k, seed=91))))
    sm = sm_of(128)
    out, lse, idx, _ = _emulated_split(inp, G, k, sm)
    w_out, w_lse, w_idx = dsa.dsa_decode_kv8(inp, k, max(lens), sm_scale=sm)
    torch.cuda.synchronize()
    assert torch.equal(idx, w_idx)
    ro, rl = _attention_over(inp, idx.cpu().numpy(), sm, fp8=True)
    assert_attn_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, "split kv8")


def test_split_decode_ragged_1m_fullsize():
    """The ragged long-context workload (1M, 768K, 512K, 256K positions, k 512)
    split over 8 shards: the selection equals the whole-context decode's and
    the output agrees with it within the attention tolerance."""
    spec = dsa_synth.decode_spec("dec_ragged")
    inp = dsa_synth.make_decode(spec, device="cuda")
    sm = sm_of(spec.d)
    out, lse, idx, _ = _emulated_split(inp, 8, spec.k, sm)
    w_out, w_lse, w_idx = dsa.dsa_decode(inp, spec.k, max(spec.context_lens), sm)
    torch.cuda.synchronize()
    assert torch.equal(idx, w_idx)
    # both outputs are bf16 roundings of one fp32-accurate result: within two bf16 ulps
    diff = (out.float() - w_out.float()).abs()
    assert float(diff.max()) <= 2e-2, float(diff.max())
    assert float((lse - w_lse).abs().max()) <= 1e-3


def test_merge_selections_ties_padding_and_strides():
    """Hand-made candidate lists: equal scores across shards go to the lower
    position; -1 entries never win; shorter unions are -1 padded; the lists
    read through a dim-0 stride (a packed message) as well as densely."""
    rng = np.random.default_rng(3)
    G, B, k = 5, 6, 96
    pos = np.full((G, B, k), -1, np.int32)
    sc = np.full((G, B, k), -np.inf, np.float32)
    for b in range(B):
        base = 0
        for g in range(G):
            n = int(rng.integers(0, k + 1)) if b != 5 else 3   # row 5: union smaller than k
            p = np.sort(rng.choice(1000, size=n, replace=False)).astype(np.int32) + base
            s = rng.integers(-4, 5, size=n).astype(np.float32)      # many exact ties
            pos[g, b, :n], sc[g, b, :n] = p, s
            base += 1000
    want = np.full((B, k), -1, np.int32)
    for b in range(B):
        m = pos[:, b, :].reshape(-1) >= 0
        p, s = pos[:, b, :].reshape(-1)[m], sc[:, b, :].reshape(-1)[m]
        order = np.lexsort((p, -s.astype(np.float64)))[:k]
        sel = np.sort(p[order])
        want[b, :sel.size] = sel
    dp, ds = torch.from_numpy(pos).cuda(), torch.from_numpy(sc).cuda()
    got = dsa.dsa_merge_selections(dp, ds)
    assert np.array_equal(got.cpu().numpy(), want)
    packed = torch.empty((G, 2, B, k), dtype=torch.int32, device="cuda")
    pv, sv = split_decode.candidate_views(packed)
    pv.copy_(dp); sv.copy_(ds)
    got2 = dsa.dsa_merge_selections(pv, sv)
    assert np.array_equal(got2.cpu().numpy(), want)


def test_merge_partials_lse_formula():
    """out = sum_g exp(lse_g - lse) out_g, lse = log sum_g exp(lse_g), with a
    head whose partials are all empty (-inf: zeros out) and empty partials
    mixed with full ones."""
    g = torch.Generator().manual_seed(9)
    G, B, H, d = 3, 4, 256, 128
    po = torch.randn((G, B, H, d), generator=g).to(torch.bfloat16)
    pl = (torch.randn((G, B, H), generator=g) * 3).float()
    pl[1, 0, :] = -math.inf
    pl[:, 2, 7] = -math.inf
    po[1, 0] = 0
    po[:, 2, 7] = 0
    lse64 = torch.logsumexp(pl.double(), dim=0)
    wts = torch.exp(pl.double() - lse64[None])
    wts[torch.isnan(wts)] = 0
    want = (wts[..., None] * po.double()).sum(0)
    out, lse = dsa.dsa_merge_partials(po.cuda(), pl.cuda())
    torch.cuda.synchronize()
    fin = torch.isfinite(lse64)
    assert torch.equal(torch.isneginf(lse.cpu()), ~fin)
    assert float((lse.cpu().double()[fin] - lse64[fin]).abs().max()) <= 1e-4
    # one bf16 rounding of the fp32 merge: half an ulp, 2^-9 relative
    err = (out.cpu().double() - want).abs()
    assert bool((err <= 1e-3 + 4e-3 * want.abs()).all()), float(err.max())
    assert float(out.cpu()[2, 7].abs().max()) == 0.0
    # G = 1 reproduces its only partial
    o1, l1 = dsa.dsa_merge_partials(po[:1].cuda(), pl[:1].cuda())
    assert torch.equal(o1.cpu(), po[0]) and torch.equal(l1.cpu(), pl[0])


def test_decode_select_reports_negative_base():
    inp = to_dev(dsa_synth.make_decode(_spec((300, 200), 64, seed=95)))
    base = torch.tensor([0, -5], dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.split_workspace_size(1, 2, 300, 128, 128, 64), "cuda")
    pos, _ = dsa.dsa_decode_select(inp, base, 64, 300, ws=ws)
    assert dsa.dsa_stream_status(ws) == 1                           # DSA_ERR_INVALID_ARG
    assert int((pos[1] >= 0).sum()) == 0 and int((pos[0] >= 0).sum()) == 64


def test_split_single_shard_equals_decode_bit_for_bit():
    """G = 1: the merge of one candidate list is that list, the attention is the
    whole-context decode's own, and the merge of one partial multiplies by
    exp(0) = 1 -- every output equals dsa_decode's bit for bit."""
    lens, k = (5000, 3000, 777), 512
    inp = to_dev(dsa_synth.make_decode(_spec(lens, k, seed=97)))
    sm = sm_of(128)
    out, lse, idx, _ = _emulated_split(inp, 1, k, sm)
    w_out, w_lse, w_idx = dsa.dsa_decode(inp, k, max(lens), sm)
    torch.cuda.synchronize()
    assert torch.equal(idx, w_idx) and torch.equal(out, w_out) and torch.equal(lse, w_lse)


def test_split_shard_holding_none_of_the_selection():
    """Shard 0's index keys are zeroed (their scores are 0 while the others'
    are positive), so the merged selection holds none of its positions: its
    partial is empty (lse -inf, zeros) and the merge must ignore it."""
    lens, k, G = (6000, 4000, 9000), 256, 4
    inp = dsa_synth.make_decode(_spec(lens, k, seed=98))
    ps = inp["kidx_cache"].shape[1]
    flat = inp["kidx_cache"].view(-1, inp["kidx_cache"].shape[2])
    for b, n in enumerate(lens):
        p = torch.arange(n // G)
        flat[inp["block_table"][b, p // ps].long() * ps + p % ps] = 0
    inp = to_dev(inp)
    sm = sm_of(128)
    out, lse, idx, (p_out, p_lse) = _emulated_split(inp, G, k, sm)
    w_out, w_lse, w_idx = dsa.dsa_decode(inp, k, max(lens), sm)
    torch.cuda.synchronize()
    assert torch.equal(idx, w_idx)
    for b, n in enumerate(lens):
        sel = idx[b][idx[b] >= 0]
        assert int(sel.numel()) == k and int((sel < n // G).sum()) == 0
    assert bool(torch.isneginf(p_lse[0]).all()) and float(p_out[0].float().abs().max()) == 0.0
    ro, rl = _attention_over(inp, idx.cpu().numpy(), sm)
    assert_attn_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, "shard without selection")


def test_split_zero_length_shard_is_reported():
    """A sequence shorter than G leaves some shards without positions: the
    select reports DSA_ERR_INVALID_ARG and returns no candidates for it, the
    other sequences' candidates are unaffected."""
    lens, k, G = (2, 300), 64, 4
    inp = to_dev(dsa_synth.make_decode(_spec(lens, k, seed=99)))
    shards = dsa_synth.split_decode_input(inp, G)
    sh, base = shards[0]
    assert sh["context_lens"].tolist() == [0, 75]
    ws = dsa.workspace(dsa.split_workspace_size(G, 2, 75, 128, 128, k), "cuda")
    pos, score = dsa.dsa_decode_select(sh, base, k, 75, ws=ws)
    assert dsa.dsa_stream_status(ws) == 1                           # DSA_ERR_INVALID_ARG
    assert bool((pos[0] == -1).all()) and bool(torch.isneginf(score[0]).all())
    assert int((pos[1] >= 0).sum()) == k and int(pos[1].max()) < 75
