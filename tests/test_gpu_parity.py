"""Stage-by-stage parity of the CUDA path (through the C ABI) with the fp64
CPU oracle, on seeded inputs small enough for the oracle to finish in seconds
but spanning several tiles and ragged tails.  Tolerances: see gpu_common."""
import math

import numpy as np
import pytest
import torch

import dsa_synth
from oracle import oracle
from long_context_fp8_b200 import dsa

from gpu_common import (ATT_ATOL, OVERLAP_MIN, assert_attn_close, assert_scores_close,
                        check_selection_valid, overlap, sm_of, to_dev)

pytestmark = pytest.mark.gpu


def fp8_spec(L, H_I=64, H_q=16, k=128, seed=11, n_needles=None, d=128):
    return dsa_synth.PrefillSpec("mid", L=L, H_I=H_I, d_I=128, k=k, H_q=H_q, d=d, fp8=True,
                                 n_needles=max(1, L // 100) if n_needles is None else n_needles,
                                 seed=seed)


# ------------------------------------------------------------------ indexer

@pytest.mark.parametrize("L,H_I,rows", [(1000, 64, (0, 1000)), (777, 64, (130, 333)),
                                        (300, 8, (0, 300)), (1, 64, (0, 1)), (513, 128, (500, 13)),
                                        (900, 12, (100, 700)), (700, 32, (0, 700)), (400, 1, (0, 400))])
def test_index_scores_fp8(L, H_I, rows):
    inp = dsa_synth.make_prefill(fp8_spec(L, H_I=H_I, seed=L + H_I))
    dev = to_dev(inp)
    r0, n = rows
    got = dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"], dev["w"],
                               row_begin=r0, row_count=n).cpu().numpy()
    ref = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"],
                              np.arange(r0, r0 + n))
    assert_scores_close(got, ref, f"L={L} H={H_I}")


def test_index_scores_fp8_leading_dim_and_empty():
    inp = dsa_synth.make_prefill(fp8_spec(200))
    dev = to_dev(inp)
    out = torch.full((50, 300), 7.0, device="cuda")
    dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"], dev["w"],
                         row_begin=150, row_count=50, out=out, ld=300)
    o = out.cpu().numpy()
    assert np.all(o[:, 200:] == 7.0)            # columns past T untouched
    ref = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"],
                              np.arange(150, 200))
    assert_scores_close(o[:, :200], ref)
    empty = dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"],
                                 dev["w"], row_begin=200, row_count=0)
    assert empty.shape[0] == 0


def test_index_scores_f32_tiny():
    spec = dsa_synth.prefill_spec("tiny")
    inp = dsa_synth.make_prefill(spec)
    dev = to_dev(inp)
    got = dsa.dsa_index_scores(dev["q_idx"], None, dev["k_idx"], None, dev["w"]).cpu().numpy()
    ref = oracle.index_scores(inp["q_idx"], None, inp["k_idx"], None, inp["w"], np.arange(spec.L))
    assert_scores_close(got, ref, "tiny")


# ------------------------------------------------------------------ top-k

def _topk_check(scores_np, k, row_begin=0):
    rows = np.arange(row_begin, row_begin + scores_np.shape[0])
    s = torch.from_numpy(scores_np.astype(np.float32)).cuda()
    got = dsa.dsa_topk(s, k, row_begin=row_begin).cpu().numpy()
    ref = oracle.topk(scores_np.astype(np.float32).astype(np.float64), rows, k)
    np.testing.assert_array_equal(got, ref)
    return got


@pytest.mark.parametrize("k", [1, 5, 64, 300, 2048])
def test_topk_bit_exact_random_with_ties(k):
    rng = np.random.default_rng(k)
    T = 3000
    sc = (np.round(rng.standard_normal((T, T)) * 64) / 64).astype(np.float32)   # many ties
    rows = np.sort(rng.choice(T, 200, replace=False))
    rows[-1] = T - 1
    # topk reads rows as positions row_begin + r, so build a dense block per test row
    for r0 in (0, 1500, T - 64):
        _topk_check(sc[r0:r0 + 64], k, row_begin=r0)


def test_topk_degenerate_rows():
    T, k = 5000, 100
    sc = np.zeros((8, T), np.float32)
    sc[1] = -0.0
    sc[2, ::2] = -0.0                         # +0 / -0 mixed: equal keys
    sc[3] = np.arange(T, dtype=np.float32)    # monotone: the last k
    sc[4] = -np.arange(T, dtype=np.float32)   # decreasing: the first k
    sc[5] = 1e30
    sc[5, 4000:] = -1e30
    sc[6] = np.float32(1.0) + np.float32(2 ** -23) * (np.arange(T) % 3)   # near ties across one ulp
    sc[7] = -np.inf
    sc[7, 4321] = 0.0
    got = _topk_check(sc, k, row_begin=T - 8)
    assert got[0].tolist() == list(range(k))


def test_topk_on_gpu_indexer_scores():
    inp = dsa_synth.make_prefill(fp8_spec(2500, seed=5))
    dev = to_dev(inp)
    sc = dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"], dev["w"])
    got = dsa.dsa_topk(sc, 256).cpu().numpy()
    ref = oracle.topk(sc.cpu().numpy().astype(np.float64), np.arange(2500), 256)
    np.testing.assert_array_equal(got, ref)
    check_selection_valid(got, np.arange(2500), 256)


# ------------------------------------------------------------------ sparse attention

def _rand_idx(T, k, seed, causal=True, holes=True):
    rng = np.random.default_rng(seed)
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        n = min(k, t + 1) if causal else k
        sel = np.sort(rng.choice(t + 1 if causal else T, n, replace=False))
        idx[t, :n] = sel
        if holes and t % 7 == 3 and n > 2:
            idx[t, 1] = -1                     # a hole inside the list
    return idx


@pytest.mark.parametrize("H_q,d,k", [(16, 128, 200), (128, 128, 64), (8, 64, 100), (24, 128, 70),
                                     (256, 128, 65)])
def test_sparse_attn_bf16(H_q, d, k):
    T = 300
    g = torch.Generator().manual_seed(H_q * 1000 + k)
    q = torch.randn((T, H_q, d), generator=g).to(torch.bfloat16)
    K = torch.randn((T, d), generator=g).to(torch.bfloat16)
    V = torch.randn((T, d), generator=g).to(torch.bfloat16)
    idx = _rand_idx(T, k, seed=k)
    out, lse = dsa.dsa_sparse_attn(q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(idx).cuda(), sm_of(d))
    ref, ref_lse = oracle.sparse_attn(q, K, V, idx, np.arange(T), sm_of(d))
    assert_attn_close(out.float().cpu().numpy(), ref, lse.cpu().numpy(), ref_lse, f"H={H_q} d={d}")


def test_sparse_attn_empty_and_single_rows():
    T, H_q, d, k = 50, 16, 128, 8
    g = torch.Generator().manual_seed(3)
    q = torch.randn((T, H_q, d), generator=g).to(torch.bfloat16)
    K = torch.randn((T, d), generator=g).to(torch.bfloat16)
    V = torch.randn((T, d), generator=g).to(torch.bfloat16)
    idx = np.full((T, k), -1, np.int32)
    idx[1::2, 0] = np.arange(1, T, 2)          # odd rows: exactly one selected row (itself)
    idx[10, 3] = 10_000                          # out of range: ignored
    out, lse = dsa.dsa_sparse_attn(q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(idx).cuda())
    out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(out[0::2] == 0.0) and np.all(np.isneginf(lse[0::2]))
    np.testing.assert_allclose(out[1::2], np.repeat(V.float().numpy()[1::2][:, None], H_q, 1), atol=0)


def test_sparse_attn_f32_tiny():
    spec = dsa_synth.prefill_spec("tiny")
    inp = dsa_synth.make_prefill(spec)
    idx = _rand_idx(spec.L, spec.k, seed=1)
    out, lse = dsa.dsa_sparse_attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(),
                                   torch.from_numpy(idx).cuda(), sm_of(spec.d))
    ref, ref_lse = oracle.sparse_attn(inp["q"], inp["k"], inp["v"], idx, np.arange(spec.L), sm_of(spec.d))
    assert_attn_close(out.cpu().numpy(), ref, lse.cpu().numpy(), ref_lse, "tiny")


# ------------------------------------------------------------------ fused prefill

@pytest.mark.parametrize("name", ["tiny", "fp8-1500", "fp8-small-ws"])
def test_prefill_end_to_end(name):
    if name == "tiny":
        spec = dsa_synth.prefill_spec("tiny")
    else:
        spec = fp8_spec(1500, H_q=16, k=256, seed=17)
    inp = dsa_synth.make_prefill(spec)
    dev = to_dev(inp)
    ws = None
    if name == "fp8-small-ws":      # a fifth of the default: several passes of 128-row blocks
        full = dsa.prefill_workspace_size(spec.L, spec.H_I, spec.d_I, spec.H_q, spec.d, spec.k)
        ws = dsa.workspace(full // 5, "cuda")
    out, lse, idx = dsa.dsa_prefill(dev, spec.k, sm_of(spec.d), ws=ws)
    idx = idx.cpu().numpy()
    rows = np.arange(spec.L)
    check_selection_valid(idx, rows, spec.k)
    ref = oracle.prefill(inp, spec.k, sm_of(spec.d), rows)
    mean_ov, min_ov = overlap(idx, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    # attention parity given the GPU's own selection
    ref_out, ref_lse = oracle.sparse_attn(inp["q"], inp["k"], inp["v"], idx, rows, sm_of(spec.d))
    assert_attn_close(out.float().cpu().numpy(), ref_out, lse.cpu().numpy(), ref_lse, name)


def test_prefill_needles_recovered():
    """Sanity metric: needle recall of the GPU selection equals the oracle's."""
    spec = fp8_spec(2000, k=64, seed=23, n_needles=40)
    inp = dsa_synth.make_prefill(spec)
    _, _, idx = dsa.dsa_prefill(to_dev(inp), spec.k)
    idx = idx.cpu().numpy()
    src = inp["needle_src"].numpy()
    ref = oracle.prefill(inp, spec.k, sm_of(spec.d), src)
    pos = inp["needle_pos"].tolist()
    hits_g = sum(p in set(idx[t].tolist()) for p, t in zip(pos, src))
    hits_o = sum(p in set(ref["idx"][i].tolist()) for i, p in enumerate(pos))
    assert hits_g == hits_o and hits_o > 0, (hits_g, hits_o)


# ------------------------------------------------------------------ decode

def small_decode_spec(lens=(1000, 64, 1, 2049, 777), k=128, H_q=16, seed=31, ps=64):
    return dsa_synth.DecodeSpec("dsmall", context_lens=tuple(lens), H_I=64, d_I=128, k=k,
                                H_q=H_q, d=128, page_size=ps, needle_frac=0.01,
                                needle_min_age=0, seed=seed)


def decode_reference_attention(inp, idx, sm):
    """Oracle attention of each sequence's query over the GPU-selected positions."""
    bt = inp["block_table"].numpy()
    ps = inp["kidx_cache"].shape[1]
    kc = inp["k_cache"].reshape(-1, inp["k_cache"].shape[-1])
    vc = inp["v_cache"].reshape(-1, inp["v_cache"].shape[-1])
    B = idx.shape[0]
    outs, lses = [], []
    for b in range(B):
        sel = idx[b][idx[b] >= 0]
        slot = bt[b, sel // ps].astype(np.int64) * ps + sel % ps
        o, l = oracle.sparse_attn(inp["q"][b:b + 1], kc[slot], vc[slot],
                                  np.arange(sel.size, dtype=np.int32)[None, :], [0], sm)
        outs.append(o[0]); lses.append(l[0])
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("lens,k,H_q,ps", [((1000, 64, 1, 2049, 777), 128, 16, 64),
                                           ((5000, 3000), 512, 128, 16),
                                           ((300,) * 9, 64, 32, 32),
                                           ((1500, 129, 640), 100, 16, 128),
                                           ((700, 300), 64, 16, 256),
                                           ((900, 17), 64, 16, 48),       # 48: mma.sync indexer
                                           ((3000, 1000, 5000) * 6, 256, 16, 64),    # 18 short rows: whole rows on chip
                                           ((40000, 20000, 9000), 512, 16, 64)])    # chunked sampled threshold
def test_decode_end_to_end(lens, k, H_q, ps):
    spec = small_decode_spec(lens, k, H_q, seed=len(lens) + k, ps=ps)
    inp = dsa_synth.make_decode(spec)
    dev = to_dev(inp)
    out, lse, idx = dsa.dsa_decode(dev, k, max(lens), sm_of(128))
    ws_status = None
    idx = idx.cpu().numpy()
    ref = oracle.decode(inp, k, sm_of(128))
    check_selection_valid(idx, [n - 1 for n in lens], k)
    mean_ov, min_ov = overlap(idx, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    ro, rl = decode_reference_attention(inp, idx, sm_of(128))
    assert_attn_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, "decode")


def test_decode_bad_page_reported_not_faulted():
    spec = small_decode_spec((500, 300), 64, 16)
    inp = dsa_synth.make_decode(spec)
    dev = to_dev(inp)
    dev["block_table"][1, 2] = 10 ** 6           # out of range page id: checked in-kernel
    ws = dsa.workspace(dsa.decode_workspace_size(2, 500, 16, 128, 64), "cuda")
    dsa.dsa_decode(dev, 64, 500, ws=ws)
    assert dsa.dsa_stream_status(ws) == 1        # DSA_ERR_INVALID_ARG
    assert dsa.dsa_stream_status(ws) == 0        # reset by the read
    dev["block_table"][1, 2] = inp["block_table"][1, 2].item()
    out, _, _ = dsa.dsa_decode(dev, 64, 500, ws=ws)
    assert dsa.dsa_stream_status(ws) == 0
    assert torch.isfinite(out.float()).all()


def test_index_scores_fill_upper_off_leaves_upper_untouched():
    inp = dsa_synth.make_prefill(fp8_spec(700, seed=41))
    dev = to_dev(inp)
    out = torch.full((300, 700), 5.0, device="cuda")
    dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"], dev["w"],
                         row_begin=257, row_count=300, out=out, ld=700, fill_upper=False)
    o = out.cpu().numpy()
    ref = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"],
                              np.arange(257, 557))
    for r in range(300):
        t = 257 + r
        assert np.all(o[r, t + 1:] == 5.0)
        o[r, t + 1:] = -np.inf
    assert_scores_close(o, ref, "fill_upper=False")


def test_topk_candidate_overflow_falls_back_exactly():
    """Rows whose threshold bin holds more keys than fit on chip take the
    global-memory path; the result is still exact."""
    T, k = 30000, 100
    rng = np.random.default_rng(9)
    sc = np.zeros((4, T), np.float32)                       # 30000 equal keys
    sc[1] = np.float32(3.0) + np.float32(2 ** -20) * rng.integers(0, 4, T)   # 4 distinct, huge bins
    sc[2] = rng.standard_normal(T).astype(np.float32)       # ordinary row (on-chip path)
    sc[3, ::2] = 1.0                                         # 15000 ties at the top
    _topk_check(sc, k, row_begin=T - 4)


def test_decode_all_equal_scores_take_the_lowest_positions():
    """Every index key zero: all scores tie at 0, the selection is the k lowest
    positions; long rows overflow the on-chip candidate slots and take the
    global-memory path."""
    spec = small_decode_spec((40000, 9000, 100), k=300, H_q=16, seed=3)
    inp = dsa_synth.make_decode(spec)
    inp["kidx_cache"].zero_()
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_decode(dev, spec.k, 40000, sm_of(128))
    idx = idx.cpu().numpy()
    for b, n in enumerate(spec.context_lens):
        expect = list(range(min(n, spec.k))) + [-1] * (spec.k - min(n, spec.k))
        assert idx[b].tolist() == expect
    ref = oracle.decode(inp, spec.k, sm_of(128))
    np.testing.assert_array_equal(idx, ref["idx"])


def test_sparse_attn_running_max_jump_per_head():
    """A key whose logit is huge for one head only, placed in a later 128-row
    block: that head's running max jumps (its output is rescaled) while the
    other heads of the same warp keep theirs."""
    T, H, d, k = 400, 128, 128, 1024
    g = torch.Generator().manual_seed(77)
    q = torch.randn((T, H, d), generator=g).to(torch.bfloat16)
    K = torch.randn((T, d), generator=g).to(torch.bfloat16)
    V = torch.randn((T, d), generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(77)
    idx = np.full((T, k), -1, np.int32)
    for t in range(T):
        n = min(k, t + 1)
        idx[t, :n] = np.arange(n)
    # row t >= 300: key 290 (third block) aligned with head t % H, scaled up
    for t in range(300, T, 7):
        K[290] = (q[t, t % H].float() * 3.0).to(torch.bfloat16)
        break
    out, lse = dsa.dsa_sparse_attn(q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(idx).cuda(), sm_of(d))
    ref, ref_lse = oracle.sparse_attn(q, K, V, idx, np.arange(T), sm_of(d))
    assert_attn_close(out.float().cpu().numpy(), ref, lse.cpu().numpy(), ref_lse, "max jump")
    assert np.max(ref_lse) > 20.0      # the jump did happen for some (row, head)


@pytest.mark.parametrize("k", [16, 700, 2048])
def test_topk_long_rows_sampled_threshold(k):
    """Rows longer than the on-chip buffer take the sampled-threshold pass;
    the result is still bit-exact (quantised scores: many ties)."""
    T = 50000
    rng = np.random.default_rng(k + 5)
    sc = (np.round(rng.standard_normal((6, T)) * 256) / 256).astype(np.float32)
    sc[1, 40000:] += 3.0                      # the best keys all at the end
    sc[2, :100] += 3.0                        # ... or all at the start
    _topk_check(sc, k, row_begin=T - 6)


def test_decode_cuda_graph_replay_matches_eager():
    """The decode step captured in a CUDA graph (the kernels after the indexer
    are launched so that each may start while the one before it finishes)
    replays to exactly the eager step's outputs, replay after replay."""
    spec = small_decode_spec((40000, 20000, 9000, 3000), k=512, H_q=128, seed=5)
    inp = dsa_synth.make_decode(spec)
    dev = to_dev(inp)
    maxc, sm = 40000, sm_of(128)
    lib = dsa.load()
    ws = dsa.workspace(lib.dsa_decode_workspace_size(len(spec.context_lens), maxc, 128, 128, spec.k), "cuda")
    out0, lse0, idx0 = dsa.dsa_decode(dev, spec.k, maxc, sm, ws=ws)
    assert dsa.dsa_stream_status(ws) == 0
    out, lse, idx = torch.empty_like(out0), torch.empty_like(lse0), torch.empty_like(idx0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        dsa.dsa_decode(dev, spec.k, maxc, sm, out=out, lse=lse, idx_out=idx, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dsa.dsa_decode(dev, spec.k, maxc, sm, out=out, lse=lse, idx_out=idx, ws=ws)
    for _ in range(3):
        out.zero_()
        lse.zero_()
        idx.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(idx, idx0)
        assert torch.equal(out, out0)
        assert torch.equal(lse, lse0)
    assert dsa.dsa_stream_status(ws) == 0
    del g
