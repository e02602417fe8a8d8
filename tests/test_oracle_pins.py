"""Pins of the fp64 CPU oracle against things other than itself.

Each test ties one oracle function to the format definition, a hand-derived
worked example, a closed form, a library routine (numpy matmul, torch SDPA,
torch's float8/bf16 conversions), an invariant of the mathematics, or the
brute-force dense-mask restatement in ``oracle/brute.py``.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import dsa_synth
from oracle import brute, oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- formats

def test_e4m3_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(got)
        else:
            assert got == ref[c], hex(c)
            assert math.copysign(1.0, got) == math.copysign(1.0, ref[c])


def test_e4m3_spec_points():
    g = _golden("e4m3_spec_points.json")
    for code, val, _ in g["points"]:
        got = oracle.e4m3(int(code, 16))
        assert got == val and math.copysign(1, got) == math.copysign(1, val), code
    for code in g["nan_codes"]:
        assert math.isnan(oracle.e4m3(int(code, 16)))


def test_bf16_matches_torch():
    rng = np.random.default_rng(5)
    bits = np.concatenate([rng.integers(0, 1 << 16, 4000), [0, 0x8000, 0x3F80, 0x7F7F, 0x0001, 0xFF7F]])
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]          # drop inf/nan patterns
    t = torch.from_numpy(bits.astype(np.int32)).to(torch.int16).view(torch.bfloat16)
    ref = t.to(torch.float64).numpy()
    for b, r in zip(bits, ref):
        assert oracle.bf16(int(b)) == r


# ---------------------------------------------------------------- worked example

def test_worked_example_indexer_and_topk():
    g = _golden("worked_example.json")["indexer"]
    q = np.array(g["q_idx"], np.float32)
    k = np.array(g["k_idx"], np.float32)
    w = np.array(g["w"], np.float32)
    sc = oracle.index_scores(q, None, k, None, w, rows=[0, 1, 2])
    for t, row in enumerate(g["scores"]):
        for s, v in enumerate(row):
            if v is None:
                assert sc[t, s] == -np.inf
            else:
                assert sc[t, s] == v
    for kk, expect in g["topk"].items():
        got = oracle.topk(sc, [0, 1, 2], int(kk))
        assert got.tolist() == expect, kk


def test_worked_example_attention():
    g = _golden("worked_example.json")["attention"]
    out, lse = oracle.sparse_attn(np.array(g["q"], np.float32), np.array(g["K"], np.float32),
                                  np.array(g["V"], np.float32), np.array(g["idx"], np.int32),
                                  rows=[0], sm_scale=math.log(3.0))
    np.testing.assert_allclose(out, np.array(g["out"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- indexer

def _small_fp8(L=96, H=3, D=32, seed=7):
    spec = dsa_synth.PrefillSpec("t", L=L, H_I=H, d_I=D, k=8, H_q=2, d=16, fp8=True,
                                 n_needles=4, seed=seed)
    return dsa_synth.make_prefill(spec)


def test_index_single_head_is_relu_matmul():
    """H_I = 1 and w = 1: the score matrix is ReLU(Qhat Khat^T) (numpy matmul)."""
    inp = _small_fp8(L=80, H=1, D=64)
    w = torch.ones((80, 1), dtype=torch.bfloat16)
    qh = brute.decode_storage(inp["q_idx"])[:, 0, :] * inp["q_scale"].double().numpy()[:, None]
    kh = brute.decode_storage(inp["k_idx"]) * inp["k_scale"].double().numpy()[:, None]
    ref = np.maximum(qh @ kh.T, 0.0)
    got = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], w,
                              rows=np.arange(80))
    tril = np.tril(np.ones((80, 80), bool))
    np.testing.assert_allclose(got[tril], ref[tril], rtol=1e-12, atol=1e-12)
    assert np.all(np.isneginf(got[~tril]))


@pytest.mark.parametrize("fp8", [False, True])
def test_index_matches_brute(fp8):
    if fp8:
        inp = _small_fp8()
    else:
        spec = dsa_synth.prefill_spec("tiny", L=100)
        inp = dsa_synth.make_prefill(spec)
    T = inp["q_idx"].shape[0]
    got = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"],
                              rows=np.arange(T))
    ref = brute.dense_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"])
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got))
    np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-12, atol=1e-12)


def test_index_invariants():
    inp = _small_fp8(L=64)
    rows = np.arange(64)
    base = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"], rows)
    fin = np.isfinite(base)
    assert np.all(base[fin] >= 0.0)                     # w >= 0  =>  I >= 0
    # scaling one key's scale by 2 doubles exactly that column (positive homogeneity of ReLU)
    ks = inp["k_scale"].clone()
    ks[10] *= 2.0
    col = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], ks, inp["w"], rows)
    np.testing.assert_array_equal(col[:, 10][fin[:, 10]], 2.0 * base[:, 10][fin[:, 10]])
    other = np.ones(64, bool); other[10] = False
    np.testing.assert_array_equal(col[:, other], base[:, other])
    # doubling w doubles I; negating w negates I
    w2 = (inp["w"].float() * 2).to(torch.bfloat16)
    dbl = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], w2, rows)
    np.testing.assert_array_equal(dbl[fin], 2.0 * base[fin])
    neg = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], -inp["w"], rows)
    np.testing.assert_array_equal(neg[fin], -base[fin])
    # a query scale only rescales its own row
    qs = inp["q_scale"].clone(); qs[20] *= 4.0
    row = oracle.index_scores(inp["q_idx"], qs, inp["k_idx"], inp["k_scale"], inp["w"], rows)
    np.testing.assert_array_equal(row[20][fin[20]], 4.0 * base[20][fin[20]])


def test_index_row_subset_and_causality():
    inp = _small_fp8(L=50)
    full = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"], np.arange(50))
    sub = oracle.index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"], [49, 0, 17])
    np.testing.assert_array_equal(sub, full[[49, 0, 17]])
    for r, t in enumerate([49, 0, 17]):
        assert np.all(np.isfinite(sub[r, : t + 1])) and np.all(np.isneginf(sub[r, t + 1:]))


# ---------------------------------------------------------------- top-k

def _brute_topk_rows(scores, rows, k):
    out = np.full((len(rows), k), -1, np.int32)
    for r, t in enumerate(rows):
        order = sorted(range(t + 1), key=lambda s: (-scores[r, s], s))
        sel = sorted(order[: min(k, t + 1)])
        out[r, : len(sel)] = sel
    return out


def test_topk_vs_sort_with_ties():
    rng = np.random.default_rng(3)
    T = 300
    scores = np.round(rng.standard_normal((40, T)) * 4) / 4        # many exact ties
    scores[5] = 0.0
    scores[6, :] = -0.0
    scores[6, ::3] = 0.0                                             # +0 and -0 compare equal
    rows = rng.integers(0, T, 40)
    rows[:3] = [0, T - 1, 16]
    for k in (1, 7, 16, 64, 299, 400):
        got = oracle.topk(scores, rows, k)
        np.testing.assert_array_equal(got, _brute_topk_rows(scores, rows, k))


def test_topk_closed_forms():
    T, k = 200, 17
    eq = np.full((3, T), 1.25)
    got = oracle.topk(eq, [199, 50, 5], k)
    assert got[0].tolist() == list(range(k))                 # all equal -> lowest indices
    assert got[1].tolist() == list(range(k))
    assert got[2].tolist() == list(range(6)) + [-1] * (k - 6)  # k >= t+1 -> {0..t}
    inc = np.tile(np.arange(T, dtype=np.float64), (1, 1))
    got = oracle.topk(inc, [150], k)
    assert got[0].tolist() == list(range(151 - k, 151))      # monotone scores -> the last k


def test_topk_properties_random():
    rng = np.random.default_rng(11)
    T, k = 500, 32
    scores = rng.standard_normal((60, T))
    rows = rng.integers(0, T, 60)
    got = oracle.topk(scores, rows, k)
    for r, t in enumerate(rows):
        sel = got[r][got[r] >= 0]
        assert sel.size == min(k, t + 1)
        assert np.all(np.diff(sel) > 0) and sel.max() <= t
        assert np.all(got[r][sel.size:] == -1)
        # every selected score >= every unselected candidate score
        mask = np.zeros(t + 1, bool); mask[sel] = True
        if (~mask).any():
            assert scores[r, :t + 1][mask].min() >= scores[r, :t + 1][~mask].max()


# ---------------------------------------------------------------- attention

def test_attention_dense_when_k_covers_history():
    """k >= L: DSA reduces to dense causal attention (torch SDPA, fp64)."""
    rng = np.random.default_rng(2)
    T, H, D = 40, 3, 16
    q = rng.standard_normal((T, H, D)).astype(np.float32)
    K = rng.standard_normal((T, D)).astype(np.float32)
    V = rng.standard_normal((T, D)).astype(np.float32)
    idx = np.full((T, T), -1, np.int32)
    for t in range(T):
        idx[t, : t + 1] = np.arange(t + 1)
    out, _ = oracle.sparse_attn(q, K, V, idx, np.arange(T), 1 / math.sqrt(D))
    qt = torch.from_numpy(q).double().permute(1, 0, 2)[None]
    kt = torch.from_numpy(K).double()[None, None].expand(1, H, T, D)
    vt = torch.from_numpy(V).double()[None, None].expand(1, H, T, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_single_row_and_constant_value():
    rng = np.random.default_rng(4)
    T, H, D, k = 30, 2, 8, 5
    q = rng.standard_normal((T, H, D)).astype(np.float32)
    K = rng.standard_normal((T, D)).astype(np.float32)
    V = rng.standard_normal((T, D)).astype(np.float32)
    idx = np.full((T, k), -1, np.int32)
    idx[:, 0] = rng.integers(0, T, T)
    out, lse = oracle.sparse_attn(q, K, V, idx, np.arange(T), 0.3)
    np.testing.assert_array_equal(out, np.repeat(V[idx[:, 0]][:, None, :], H, 1).astype(np.float64))
    np.testing.assert_allclose(lse, 0.3 * np.einsum("thd,td->th", q.astype(np.float64), K[idx[:, 0]].astype(np.float64)), rtol=1e-12)
    # constant V: weights sum to one, so every output equals that constant
    idx2 = np.stack([rng.permutation(T)[:k] for _ in range(T)]).astype(np.int32)
    Vc = np.full((T, D), 0.75, np.float32)
    out2, _ = oracle.sparse_attn(q, K, Vc, idx2, np.arange(T), 1.0)
    np.testing.assert_allclose(out2, 0.75, rtol=1e-14)


@pytest.mark.parametrize("name", ["tiny", "fp8"])
def test_end_to_end_matches_dense_mask(name):
    if name == "tiny":
        inp = dsa_synth.make_prefill(dsa_synth.prefill_spec("tiny", L=160))
        k, D = 64, 64
    else:
        inp = _small_fp8(L=120)
        k, D = 8, 16
    T = inp["q"].shape[0]
    sm = 1 / math.sqrt(D)
    res = oracle.prefill(inp, k, sm, np.arange(T))
    scores = brute.dense_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"])
    mask = brute.dense_topk_mask(scores, k)
    np.testing.assert_array_equal(res["idx"], brute.mask_to_idx(mask, k))
    out, lse = brute.dense_masked_attention(inp["q"], inp["k"], inp["v"], mask, sm)
    np.testing.assert_allclose(res["out"], out, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["lse"], lse, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- decode

def test_decode_matches_unpaged_dense_mask():
    spec = dsa_synth.DecodeSpec("d", context_lens=(130, 64, 1, 257), H_I=4, d_I=32, k=16,
                                H_q=3, d=16, page_size=16, needle_frac=0.05,
                                needle_min_age=4, seed=9)
    inp = dsa_synth.make_decode(spec)
    sm = 0.25
    res = oracle.decode(inp, spec.k, sm, want_scores=True)
    bt = inp["block_table"].numpy()
    for b, n in enumerate(spec.context_lens):
        pos = np.arange(n)
        slot = bt[b, pos // 16].astype(np.int64) * 16 + pos % 16
        kk = inp["kidx_cache"].reshape(-1, 32)[slot]
        ks = inp["kscale_cache"].reshape(-1)[slot]
        # the query row is placed at position n-1 of a contiguous prefix
        qi = torch.zeros((n, 4, 32), dtype=torch.uint8); qi[n - 1] = inp["q_idx"][b]
        qs = torch.ones(n); qs[n - 1] = inp["q_scale"][b]
        ww = torch.zeros((n, 4), dtype=torch.bfloat16); ww[n - 1] = inp["w"][b]
        sc = brute.dense_scores(qi, qs, kk, ks, ww)[n - 1]
        np.testing.assert_allclose(res["scores"][b, :n], sc, rtol=1e-12, atol=1e-12)
        mask = brute.dense_topk_mask(sc[None, :].repeat(n, 0), spec.k)[n - 1]
        sel = np.nonzero(mask)[0]
        assert res["idx"][b][: sel.size].tolist() == sel.tolist()
        assert np.all(res["idx"][b][sel.size:] == -1)
        kc = inp["k_cache"].reshape(-1, 16)[slot]
        vc = inp["v_cache"].reshape(-1, 16)[slot]
        qq = torch.zeros((n, 3, 16), dtype=torch.bfloat16); qq[n - 1] = inp["q"][b]
        m = np.zeros((n, n), bool); m[n - 1] = mask
        m[: n - 1, 0] = True                            # keep other rows finite; unused
        out, lse = brute.dense_masked_attention(qq, kc, vc, m, sm)
        np.testing.assert_allclose(res["out"][b], out[n - 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][b], lse[n - 1], rtol=1e-12, atol=1e-12)


def test_needles_are_selected():
    """Sanity (not a parity criterion): planted needles rank high in their source row."""
    inp = _small_fp8(L=200, H=4, D=64, seed=21)
    src = inp["needle_src"].numpy()
    pos = inp["needle_pos"].numpy()
    res = oracle.prefill(inp, 16, 0.25, src)
    hits = [p in set(res["idx"][i].tolist()) for i, p in enumerate(pos)]
    assert np.mean(hits) >= 0.5
