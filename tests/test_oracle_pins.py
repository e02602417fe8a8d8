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


# ---------------------------------------------------------------- FP8 quantisation (stage 6)

def _finite_codes():
    return [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_e4m3_encode_round_trips_every_code():
    """Every finite code's own value encodes back to that code (-0 to 0x80)."""
    for c in _finite_codes():
        v = oracle.e4m3(c)
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_e4m3_encode_golden_points():
    g = _golden("e4m3_rounding_points.json")
    for val, code, why in g["encode"]:
        assert oracle.e4m3_encode(val) == int(code, 16), why


def test_e4m3_encode_matches_torch_conversion():
    """The library's float -> float8_e4m3fn conversion (round to nearest even) on
    values inside the finite range: random magnitudes over every binade, the
    exact midpoints between neighbouring codes, and values just beside them."""
    rng = np.random.default_rng(8)
    vals = [rng.standard_normal(20000).astype(np.float32) * np.float32(2.0) ** rng.integers(-14, 9, 20000)]
    pos = np.array([oracle.e4m3(c) for c in range(0x7F)])
    mid = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    vals += [mid, -mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))]
    x = np.concatenate(vals).astype(np.float32)
    x = np.clip(x, -448.0, 448.0).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(x[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_quantize_golden_rows():
    g = _golden("e4m3_rounding_points.json")["quantize"]
    for ex in g:
        x = np.array([ex["x"]], np.float32)
        codes, scale = oracle.quantize_e4m3(x)
        want = np.float32(3.0) / np.float32(448.0) if "scale_expr" in ex else np.float32(ex["scale"])
        assert scale[0] == want, ex["why"]
        assert [hex(c) for c in codes[0]] == [hex(int(c, 16)) for c in ex["codes"]], ex["why"]


def test_quantize_matches_torch_per_token():
    """amax/448 in fp32 and torch's float8 conversion of x / scale, bf16 and fp32 rows."""
    rng = np.random.default_rng(12)
    x32 = (rng.standard_normal((64, 300)) * 10.0 ** rng.uniform(-6, 6, (64, 1))).astype(np.float32)
    for x in (torch.from_numpy(x32), torch.from_numpy(x32).to(torch.bfloat16)):
        codes, scale = oracle.quantize_e4m3(x)
        xf = x.float()
        amax = xf.abs().amax(dim=1)
        ref_scale = amax / 448.0
        ref = (xf / ref_scale[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
        np.testing.assert_array_equal(scale, ref_scale.numpy())
        np.testing.assert_array_equal(codes, ref.numpy())


def test_quantize_invariants():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((32, 128)).astype(np.float32) * rng.uniform(0.01, 100, (32, 1)).astype(np.float32)
    codes, scale = oracle.quantize_e4m3(x)
    am = np.argmax(np.abs(x), axis=1)
    # the row's largest magnitude maps to the largest finite code, with its sign
    for r in range(32):
        assert codes[r, am[r]] & 0x7F == 0x7E
        assert (codes[r, am[r]] >> 7) == (x[r, am[r]] < 0)
    # dequantised error: at most half a step (2^-4 relative in the normal range,
    # 2^-10 * scale below the smallest normal 2^-6 * scale)
    deq = np.vectorize(oracle.e4m3)(codes) * scale[:, None].astype(np.float64)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scale[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound)
    # rows quantise independently; scaling a row by a power of two scales only its scale
    x2 = x.copy(); x2[5] *= 8.0
    c2, s2 = oracle.quantize_e4m3(x2)
    np.testing.assert_array_equal(c2, codes)
    assert s2[5] == scale[5] * 8 and np.array_equal(np.delete(s2, 5), np.delete(scale, 5))


def test_quantize_degenerate_rows():
    x = np.zeros((3, 16), np.float32)
    x[1, 3] = 1e-44                                   # amax/448 underflows to 0: scale 1
    x[2, :] = -0.0
    codes, scale = oracle.quantize_e4m3(x)
    assert scale.tolist() == [1.0, 1.0, 1.0]
    assert np.all(codes[0] == 0) and np.all(codes[1] == 0) and np.all(codes[2] == 0x80)


def _paged_caches(rng, P, ps, D_I, D):
    return dict(kidx_cache=rng.integers(0, 0x7E, (P, ps, D_I)).astype(np.uint8),
                kscale_cache=rng.uniform(0.5, 2, (P, ps)).astype(np.float32),
                k_cache=rng.integers(0, 1 << 15, (P, ps, D)).astype(np.uint16),
                v_cache=rng.integers(0, 1 << 15, (P, ps, D)).astype(np.uint16))


def test_cache_append_writes_exactly_the_addressed_slots():
    rng = np.random.default_rng(14)
    B, P, ps, D_I, D, maxp = 5, 40, 16, 32, 24, 6
    bt = np.stack([rng.permutation(P)[:maxp] for _ in range(B)]).astype(np.int32)
    caches = _paged_caches(rng, P, ps, D_I, D)
    before = {k: v.copy() for k, v in caches.items()}
    N = 9
    seq = np.array([0, 1, 2, 3, 4, 0, 0, 3, 2], np.int32)
    pos = np.array([0, 15, 16, 95, 40, 1, 2, 17, 33], np.int32)
    kin = torch.from_numpy(rng.standard_normal((N, D_I)).astype(np.float32)).to(torch.bfloat16)
    kn = rng.integers(0, 1 << 15, (N, D)).astype(np.uint16)
    vn = rng.integers(0, 1 << 15, (N, D)).astype(np.uint16)
    assert oracle.cache_append(caches, kin, kn, vn, seq, pos, bt) == 0
    codes, scale = oracle.quantize_e4m3(kin)
    touched = np.zeros((P, ps), bool)
    for i in range(N):
        page, slot = bt[seq[i], pos[i] // ps], pos[i] % ps
        touched[page, slot] = True
        np.testing.assert_array_equal(caches["kidx_cache"][page, slot], codes[i])
        assert caches["kscale_cache"][page, slot] == scale[i]
        np.testing.assert_array_equal(caches["k_cache"][page, slot], kn[i])
        np.testing.assert_array_equal(caches["v_cache"][page, slot], vn[i])
    for name in caches:
        np.testing.assert_array_equal(caches[name][~touched], before[name][~touched])


def test_cache_append_rejects_out_of_range():
    rng = np.random.default_rng(15)
    B, P, ps, maxp = 2, 8, 16, 2
    bt = np.array([[0, 1], [2, 99]], np.int32)                    # page 99 does not exist
    caches = _paged_caches(rng, P, ps, 16, 8)
    kin = np.ones((1, 16), np.float32)
    kv = np.zeros((1, 8), np.uint16)
    for seq, pos in ((0, 32), (0, -1), (1, 20), (2, 0)):
        assert oracle.cache_append(caches, kin, kv, kv, [seq], [pos], bt) == -2, (seq, pos)
    assert oracle.cache_append(caches, kin, kv, kv, [1], [3], bt) == 0


# ---------------------------------------------------------------- sliding window + top-k (stage 5)

def _brute_window_rows(scores, rows, k, W):
    out = np.full((len(rows), k + W), -1, np.int32)
    for r, t in enumerate(rows):
        n = t + 1
        older = max(0, n - W)
        order = sorted(range(older), key=lambda s: (-scores[r, s], s))
        sel = sorted(order[: min(k, older)]) + list(range(older, n))
        out[r, : len(sel)] = sel
    return out


def test_topk_window_vs_sort():
    rng = np.random.default_rng(16)
    T = 260
    scores = np.round(rng.standard_normal((50, T)) * 4) / 4
    rows = rng.integers(0, T, 50)
    rows[:4] = [0, T - 1, 9, 10]
    for k, W in ((1, 1), (8, 10), (16, 3), (64, 100), (300, 5), (5, 400)):
        got = oracle.topk_window(scores, rows, k, W)
        np.testing.assert_array_equal(got, _brute_window_rows(scores, rows, k, W), err_msg=f"k={k} W={W}")


def test_topk_window_special_cases():
    rng = np.random.default_rng(17)
    T, k = 200, 12
    scores = rng.standard_normal((30, T))
    rows = rng.integers(0, T, 30)
    # W = 0 is the plain selector
    np.testing.assert_array_equal(oracle.topk_window(scores, rows, k, 0), oracle.topk(scores, rows, k))
    # the window positions are taken whatever their scores
    low = scores.copy(); low[:, :] = 5.0
    for r, t in enumerate(rows):
        low[r, max(0, t - 7): t + 1] = -1e300
    got = oracle.topk_window(low, rows, k, 8)
    for r, t in enumerate(rows):
        n = t + 1
        sel = got[r][got[r] >= 0]
        assert sel.size == min(k, max(0, n - 8)) + min(8, n)
        assert set(range(max(0, n - 8), n)) <= set(sel.tolist())
        assert np.all(np.diff(sel) > 0) and np.all(got[r][sel.size:] == -1)
    # k + W >= t + 1: every causal position
    got = oracle.topk_window(scores, [50], 20, 31)
    assert got[0].tolist() == list(range(51))


def test_decode_window_matches_dense_mask():
    """Decode with a window: dense masked attention over window U top-k(older)."""
    spec = dsa_synth.DecodeSpec("dw", context_lens=(130, 9, 1, 257), H_I=4, d_I=32, k=12,
                                H_q=3, d=16, page_size=16, needle_frac=0.05,
                                needle_min_age=4, seed=19)
    inp = dsa_synth.make_decode(spec)
    sm, W = 0.25, 20
    res = oracle.decode(inp, spec.k, sm, want_scores=True, window=W)
    bt = inp["block_table"].numpy()
    for b, n in enumerate(spec.context_lens):
        pos = np.arange(n)
        slot = bt[b, pos // 16].astype(np.int64) * 16 + pos % 16
        sc = res["scores"][b, :n]
        older = max(0, n - W)
        order = np.argsort(-sc[:older], kind="stable")[: min(spec.k, older)]
        mask = np.zeros(n, bool); mask[order] = True; mask[older:] = True
        sel = np.nonzero(mask)[0]
        assert res["idx"][b][: sel.size].tolist() == sel.tolist()
        assert np.all(res["idx"][b][sel.size:] == -1)
        kc = inp["k_cache"].reshape(-1, 16)[slot]
        vc = inp["v_cache"].reshape(-1, 16)[slot]
        qq = torch.zeros((n, 3, 16), dtype=torch.bfloat16); qq[n - 1] = inp["q"][b]
        m = np.zeros((n, n), bool); m[n - 1] = mask
        m[: n - 1, 0] = True
        out, lse = brute.dense_masked_attention(qq, kc, vc, m, sm)
        np.testing.assert_allclose(res["out"][b], out[n - 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][b], lse[n - 1], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- FP8 K/V (stage 7)

def test_decode_fp8_kv_matches_dense_mask():
    """Decode over E4M3 K/V caches with per-token scales: dense masked attention
    over the dequantised rows (torch's float8 decode times the scale)."""
    spec = dsa_synth.DecodeSpec("dk", context_lens=(130, 64, 1, 257), H_I=4, d_I=32, k=16,
                                H_q=3, d=16, page_size=16, needle_frac=0.05,
                                needle_min_age=4, seed=29)
    inp = dsa_synth.decode_kv_to_fp8(dsa_synth.make_decode(spec))
    sm = 0.25
    res = oracle.decode(inp, spec.k, sm)
    bt = inp["block_table"].numpy()
    for b, n in enumerate(spec.context_lens):
        pos = np.arange(n)
        slot = bt[b, pos // 16].astype(np.int64) * 16 + pos % 16
        kd = brute.decode_storage(inp["k_cache"].reshape(-1, 16)[slot]) * inp["k_cache_scale"].reshape(-1)[slot].double().numpy()[:, None]
        vd = brute.decode_storage(inp["v_cache"].reshape(-1, 16)[slot]) * inp["v_cache_scale"].reshape(-1)[slot].double().numpy()[:, None]
        sel = res["idx"][b][res["idx"][b] >= 0]
        mask = np.zeros((n, n), bool); mask[n - 1, sel] = True
        mask[: n - 1, 0] = True
        qq = torch.zeros((n, 3, 16), dtype=torch.bfloat16); qq[n - 1] = inp["q"][b]
        out, lse = brute.dense_masked_attention(qq, kd, vd, mask, sm)
        np.testing.assert_allclose(res["out"][b], out[n - 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][b], lse[n - 1], rtol=1e-12, atol=1e-12)


def test_decode_fp8_kv_power_of_two_scales_equal_bf16_path():
    """With power-of-two scales every dequantised value is exact in bf16, so the
    FP8 K/V decode equals the bf16 decode over those values (a dropped or
    misplaced scale fails this)."""
    spec = dsa_synth.DecodeSpec("dp", context_lens=(90, 33), H_I=4, d_I=32, k=8, H_q=2, d=16,
                                page_size=16, needle_frac=0.0, needle_min_age=0, seed=31)
    inp = dsa_synth.make_decode(spec)
    rng = np.random.default_rng(3)
    P, ps = inp["kidx_cache"].shape[:2]
    kv8 = dict(inp)
    bf = dict(inp)
    for name in ("k", "v"):
        codes = torch.from_numpy(rng.integers(0, 0x7F, (P, ps, 16)).astype(np.uint8))
        codes[codes == 0x7F] = 0
        codes |= torch.from_numpy((rng.integers(0, 2, (P, ps, 16)) << 7).astype(np.uint8))
        codes[(codes & 0x7F) == 0x7F] = 0
        scale = torch.from_numpy((2.0 ** rng.integers(-6, 6, (P, ps))).astype(np.float32))
        kv8[name + "_cache"], kv8[name + "_cache_scale"] = codes, scale
        vals = codes.view(torch.float8_e4m3fn).float() * scale[..., None]
        bf[name + "_cache"] = vals.to(torch.bfloat16)
        assert torch.equal(bf[name + "_cache"].float(), vals)        # exact in bf16
    a = oracle.decode(kv8, spec.k, 0.3)
    b = oracle.decode(bf, spec.k, 0.3)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(a["lse"], b["lse"], rtol=1e-15, atol=1e-15)


def test_cache_append_fp8_kv_quantises_k_and_v():
    rng = np.random.default_rng(33)
    B, P, ps, D_I, D, maxp = 3, 20, 16, 32, 24, 4
    bt = np.stack([rng.permutation(P)[:maxp] for _ in range(B)]).astype(np.int32)
    caches = dict(kidx_cache=rng.integers(0, 0x7E, (P, ps, D_I)).astype(np.uint8),
                  kscale_cache=np.ones((P, ps), np.float32),
                  k_cache=rng.integers(0, 0x7E, (P, ps, D)).astype(np.uint8),
                  v_cache=rng.integers(0, 0x7E, (P, ps, D)).astype(np.uint8),
                  k_cache_scale=np.ones((P, ps), np.float32), v_cache_scale=np.ones((P, ps), np.float32))
    before = {k: v.copy() for k, v in caches.items()}
    seq = np.array([0, 1, 2, 2], np.int32)
    pos = np.array([5, 63, 0, 17], np.int32)
    kin = torch.from_numpy(rng.standard_normal((4, D_I)).astype(np.float32)).to(torch.bfloat16)
    kn = torch.from_numpy(rng.standard_normal((4, D)).astype(np.float32) * 5).to(torch.bfloat16)
    vn = torch.from_numpy(rng.standard_normal((4, D)).astype(np.float32) / 5).to(torch.bfloat16)
    assert oracle.cache_append(caches, kin, kn, vn, seq, pos, bt) == 0
    kc, ksc = oracle.quantize_e4m3(kn)
    vc, vsc = oracle.quantize_e4m3(vn)
    touched = np.zeros((P, ps), bool)
    for i in range(4):
        page, slot = bt[seq[i], pos[i] // ps], pos[i] % ps
        touched[page, slot] = True
        np.testing.assert_array_equal(caches["k_cache"][page, slot], kc[i])
        np.testing.assert_array_equal(caches["v_cache"][page, slot], vc[i])
        assert caches["k_cache_scale"][page, slot] == ksc[i] and caches["v_cache_scale"][page, slot] == vsc[i]
    for name in caches:
        np.testing.assert_array_equal(caches[name][~touched], before[name][~touched])
