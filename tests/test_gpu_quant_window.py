"""Parity of the FP8 quantiser, the paged cache append and the sliding-window
selection (CUDA path through the C ABI) with the fp64/fp32 CPU oracle.

Bars: codes, scales, cache bytes and selections bit-exact (integer and byte
results; the quantiser's fp32 decisions are taken in fp32 on both sides);
attention within 2e-2 + 1e-2 |o| (gpu_common); end-to-end selection overlap
with the oracle's own selection >= 0.999."""
import numpy as np
import pytest
import torch

import dsa_synth
from oracle import oracle
from long_context_fp8_b200 import dsa

from gpu_common import OVERLAP_MIN, assert_attn_close, overlap, sm_of, to_dev

pytestmark = pytest.mark.gpu


def _rows_with_edge_cases(rows, cols, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((rows, cols), generator=g)
    x *= torch.pow(10.0, torch.empty((rows, 1)).uniform_(-6, 6, generator=g))
    if rows >= 6:
        x[0] = 0.0                                   # amax 0: scale 1, codes 0
        x[1] = 0.0
        x[1, cols // 2] = -3.0                       # one non-zero value
        x[2] = -0.0                                  # negative zeros keep their sign bit
        x[3] *= 1e-30                                # tiny magnitudes
        x[4] = x[4].sign() * 448.0                   # already on the largest code
        x[5, ::2] = 0.0
    return x.to(dtype)


@pytest.mark.parametrize("rows,cols,dtype", [(300, 8192, torch.bfloat16), (777, 128, torch.bfloat16),
                                             (513, 128, torch.float32), (9, 16384, torch.bfloat16),
                                             (101, 264, torch.float32), (7, 8, torch.bfloat16),
                                             (1, 2048, torch.float32), (65, 2056, torch.bfloat16)])
def test_quantize_bit_exact(rows, cols, dtype):
    x = _rows_with_edge_cases(rows, cols, rows * 7 + cols, dtype)
    codes, scale = dsa.dsa_quantize_e4m3(x.cuda())
    ref_codes, ref_scale = oracle.quantize_e4m3(x)
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_scale)
    got = codes.cpu().numpy()
    bad = np.argwhere(got != ref_codes)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"


def test_quantize_values_beside_every_rounding_midpoint():
    """Rows whose quotients x / scale land on, and a few ulps beside, every
    midpoint between neighbouring E4M3 values (where the rounding of the fp32
    quotient decides the code), with scales whose reciprocals are inexact."""
    codes_pos = np.array([oracle.e4m3(c) for c in range(0x7F)])
    mids = (codes_pos[1:] + codes_pos[:-1]) / 2
    rows = []
    for amax in (3.0, 7.0, 0.1, 1e-20, 5e4):
        s = np.float32(amax) / np.float32(448.0)
        base = (mids * np.float64(s)).astype(np.float32)
        vals = [np.float32(amax)]
        for k in range(-6, 7):
            v = base.copy()
            for _ in range(abs(k)):
                v = np.nextafter(v, np.float32(np.inf if k > 0 else 0)).astype(np.float32)
            vals.append(v)
            vals.append(-v)
        row = np.concatenate([np.atleast_1d(np.asarray(a, np.float32)) for a in vals])
        row = row[np.abs(row) <= np.float32(amax)]
        rows.append(row[: (row.size // 8) * 8])
    width = max(r.size for r in rows)
    x = np.zeros((len(rows), width), np.float32)
    for i, r in enumerate(rows):
        x[i, : r.size] = r
    codes, scale = dsa.dsa_quantize_e4m3(torch.from_numpy(x).cuda())
    ref_codes, ref_scale = oracle.quantize_e4m3(x)
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_scale)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)


def test_quantize_matches_the_input_generator():
    """The generator packs its sources with torch (amax / 448, float8 cast);
    the kernel reproduces those bytes from the same sources."""
    g = torch.Generator().manual_seed(3)
    src = torch.randn((2000, 64, 128), generator=g)
    ref_codes, ref_scale = dsa_synth.quantize_e4m3_per_token(src)
    codes, scale = dsa.dsa_quantize_e4m3(src.cuda())
    assert torch.equal(scale.cpu(), ref_scale)
    assert torch.equal(codes.cpu(), ref_codes)


def test_quantize_fullsize_query_128k_sampled():
    """The 128K prefill's index query [131072, 64 * 128] in bf16, quantised
    whole on the GPU; sampled rows checked against the oracle, every row's
    scale and largest code checked by their closed forms."""
    T, H, D = 131072, 64, 128
    g = torch.Generator(device="cuda").manual_seed(2)
    x = torch.randn((T, H, D), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    codes, scale = dsa.dsa_quantize_e4m3(x)
    torch.cuda.synchronize()
    # fp32 amax / 448 computed on the host (a true division per element)
    amax = x.float().abs().amax(dim=(1, 2)).cpu()
    assert torch.equal(scale.cpu(), amax / 448.0)
    mag = (codes.view(T, -1) & 0x7F).amax(dim=1)
    assert bool((mag == 0x7E).all())
    rows = torch.tensor([0, 1, 4095, 65536, 99999, T - 1])
    ref_codes, ref_scale = oracle.quantize_e4m3(x[rows.cuda()].cpu())
    np.testing.assert_array_equal(codes[rows.cuda()].cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(scale[rows.cuda()].cpu().numpy(), ref_scale)


def _append_case(seed=41):
    spec = dsa_synth.DecodeSpec("app", context_lens=(1000, 64, 1, 2049, 777), H_I=64, d_I=128, k=128,
                                H_q=16, d=128, page_size=64, needle_frac=0.01, needle_min_age=0,
                                seed=seed)
    inp = dsa_synth.make_decode(spec)
    g = torch.Generator().manual_seed(seed)
    B = spec.B
    # one new token per sequence at its last position, plus a run of 70 tokens
    # written into sequence 3 (a prefill-like append crossing a page boundary)
    seq = list(range(B)) + [3] * 70
    pos = [n - 1 for n in spec.context_lens] + list(range(1900, 1970))
    N = len(seq)
    kin = (torch.randn((N, spec.d_I), generator=g) * 3).to(torch.bfloat16)
    kn = torch.randn((N, spec.d), generator=g).to(torch.bfloat16)
    vn = torch.randn((N, spec.d), generator=g).to(torch.bfloat16)
    return spec, inp, torch.tensor(seq, dtype=torch.int32), torch.tensor(pos, dtype=torch.int32), kin, kn, vn


def _np_caches(inp):
    return {k: np.ascontiguousarray(oracle._np(inp[k])) for k in ("kidx_cache", "kscale_cache", "k_cache",
                                                               "v_cache")}


def test_cache_append_bit_exact():
    spec, inp, seq, pos, kin, kn, vn = _append_case()
    ref = _np_caches(inp)
    assert oracle.cache_append(ref, kin, kn, vn, seq, pos, inp["block_table"]) == 0
    dev = to_dev(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dsa.dsa_cache_append(dev, kin.cuda(), kn.cuda(), vn.cuda(), seq.cuda(), pos.cuda(), dev["block_table"],
                         status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for name, want in ref.items():
        got = oracle._np(dev[name])
        assert np.array_equal(got, want), name


def test_cache_append_out_of_range_reported_not_faulted():
    spec, inp, seq, pos, kin, kn, vn = _append_case(seed=43)
    seq, pos = seq[:5].clone(), pos[:5].clone()
    kin, kn, vn = kin[:5], kn[:5], vn[:5]
    dev = to_dev(inp)
    dev["block_table"][2, 0] = 10 ** 6              # sequence 2's only page: out of range
    pos[4] = 10 ** 7                                  # sequence 4: position past its block table
    ref = _np_caches(inp)
    for i in (0, 1, 3):                               # the in-range tokens, one by one
        assert oracle.cache_append(ref, kin[i:i + 1], kn[i:i + 1], vn[i:i + 1], seq[i:i + 1], pos[i:i + 1],
                                   inp["block_table"]) == 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dsa.dsa_cache_append(dev, kin.cuda(), kn.cuda(), vn.cuda(), seq.cuda(), pos.cuda(), dev["block_table"],
                         status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1                    # DSA_ERR_INVALID_ARG
    for name, want in ref.items():
        assert np.array_equal(oracle._np(dev[name]), want), name


def test_decode_step_from_bf16_sources():
    """A whole decode step from the model's bf16 outputs: quantise the index
    query, append the new token's index key, K and V, then decode -- against
    the oracle's quantiser, append and decode on the same sources."""
    spec, inp, seq, pos, kin, kn, vn = _append_case(seed=47)
    B = spec.B
    seq, pos, kin, kn, vn = seq[:B], pos[:B], kin[:B], kn[:B], vn[:B]
    g = torch.Generator().manual_seed(5)
    q_src = torch.randn((B, spec.H_I, spec.d_I), generator=g).to(torch.bfloat16)
    # oracle side
    ref_inp = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    caches = _np_caches(ref_inp)
    assert oracle.cache_append(caches, kin, kn, vn, seq, pos, inp["block_table"]) == 0
    qc, qs = oracle.quantize_e4m3(q_src)
    ref_inp.update(kidx_cache=torch.from_numpy(caches["kidx_cache"]),
                   kscale_cache=torch.from_numpy(caches["kscale_cache"]),
                   k_cache=torch.from_numpy(caches["k_cache"].view(np.int16)).view(torch.bfloat16),
                   v_cache=torch.from_numpy(caches["v_cache"].view(np.int16)).view(torch.bfloat16),
                   q_idx=torch.from_numpy(qc), q_scale=torch.from_numpy(qs))
    ref = oracle.decode(ref_inp, spec.k, sm_of(spec.d))
    # GPU side
    dev = to_dev(inp)
    codes, scale = dsa.dsa_quantize_e4m3(q_src.cuda())
    dev["q_idx"], dev["q_scale"] = codes, scale
    dsa.dsa_cache_append(dev, kin.cuda(), kn.cuda(), vn.cuda(), seq.cuda(), pos.cuda(), dev["block_table"])
    out, lse, idx = dsa.dsa_decode(dev, spec.k, max(spec.context_lens), sm_of(spec.d))
    idx = idx.cpu().numpy()
    mean_ov, min_ov = overlap(idx, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    assert_attn_close(out.float().cpu().numpy(), ref["out"], lse.cpu().numpy(), ref["lse"], "decode step")


# ------------------------------------------------------------------ sliding window + top-k

@pytest.mark.parametrize("k,W", [(64, 0), (64, 16), (300, 1000), (2048, 512), (5, 4000), (1, 1)])
def test_topk_window_bit_exact(k, W):
    rng = np.random.default_rng(k + W)
    T = 3000
    sc = (np.round(rng.standard_normal((64, T)) * 64) / 64).astype(np.float32)   # many ties
    for r0 in (0, 1500, T - 64):
        rows = np.arange(r0, r0 + 64)
        got = dsa.dsa_topk_window(torch.from_numpy(sc).cuda(), k, W, row_begin=r0).cpu().numpy()
        ref = oracle.topk_window(sc.astype(np.float64), rows, k, W)
        np.testing.assert_array_equal(got, ref, err_msg=f"k={k} W={W} r0={r0}")


def test_topk_window_long_rows():
    """Rows long enough for the sampled-threshold path, with a window."""
    rng = np.random.default_rng(9)
    T, k, W = 40000, 700, 4096
    sc = rng.standard_normal((8, T)).astype(np.float32)
    r0 = T - 8
    got = dsa.dsa_topk_window(torch.from_numpy(sc).cuda(), k, W, row_begin=r0).cpu().numpy()
    ref = oracle.topk_window(sc.astype(np.float64), np.arange(r0, T), k, W)
    np.testing.assert_array_equal(got, ref)


def _check_window_selection(idx, rows, k, W):
    for r, t in enumerate(rows):
        n = t + 1
        older = max(0, n - W)
        sel = idx[r][idx[r] >= 0]
        assert sel.size == min(k, older) + min(W, n), (r, sel.size)
        assert np.all(np.diff(sel) > 0) and sel.max() <= t
        assert set(range(older, n)) <= set(sel.tolist())
        assert np.all(idx[r][sel.size:] == -1)


def test_prefill_window_end_to_end():
    L, k, W = 1500, 128, 256
    spec = dsa_synth.PrefillSpec("pw", L=L, H_I=64, d_I=128, k=k, H_q=128, d=128, fp8=True,
                                 n_needles=15, seed=51)
    inp = dsa_synth.make_prefill(spec)
    dev = to_dev(inp)
    out, lse, idx = dsa.dsa_prefill_window(dev, k, W, sm_of(128))
    idx = idx.cpu().numpy()
    rows = np.arange(0, L, 7)
    rows[-1] = L - 1
    _check_window_selection(idx[rows], rows, k, W)
    ref = oracle.prefill(inp, k, sm_of(128), rows, window=W)
    mean_ov, min_ov = overlap(idx[rows], ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    ro, rl = oracle.sparse_attn(inp["q"], inp["k"], inp["v"], idx[rows], rows, sm_of(128))
    assert_attn_close(out.float().cpu().numpy()[rows], ro, lse.cpu().numpy()[rows], rl, "prefill window")


@pytest.mark.parametrize("lens,k,W", [((1000, 64, 1, 2049, 777), 128, 300), ((40000, 20000, 9000), 512, 4096)])
def test_decode_window_end_to_end(lens, k, W):
    spec = dsa_synth.DecodeSpec("dw", context_lens=tuple(lens), H_I=64, d_I=128, k=k, H_q=16, d=128,
                                page_size=64, needle_frac=0.01, needle_min_age=0, seed=len(lens) + W)
    inp = dsa_synth.make_decode(spec)
    dev = to_dev(inp)
    out, lse, idx = dsa.dsa_decode_window(dev, k, W, max(lens), sm_of(128))
    idx = idx.cpu().numpy()
    _check_window_selection(idx, [n - 1 for n in lens], k, W)
    ref = oracle.decode(inp, k, sm_of(128), window=W)
    mean_ov, min_ov = overlap(idx, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    # attention given the GPU's selection
    bt = inp["block_table"].numpy()
    ps = spec.page_size
    kc = inp["k_cache"].reshape(-1, 128)
    vc = inp["v_cache"].reshape(-1, 128)
    for b in range(spec.B):
        sel = idx[b][idx[b] >= 0]
        slot = torch.from_numpy(bt[b, sel // ps].astype(np.int64) * ps + sel % ps)
        ro, rl = oracle.sparse_attn(inp["q"][b:b + 1], kc[slot], vc[slot],
                                    np.arange(sel.size, dtype=np.int32)[None], [0], sm_of(128))
        assert_attn_close(out[b:b + 1].float().cpu().numpy(), ro, lse[b:b + 1].cpu().numpy(), rl, f"seq {b}")


def test_decode_window_zero_is_decode():
    spec = dsa_synth.DecodeSpec("dw0", context_lens=(3000, 50, 7000), H_I=64, d_I=128, k=256, H_q=128,
                                d=128, page_size=64, needle_frac=0.01, needle_min_age=0, seed=61)
    dev = to_dev(dsa_synth.make_decode(spec))
    a = dsa.dsa_decode(dev, spec.k, 7000, sm_of(128))
    b = dsa.dsa_decode_window(dev, spec.k, 0, 7000, sm_of(128))
    for x, y in zip(a, b):
        assert torch.equal(x, y)
