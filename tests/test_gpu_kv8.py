"""Parity of the decode over FP8 K/V caches (E4M3 codes, one fp32 scale per
cached token; dsa_decode_kv8 and dsa_cache_append_kv8 through the C ABI) with
the fp64 CPU oracle.

Bars: selection overlap with the oracle's own selection >= 0.999; attention
over the GPU's selection within 2e-2 + 1e-2 |o| of the fp64 attention over the
dequantised rows; cache bytes bit-exact; with power-of-two scales (every
dequantised value exact in bf16) the FP8 kernel's outputs equal the bf16
kernel's bit for bit."""
import numpy as np
import pytest
import torch

import dsa_synth
from oracle import brute, oracle
from long_context_fp8_b200 import dsa

from gpu_common import OVERLAP_MIN, assert_attn_close, overlap, sm_of, to_dev

pytestmark = pytest.mark.gpu


def _spec(lens, k, H_q=128, seed=71, ps=64):
    return dsa_synth.DecodeSpec("kv8", context_lens=tuple(lens), H_I=64, d_I=128, k=k, H_q=H_q, d=128,
                                page_size=ps, needle_frac=0.01, needle_min_age=0, seed=seed)


def _attention_over(inp8, idx, sm):
    """fp64 attention of each sequence's query over the listed positions of the
    FP8 caches, rows dequantised as e4m3(code) * scale."""
    bt = inp8["block_table"].numpy()
    ps = inp8["kidx_cache"].shape[1]
    d = inp8["q"].shape[-1]
    k8, v8 = inp8["k_cache"].reshape(-1, d), inp8["v_cache"].reshape(-1, d)
    ks, vs = inp8["k_cache_scale"].reshape(-1), inp8["v_cache_scale"].reshape(-1)
    outs, lses = [], []
    for b in range(idx.shape[0]):
        sel = idx[b][idx[b] >= 0]
        slot = torch.from_numpy(bt[b, sel // ps].astype(np.int64) * ps + sel % ps)
        K = brute.decode_storage(k8[slot]) * ks[slot].double().numpy()[:, None]
        V = brute.decode_storage(v8[slot]) * vs[slot].double().numpy()[:, None]
        o, l = brute.dense_masked_attention(inp8["q"][b:b + 1], K, V, np.ones((1, sel.size), bool), sm)
        outs.append(o[0]); lses.append(l[0])
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("lens,k,W", [((1000, 64, 1, 2049, 777), 128, 0), ((5000, 3000), 512, 0),
                                      ((40000, 20000, 9000), 512, 0), ((3000, 700, 9000), 256, 1024)])
def test_decode_kv8_end_to_end(lens, k, W):
    inp8 = dsa_synth.decode_kv_to_fp8(dsa_synth.make_decode(_spec(lens, k, seed=len(lens) + k + W)))
    dev = to_dev(inp8)
    out, lse, idx = dsa.dsa_decode_kv8(dev, k, max(lens), window=W, sm_scale=sm_of(128))
    idx = idx.cpu().numpy()
    ref = oracle.decode(inp8, k, sm_of(128), window=W)
    mean_ov, min_ov = overlap(idx, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    ro, rl = _attention_over(inp8, idx, sm_of(128))
    assert_attn_close(out.float().cpu().numpy(), ro, lse.cpu().numpy(), rl, "decode kv8")
    # where the selections agree, the oracle's own attention agrees too
    same = [b for b in range(len(lens)) if np.array_equal(idx[b], ref["idx"][b])]
    assert same
    assert_attn_close(out.float().cpu().numpy()[same], ref["out"][same], lse.cpu().numpy()[same],
                      ref["lse"][same], "decode kv8 vs oracle")


def test_decode_kv8_power_of_two_scales_equal_bf16_kernel():
    """Codes times power-of-two scales are exact in bf16, so the widened tiles
    equal the bf16 kernel's gathered tiles and the outputs match bit for bit."""
    spec = _spec((3000, 129, 6000), 256, seed=73)
    inp = dsa_synth.make_decode(spec)
    rng = np.random.default_rng(5)
    P, ps = inp["kidx_cache"].shape[:2]
    inp8, bf = dict(inp), dict(inp)
    for name in ("k", "v"):
        codes = torch.from_numpy(rng.integers(0, 0xFF, (P, ps, 128)).astype(np.uint8))
        codes[(codes & 0x7F) == 0x7F] = 0                          # no NaN codes
        scale = torch.from_numpy((2.0 ** rng.integers(-8, 4, (P, ps))).astype(np.float32))
        inp8[name + "_cache"], inp8[name + "_cache_scale"] = codes, scale
        vals = codes.view(torch.float8_e4m3fn).float() * scale[..., None]
        bf[name + "_cache"] = vals.to(torch.bfloat16)
        assert torch.equal(bf[name + "_cache"].float(), vals)
    a = dsa.dsa_decode_kv8(to_dev(inp8), spec.k, 6000, sm_scale=sm_of(128))
    b = dsa.dsa_decode(to_dev(bf), spec.k, 6000, sm_of(128))
    for x, y, what in zip(a, b, ("out", "lse", "idx")):
        assert torch.equal(x, y), what


def test_cache_append_kv8_bit_exact():
    spec = _spec((1000, 64, 1, 2049, 777), 128, seed=75)
    inp8 = dsa_synth.decode_kv_to_fp8(dsa_synth.make_decode(spec))
    g = torch.Generator().manual_seed(7)
    seq = torch.tensor(list(range(spec.B)) + [3] * 70, dtype=torch.int32)
    pos = torch.tensor([n - 1 for n in spec.context_lens] + list(range(1900, 1970)), dtype=torch.int32)
    N = seq.numel()
    kin = (torch.randn((N, 128), generator=g) * 3).to(torch.bfloat16)
    kn = (torch.randn((N, 128), generator=g) * 20).to(torch.bfloat16)
    vn = (torch.randn((N, 128), generator=g) / 20).to(torch.bfloat16)
    names = ("kidx_cache", "kscale_cache", "k_cache", "v_cache", "k_cache_scale", "v_cache_scale")
    ref = {n: np.ascontiguousarray(oracle._np(inp8[n])) for n in names}
    assert oracle.cache_append(ref, kin, kn, vn, seq, pos, inp8["block_table"]) == 0
    dev = to_dev(inp8)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dsa.dsa_cache_append_kv8(dev, kin.cuda(), kn.cuda(), vn.cuda(), seq.cuda(), pos.cuda(), dev["block_table"],
                             status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for n in names:
        assert np.array_equal(oracle._np(dev[n]), ref[n]), n


def test_decode_kv8_rejects_unsupported_heads():
    inp8 = dsa_synth.decode_kv_to_fp8(dsa_synth.make_decode(_spec((300, 200), 64, H_q=16, seed=77)))
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_decode_kv8(to_dev(inp8), 64, 300)
    assert e.value.status == 2                                    # DSA_ERR_UNSUPPORTED
