"""The algorithmic work bench.py divides by (the numerators of every roofline
fraction it reports), recomputed here from the definitions: what the method
must read and write per decode step, and the FLOPs of the 128K prefill."""
import bench
import dsa_synth


def test_decode_step_bytes():
    s = dsa_synth.decode_spec("dec64x64k")
    B, n, k, d, H_q, H_I, d_I = 64, 65536, 2048, 128, 128, 64, 128
    keys = B * n * (d_I + 4)                     # FP8 index key + fp32 scale per cached token
    gather = B * k * 2 * d * 2                   # selected K and V rows, bf16
    q_out = 2 * B * H_q * d * 2                  # query in, output out, bf16
    q_idx = B * H_I * d_I + B * 4 + B * H_I * 2  # FP8 index query, its scale, bf16 head weights
    idx = B * k * 4
    want = keys + gather + q_out + q_idx + idx
    assert sum(bench.decode_hbm_bytes(s).values()) == want == 626_008_320
    # the 8K window: 8192 more gathered rows per sequence, wider index rows
    w = 8192
    want_w = want + B * w * 2 * d * 2 + B * w * 4
    assert sum(bench.decode_hbm_bytes(s, window=w).values()) == want_w == 896_540_928
    # FP8 K/V: each gathered row is d code bytes plus a 4-byte scale, for K and V
    want_8 = want - gather + B * k * 2 * (d + 4)
    assert sum(bench.decode_hbm_bytes(s, kv8=True).values()) == want_8 == 593_502_464


def test_prefill_flops():
    s = dsa_synth.prefill_spec("p128k")
    L, k = 131072, 2048
    pairs = L * (L + 1) // 2                                # causal (t, s) pairs, s <= t
    selected = k * (k + 1) // 2 + (L - k) * k               # sum over t of min(k, t + 1)
    f = dsa_synth.prefill_flops(s)
    assert f["pairs"] == pairs == 8_590_000_128
    assert f["selected"] == selected
    assert f["indexer_flop"] == 2 * 64 * 128 * pairs       # one multiply-add per head and index dim
    assert f["attn_flop"] == 4 * 128 * 128 * selected      # QK^T and PV, 128 heads, d 128
