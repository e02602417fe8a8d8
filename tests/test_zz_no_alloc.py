"""The allocation-free decode entry point (dsa_decode_noalloc) against the
workspace one (dsa_decode), through the C ABI, on two calls in a row.

dsa_decode_noalloc serves callers that cannot allocate device memory (for
example a plugin whose host has reserved all device memory in its own pool):
it runs the same kernels on a fixed scratch array inside the library.  This
file is collected last so that a stop-at-first-failure run has already run
every other test; it passes alone in a fresh process too."""
import numpy as np
import pytest
import torch

import dsa_synth
from long_context_fp8_b200 import dsa

from gpu_common import assert_attn_close

pytestmark = pytest.mark.gpu


def _decode_inputs(lens, seed, k=128, H_q=16):
    spec = dsa_synth.DecodeSpec("noalloc", context_lens=tuple(lens), H_I=64, d_I=128, k=k, H_q=H_q,
                                d=128, page_size=64, needle_frac=0.01, needle_min_age=0, seed=seed)
    inp = dsa_synth.make_decode(spec, device="cuda")
    inp.pop("needle_pos")
    return spec, inp


def _both(spec, inp):
    maxc = max(spec.context_lens)
    B, H_q = spec.B, spec.H_q
    ref_out, ref_lse, ref_idx = dsa.dsa_decode(inp, spec.k, maxc)
    out = torch.empty_like(inp["q"])
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, spec.k), dtype=torch.int32, device="cuda")
    status = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    dsa.dsa_decode_noalloc(inp, spec.k, maxc, out=out, lse=lse, idx_out=idx, status_out=status)
    torch.cuda.synchronize()
    return (ref_out, ref_lse, ref_idx), (out, lse, idx), int(status.item())


def test_noalloc_matches_workspace_entry_point_twice():
    # two calls in a row, the second smaller than the first, so that stale
    # scratch contents from the first call would show up in the second
    for lens, seed in (((3000, 700, 64, 2049), 5), ((900, 1), 6)):
        spec, inp = _decode_inputs(lens, seed)
        (ro, rl, ri), (o, l, i), status = _both(spec, inp)
        assert status == 0
        np.testing.assert_array_equal(i.cpu().numpy(), ri.cpu().numpy())
        assert_attn_close(o.float().cpu().numpy(), ro.double().cpu().numpy(),
                          l.cpu().numpy(), rl.double().cpu().numpy(), f"noalloc {lens}")


def test_noalloc_rejects_problems_beyond_the_scratch():
    spec, inp = _decode_inputs((256,), 7)
    # a declared context bound whose score buffer alone exceeds the fixed scratch
    too_long = dsa.NOALLOC_SCRATCH_BYTES // 4
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_decode_noalloc(inp, spec.k, too_long)
    assert e.value.status == 3          # DSA_ERR_WORKSPACE


def test_noalloc_reports_device_status():
    spec, inp = _decode_inputs((500, 300), 8, k=64)
    inp["block_table"][1, 2] = 10 ** 6     # out-of-range page id: caught by the kernels' bounds checks
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out, _, _ = dsa.dsa_decode_noalloc(inp, spec.k, 500, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1       # DSA_ERR_INVALID_ARG
    inp["block_table"][1, 2] = 0


def test_noalloc_second_call_reserves_no_device_memory():
    # The scratch array is reserved by the first call on a device (lazy module
    # loading); every later call must leave the device's free memory unchanged.
    spec, inp = _decode_inputs((1500, 400), 9, k=64)
    maxc = max(spec.context_lens)
    out = torch.empty_like(inp["q"])
    lse = torch.empty((spec.B, spec.H_q), dtype=torch.float32, device="cuda")
    idx = torch.empty((spec.B, spec.k), dtype=torch.int32, device="cuda")
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    dsa.dsa_decode_noalloc(inp, spec.k, maxc, out=out, lse=lse, idx_out=idx, status_out=status)
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    dsa.dsa_decode_noalloc(inp, spec.k, maxc, out=out, lse=lse, idx_out=idx, status_out=status)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, (free_before, free_after)
    assert int(status.item()) == 0
