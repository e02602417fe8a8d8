"""The device-side bounded waits, made to run out on purpose through the
library's test hook (dsa_test_stall_next): the next launch of the named
tcgen05 indexer leaves one copy unissued in CTA 0, so that CTA's consumer
waits for data that never comes.  The wait must give up after its limit, the
kernel must report DSA_ERR_TIMEOUT through the workspace status word and
return (copies and MMAs it issued landed, tensor memory freed), and the
context must stay usable: the next call on the same workspace reports no
error and returns the oracle's results.  No fault, trap or endless wait is
involved: the hook only withholds a copy."""
import math

import numpy as np
import pytest
import torch

import dsa_synth
from oracle import oracle
from long_context_fp8_b200 import dsa

from gpu_common import assert_attn_close, overlap, sm_of, to_dev

pytestmark = pytest.mark.gpu

DSA_OK, DSA_ERR_TIMEOUT = 0, 5


def test_prefill_indexer_wait_runs_out_then_the_next_call_is_exact():
    spec = dsa_synth.PrefillSpec("stall", L=2000, H_I=64, d_I=128, k=64, H_q=128, d=128, fp8=True,
                                 n_needles=20, seed=91)
    inp = dsa_synth.make_prefill(spec)
    dev = to_dev(inp)
    ws = dsa.workspace(dsa.prefill_workspace_size(spec.L, 64, 128, 128, 128, spec.k), "cuda")
    dsa.test_stall_next(dsa.STALL_PREFILL_INDEXER)
    dsa.dsa_prefill(dev, spec.k, sm_of(128), ws=ws)
    assert dsa.dsa_stream_status(ws) == DSA_ERR_TIMEOUT
    # the same workspace again: no error, and the exact selection of the GPU's own scores
    out, lse, idx = dsa.dsa_prefill(dev, spec.k, sm_of(128), ws=ws)
    assert dsa.dsa_stream_status(ws) == DSA_OK
    rows = np.arange(spec.L)
    sc = dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"], dev["w"]).cpu().numpy()
    np.testing.assert_array_equal(idx.cpu().numpy(), oracle.topk(sc.astype(np.float64), rows, spec.k))
    sel = idx.cpu().numpy()
    pick = rows[::97]
    ro, rl = oracle.sparse_attn(inp["q"][torch.from_numpy(pick)], inp["k"], inp["v"], sel[pick], pick, sm_of(128),
                                compact=True)
    assert_attn_close(out.float().cpu().numpy()[pick], ro, lse.cpu().numpy()[pick], rl, "after stall")


def test_decode_indexer_wait_runs_out_then_the_next_call_is_exact():
    spec = dsa_synth.DecodeSpec("stall_dec", context_lens=(3000, 700, 5000), H_I=64, d_I=128, k=128, H_q=128,
                                d=128, page_size=64, needle_frac=0.01, needle_min_age=0, seed=92)
    inp = dsa_synth.make_decode(spec)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items() if k != "needle_pos"}
    maxc = max(spec.context_lens)
    ws = dsa.workspace(dsa.decode_workspace_size(spec.B, maxc, spec.H_q, spec.d, spec.k), "cuda")
    dsa.test_stall_next(dsa.STALL_DECODE_INDEXER)
    dsa.dsa_decode(dev, spec.k, maxc, ws=ws)
    assert dsa.dsa_stream_status(ws) == DSA_ERR_TIMEOUT
    out, lse, idx = dsa.dsa_decode(dev, spec.k, maxc, ws=ws)
    assert dsa.dsa_stream_status(ws) == DSA_OK
    ref = oracle.decode(inp, spec.k, sm_of(128))
    mean_ov, _ = overlap(idx.cpu().numpy(), ref["idx"])
    assert mean_ov >= 0.999
    if np.array_equal(idx.cpu().numpy(), ref["idx"]):
        assert_attn_close(out.float().cpu().numpy(), ref["out"], lse.cpu().numpy(), ref["lse"], "decode after stall")


def test_stall_hook_is_one_shot_and_can_be_disarmed():
    dsa.test_stall_next(dsa.STALL_PREFILL_INDEXER)
    dsa.test_stall_next(dsa.STALL_NONE)                 # disarmed before any launch
    spec = dsa_synth.PrefillSpec("stall_off", L=600, H_I=64, d_I=128, k=32, H_q=16, d=128, fp8=True,
                                 n_needles=4, seed=93)
    dev = to_dev(dsa_synth.make_prefill(spec))
    ws = dsa.workspace(dsa.prefill_workspace_size(spec.L, 64, 128, 16, 128, spec.k), "cuda")
    dsa.dsa_prefill(dev, spec.k, sm_of(128), ws=ws)
    assert dsa.dsa_stream_status(ws) == DSA_OK
