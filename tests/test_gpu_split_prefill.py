"""The single-sequence prefill split on one GPU: the ranks' zigzag row sets
run one after another through dsa_prefill_rows (each with only its own query
rows and the whole key side, as the all-gather leaves it) and must reproduce
dsa_prefill of the whole sequence bit for bit: the same selection, the same
bf16 outputs and log-sum-exps.  (The NCCL all-gather itself is not run here:
every call has one GPU.)"""
import numpy as np
import pytest
import torch

import dsa_synth
from long_context_fp8_b200 import dsa, split_prefill

from gpu_common import sm_of, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,k,H_q,G", [(9000, 512, 128, 2), (9000, 512, 128, 3), (5000, 256, 16, 4),
                                       (20000, 2048, 128, 8), (700, 64, 128, 1)])
def test_split_prefill_rows_match_the_whole_prefill(L, k, H_q, G):
    spec = dsa_synth.PrefillSpec("split_prefill", L=L, H_I=64, d_I=128, k=k, H_q=H_q, d=128, fp8=True,
                                 n_needles=max(1, L // 200), seed=L + G)
    inp = to_dev(dsa_synth.make_prefill(spec))
    out, lse, idx = dsa.dsa_prefill(inp, k, sm_of(128))
    keys = {f: inp[f] for f in split_prefill.KEY_FIELDS}
    seen = torch.zeros(L, dtype=torch.int32, device="cuda")
    for g in range(G):
        for b, e in split_prefill.rank_rows(L, G, g):
            rows = {f: inp[f][b:e].clone() for f in split_prefill.QUERY_FIELDS}
            o, l, i = dsa.dsa_prefill_rows(rows, keys, b, k, sm_of(128))
            torch.cuda.synchronize()
            assert torch.equal(i, idx[b:e]), (g, b, e)
            assert torch.equal(o.view(torch.int16), out[b:e].view(torch.int16)), (g, b, e)
            assert torch.equal(l, lse[b:e]), (g, b, e)
            seen[b:e] += 1
    assert bool((seen == 1).all())


def test_split_prefill_rows_unaligned_range_and_small_workspace():
    """A row range that starts inside a 128-row block, with a workspace for
    the minimum pass (128 rows), stays exact."""
    L, k = 6000, 128
    spec = dsa_synth.PrefillSpec("split_prefill", L=L, H_I=64, d_I=128, k=k, H_q=128, d=128, fp8=True,
                                 n_needles=20, seed=3)
    inp = to_dev(dsa_synth.make_prefill(spec))
    out, lse, idx = dsa.dsa_prefill(inp, k, sm_of(128))
    keys = {f: inp[f] for f in split_prefill.KEY_FIELDS}
    b, e = 4999, 5777
    rows = {f: inp[f][b:e].clone() for f in split_prefill.QUERY_FIELDS}
    full = dsa.prefill_rows_workspace_size(L, e - b, 64, 128, 128, 128, k)
    o, l, i = dsa.dsa_prefill_rows(rows, keys, b, k, sm_of(128), ws=dsa.workspace(full // 4, "cuda"))
    torch.cuda.synchronize()
    assert torch.equal(i, idx[b:e])
    assert torch.equal(o.view(torch.int16), out[b:e].view(torch.int16))
    assert torch.equal(l, lse[b:e])
