"""The fused prefill selection: dsa_prefill selects inside the indexer's
epilogue and never writes the causal score matrix.  Its selection must equal,
bit for bit, the oracle's top-k applied to the GPU's own indexer scores
(dsa_index_scores rows, the same fp32 values the fused epilogue compares),
whichever way each row is finished:

* rows whose competing positions all fit the candidate list (tau = -inf),
* rows thresholded by the sampled-key estimate and finished on chip,
* rows whose candidate count falls outside [k, cap] (massive ties), which the
  repair pass recomputes and selects with the stand-alone top-k,
* rows with a sliding window.

The inputs are seeded and synthetic; the tie-heavy ones repeat a few index
keys (identical bytes and scales give identical scores) or zero the head
weights of some rows (every score 0)."""
import numpy as np
import pytest
import torch

import dsa_synth
from oracle import oracle
from long_context_fp8_b200 import dsa

from gpu_common import OVERLAP_MIN, check_selection_valid, overlap, sm_of, to_dev

pytestmark = pytest.mark.gpu


def _spec(L, k, seed, H_q=16, H_I=64):
    return dsa_synth.PrefillSpec("fused", L=L, H_I=H_I, d_I=128, k=k, H_q=H_q, d=128, fp8=True,
                                 n_needles=max(1, L // 200), seed=seed)


def _repeat_keys(inp, period):
    """Index keys (and their scales) repeat with the given period: a row's
    scores take at most `period` distinct values."""
    T = inp["k_idx"].shape[0]
    src = torch.arange(T) % period
    inp["k_idx"] = inp["k_idx"][src].contiguous()
    inp["k_scale"] = inp["k_scale"][src].contiguous()
    return inp


def _gpu_scores(dev, r0, n):
    return dsa.dsa_index_scores(dev["q_idx"], dev["q_scale"], dev["k_idx"], dev["k_scale"], dev["w"],
                                row_begin=r0, row_count=n).cpu().numpy().astype(np.float64)


def _check_rows(dev, idx, rows, k, window=0, block=512):
    """idx[rows] equals the oracle's selection on the GPU's own score rows."""
    rows = np.asarray(rows, dtype=np.int64)
    got = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    # contiguous runs of rows share one dsa_index_scores call
    i = 0
    while i < rows.size:
        j = i
        while j + 1 < rows.size and rows[j + 1] == rows[j] + 1 and j + 1 - i < block:
            j += 1
        r0, n = int(rows[i]), j - i + 1
        sc = _gpu_scores(dev, r0, n)
        rr = np.arange(r0, r0 + n)
        ref = oracle.topk(sc, rr, k) if window == 0 else oracle.topk_window(sc, rr, k, window)
        np.testing.assert_array_equal(got[i:j + 1], ref, err_msg=f"rows {r0}..{r0 + n - 1}")
        i = j + 1
    return got


@pytest.mark.parametrize("L,k,seed", [(3000, 64, 1), (2500, 300, 2), (700, 128, 3), (1, 8, 4), (129, 128, 5)])
def test_fused_all_candidate_rows_bit_exact(L, k, seed):
    """Rows short enough that every competing position is a candidate."""
    inp = dsa_synth.make_prefill(_spec(L, k, seed))
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    torch.cuda.synchronize()
    _check_rows(dev, idx, np.arange(L), k)


@pytest.mark.parametrize("period", [1, 3, 37])
def test_fused_tie_heavy_bit_exact(period):
    """Few distinct scores per row: ties at the k-th score go to the lower positions."""
    L, k = 3000, 64
    inp = _repeat_keys(dsa_synth.make_prefill(_spec(L, k, 10 + period)), period)
    inp["w"][::5] = 0                                  # every fifth row scores 0 everywhere
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    torch.cuda.synchronize()
    _check_rows(dev, idx, np.arange(L), k)


@pytest.mark.parametrize("L,k,seed", [(12000, 256, 21), (9000, 1024, 22), (20000, 2048, 23)])
def test_fused_sampled_threshold_rows_bit_exact(L, k, seed):
    """Rows past the candidate capacity take the sampled threshold."""
    inp = dsa_synth.make_prefill(_spec(L, k, seed))
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    torch.cuda.synchronize()
    cap = max(4 * k, 4096)
    rows = np.unique(np.concatenate([np.arange(cap - 3, cap + 5), np.arange(L - 300, L),
                                     np.random.default_rng(seed).choice(L, 200, replace=False)]))
    rows = rows[(rows >= 0) & (rows < L)]
    _check_rows(dev, idx, rows, k)
    nsel = (idx >= 0).sum(dim=1).cpu().numpy()
    np.testing.assert_array_equal(nsel, np.minimum(k, np.arange(L) + 1))


def test_fused_repair_of_overflowing_rows_bit_exact():
    """Rows whose every score is equal overflow the candidate list at any
    threshold: the repair pass must return the lowest k positions; rows in the
    same blocks that did not fail, and in other blocks, stay exact."""
    L, k = 9000, 64
    inp = dsa_synth.make_prefill(_spec(L, k, 31))
    inp["w"][5000:5300] = 0                            # rows 5000..5299: all scores 0
    inp["w"][8000:] = 0
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(4900, 5400), np.arange(7990, 8010), np.arange(L - 20, L)])
    got = _check_rows(dev, idx, rows, k)
    zero = (rows >= 5000) & (rows < 5300) | (rows >= 8000)
    np.testing.assert_array_equal(got[zero], np.tile(np.arange(k, dtype=np.int32), (int(zero.sum()), 1)))


def test_fused_repair_of_every_row_of_a_pass():
    """All rows tie everywhere (one repeated key): every row past the capacity is repaired."""
    L, k = 6000, 32
    inp = _repeat_keys(dsa_synth.make_prefill(_spec(L, k, 41)), 1)
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    exp = np.tile(np.arange(k, dtype=np.int32), (L, 1))
    for t in range(k):                                  # short rows: all positions, then -1
        exp[t] = np.where(np.arange(k) <= t, np.arange(k), -1)
    np.testing.assert_array_equal(got, exp)


@pytest.mark.parametrize("k,W", [(128, 1000), (64, 5000)])
def test_fused_window_bit_exact(k, W):
    L = 9000
    inp = dsa_synth.make_prefill(_spec(L, k, 50 + W, H_q=128))
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill_window(dev, k, W, sm_of(128))
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(0, 40), np.arange(W - 2, W + 150), np.arange(4096 + W - 5, 4096 + W + 5),
                           np.arange(L - 100, L)])
    rows = np.unique(rows[rows < L])
    _check_rows(dev, idx, rows, k, window=W)


def test_fused_overlap_with_the_oracle_selection():
    """End to end: the fused selection against the oracle's selection on its
    own fp64 scores (the GPU's fp32 scores may order near-ties differently)."""
    spec = _spec(10000, 512, 61)
    inp = dsa_synth.make_prefill(spec)
    _, _, idx = dsa.dsa_prefill(to_dev(inp), spec.k, sm_of(128))
    rows = np.random.default_rng(0).choice(spec.L, 48, replace=False)
    rows = np.unique(np.concatenate([rows, [spec.L - 1]]))
    got = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    check_selection_valid(got, rows, spec.k)
    ref = oracle.prefill(inp, spec.k, sm_of(128), rows)
    mean_ov, min_ov = overlap(got, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)


def test_fused_repeat_calls_same_workspace():
    """A second call on the same workspace (stale candidate lists, counters
    and repair flags from the first) gives the same selection."""
    L, k = 7000, 128
    inp = dsa_synth.make_prefill(_spec(L, k, 71))
    inp["w"][6000:6100] = 0
    dev = to_dev(inp)
    ws = dsa.workspace(dsa.prefill_workspace_size(L, 64, 128, 16, 128, k), "cuda")
    _, _, a = dsa.dsa_prefill(dev, k, sm_of(128), ws=ws)
    inp2 = dsa_synth.make_prefill(_spec(L, k, 72))
    dsa.dsa_prefill(to_dev(inp2), k, sm_of(128), ws=ws)
    _, _, b = dsa.dsa_prefill(dev, k, sm_of(128), ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("L", [300, 700, 5000])
def test_prefill_host_edge_passes_match_device(L):
    """dsa_prefill_host runs a small first pass (the last rows) and a small last
    pass (the first rows) around full ones; per-row results do not depend on
    the pass split, so they equal dsa_prefill's bit for bit (one pass, two
    passes, and edge passes around a middle one)."""
    k = 256
    spec = dsa_synth.PrefillSpec("host_edges", L=L, H_I=64, d_I=128, k=k, H_q=128, d=128, fp8=True,
                                 n_needles=max(1, L // 200), seed=L)
    inp = to_dev(dsa_synth.make_prefill(spec))
    out_d, lse_d, idx_d = dsa.dsa_prefill(inp, k, sm_of(128))
    torch.cuda.synchronize()
    keys = ("q_idx", "q_scale", "k_idx", "k_scale", "w", "q", "k", "v")
    host = {key: inp[key].cpu().pin_memory() for key in keys}
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    lse_h = torch.empty(lse_d.shape, dtype=lse_d.dtype).pin_memory()
    idx_h = torch.empty(idx_d.shape, dtype=idx_d.dtype).pin_memory()
    dsa.dsa_prefill_host(host, k, out_h, sm_of(128), lse=lse_h, idx_out=idx_h)
    torch.cuda.synchronize()
    assert torch.equal(idx_h, idx_d.cpu())
    assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16))
    assert torch.equal(lse_h, lse_d.cpu())


@pytest.mark.parametrize("H_I", [1, 12, 32])
def test_fused_other_index_head_counts_bit_exact(H_I):
    """The fused selection with fewer index heads than 64: 32 (vector weight loads),
    12 and 1 (the coefficient table's scalar path) select exactly what the oracle
    selects on the GPU's own score rows, on sampled-threshold rows."""
    L, k = 9000, 256
    spec = _spec(L, k, seed=H_I + 17, H_I=H_I)
    inp = dsa_synth.make_prefill(spec)
    dev = to_dev(inp)
    _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    rows = np.concatenate([np.arange(0, 40), np.arange(L - 600, L)])
    _check_rows(dev, idx, rows, k)


@pytest.mark.parametrize("k,W", [(3000, 1024), (4096, 0), (4097, 0)])
def test_fused_large_k_bit_exact(k, W):
    """k beyond 2048 takes the finish kernel's largest candidate capacity (4 k
    candidates a row, 64 a thread); k = 4096 is the largest fused k and 4097
    takes the score-writing path.  Rows where every position is taken, where
    every competing position is a candidate, and where the sampled threshold
    applies all select exactly what the oracle selects on the GPU's scores."""
    L = 20000
    spec = _spec(L, k, seed=k + W)
    inp = dsa_synth.make_prefill(spec)
    dev = to_dev(inp)
    if W:
        idx = dsa.dsa_prefill_window(dev, k, W, sm_of(128))[2]
    else:
        _, _, idx = dsa.dsa_prefill(dev, k, sm_of(128))
    rows = np.concatenate([np.arange(k - 3, k + 3), np.arange(4 * k + W - 3, 4 * k + W + 3),
                           np.arange(L - 200, L)])
    _check_rows(dev, idx, rows, k, window=W)
