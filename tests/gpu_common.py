"""Helpers shared by the GPU parity tests (CUDA path vs the fp64 CPU oracle)."""
import math

import numpy as np
import torch

# Tolerances for the three stages (fixed per stage, stated with each test):
#  indexer: |gpu - oracle| <= 1e-3 * max|I| over the compared entries
#  attention: |gpu - oracle| <= 2e-2 + 1e-2 * |oracle|
#  end-to-end selection overlap: mean over rows of |S_gpu & S_or| / |S_or| >= 0.999
IDX_REL_TOL = 1e-3
ATT_ATOL, ATT_RTOL = 2e-2, 1e-2
OVERLAP_MIN = 0.999


def to_dev(inp, device="cuda"):
    out = {}
    for k, v in inp.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.to(device)
        elif isinstance(v, list):
            out[k] = [x.to(device) if isinstance(x, torch.Tensor) else x for x in v]
        else:
            out[k] = v
    return out


def to_cpu(inp):
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def assert_scores_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isneginf(gpu), np.isneginf(ref)), f"{what}: -inf pattern differs"
    scale = np.max(np.abs(ref[fin])) if fin.any() else 1.0
    err = np.max(np.abs(gpu[fin] - ref[fin])) if fin.any() else 0.0
    assert err <= IDX_REL_TOL * scale, f"{what}: max err {err:.3e} > {IDX_REL_TOL} * {scale:.3e}"
    return err / max(scale, 1e-30)


def assert_attn_close(gpu_out, ref_out, gpu_lse=None, ref_lse=None, what=""):
    g = np.asarray(gpu_out, dtype=np.float64)
    bad = np.abs(g - ref_out) > ATT_ATOL + ATT_RTOL * np.abs(ref_out)
    assert not bad.any(), f"{what}: {bad.sum()} outputs outside tolerance, max err {np.abs(g - ref_out).max():.3e}"
    if gpu_lse is not None:
        gl = np.asarray(gpu_lse, dtype=np.float64)
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isneginf(gl), np.isneginf(ref_lse)), f"{what}: lse -inf pattern differs"
        badl = np.abs(gl[fin] - ref_lse[fin]) > ATT_ATOL + ATT_RTOL * np.abs(ref_lse[fin])
        assert not badl.any(), f"{what}: lse max err {np.abs(gl[fin] - ref_lse[fin]).max():.3e}"


def overlap(gpu_idx, ref_idx):
    """Mean and min over rows of |S_gpu & S_ref| / |S_ref| (rows with empty S_ref skipped)."""
    vals = []
    for g, r in zip(np.asarray(gpu_idx), np.asarray(ref_idx)):
        rs = set(int(x) for x in r if x >= 0)
        if not rs:
            continue
        gs = set(int(x) for x in g if x >= 0)
        vals.append(len(gs & rs) / len(rs))
    return float(np.mean(vals)), float(np.min(vals))


def check_selection_valid(idx, rows, k):
    """Every row: min(k, t+1) distinct ascending positions <= t, then -1 padding."""
    idx = np.asarray(idx)
    for r, t in enumerate(rows):
        sel = idx[r][idx[r] >= 0]
        assert sel.size == min(k, t + 1), (r, sel.size)
        assert np.all(idx[r][sel.size:] == -1)
        assert np.all(np.diff(sel) > 0) and sel.max() <= t


def sm_of(d):
    return 1.0 / math.sqrt(d)
