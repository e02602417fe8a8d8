"""Parity at the full workload sizes, in the launch configuration the
benchmark times: the whole path runs on the GPU; the fp64 oracle checks a
sample of query rows / sequences it can compute one by one (always including
the last, longest row), plus properties that hold at any size."""
import numpy as np
import pytest
import torch

import dsa_synth
from oracle import oracle
from long_context_fp8_b200 import dsa

from gpu_common import (OVERLAP_MIN, assert_attn_close, assert_scores_close,
                        check_selection_valid, overlap, sm_of)

pytestmark = pytest.mark.gpu


def _sample_rows(L, n, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(L, n - 3, replace=False).tolist()) | {0, 2047 % L, L - 1}
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name,nrows", [("p16k", 12), ("p128k", 6)])
def test_prefill_fullsize_sampled(name, nrows):
    spec = dsa_synth.prefill_spec(name)
    inp = dsa_synth.make_prefill(spec, device="cuda")
    out, lse, idx = dsa.dsa_prefill(inp, spec.k, sm_of(spec.d))
    torch.cuda.synchronize()
    rows = _sample_rows(spec.L, nrows, seed=spec.seed)
    rt = torch.from_numpy(rows).cuda()
    idx_s = idx[rt].cpu().numpy()
    check_selection_valid(idx_s, rows, spec.k)

    # indexer parity on the sampled rows (GPU scores through dsa_index_scores)
    k_idx, k_scale = inp["k_idx"].cpu(), inp["k_scale"].cpu()
    q_rows, qs_rows, w_rows = inp["q_idx"][rt].cpu(), inp["q_scale"][rt].cpu(), inp["w"][rt].cpu()
    ref_sc = oracle.index_scores(q_rows, qs_rows, k_idx, k_scale, w_rows, rows, compact=True)
    for i, t in enumerate(rows):
        g = dsa.dsa_index_scores(inp["q_idx"], inp["q_scale"], inp["k_idx"], inp["k_scale"], inp["w"],
                                 row_begin=int(t), row_count=1).cpu().numpy()
        assert_scores_close(g, ref_sc[i:i + 1], f"{name} row {t}")
        # the selector on the GPU's own scores is bit-exact
        gsel = oracle.topk(g.astype(np.float64), [t], spec.k)
        np.testing.assert_array_equal(idx_s[i], gsel[0])
    # end-to-end overlap with the oracle's own selection
    ref_idx = oracle.topk(ref_sc, rows, spec.k)
    mean_ov, min_ov = overlap(idx_s, ref_idx)
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    # attention parity on the sampled rows, given the GPU selection
    ro, rl = oracle.sparse_attn(inp["q"][rt].cpu(), inp["k"].cpu(), inp["v"].cpu(), idx_s, rows,
                                sm_of(spec.d), compact=True)
    assert_attn_close(out[rt].float().cpu().numpy(), ro, lse[rt].cpu().numpy(), rl, name)
    # properties at every row: finite outputs, valid selection shape
    assert torch.isfinite(out.float()).all()
    nsel = (idx >= 0).sum(dim=1).cpu().numpy()
    expect = np.minimum(spec.k, np.arange(spec.L) + 1)
    np.testing.assert_array_equal(nsel, expect)


def _subset_decode(inp, bs):
    sub = dict(inp)
    for key in ("q_idx", "q_scale", "w", "q", "block_table", "context_lens"):
        sub[key] = inp[key][bs]
    return sub


@pytest.mark.parametrize("name,seqs", [("dec64x64k", [0, 17, 63]), ("dec_ragged", [0, 3])])
def test_decode_fullsize_sampled(name, seqs):
    spec = dsa_synth.decode_spec(name)
    inp = dsa_synth.make_decode(spec, device="cuda")
    out, lse, idx = dsa.dsa_decode(inp, spec.k, max(spec.context_lens), sm_of(spec.d))
    torch.cuda.synchronize()
    nsel = (idx >= 0).sum(dim=1).cpu().numpy()
    np.testing.assert_array_equal(nsel, np.minimum(spec.k, np.array(spec.context_lens)))
    bs = torch.tensor(seqs)
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()
           if k != "needle_pos"}
    sub = _subset_decode(cpu, bs)
    ref = oracle.decode(sub, spec.k, sm_of(spec.d))
    idx_s = idx[bs.cuda()].cpu().numpy()
    mean_ov, min_ov = overlap(idx_s, ref["idx"])
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    # attention given the GPU selection
    bt = sub["block_table"].numpy()
    ps = spec.page_size
    kc = cpu["k_cache"].reshape(-1, spec.d)
    vc = cpu["v_cache"].reshape(-1, spec.d)
    for i, b in enumerate(seqs):
        sel = idx_s[i][idx_s[i] >= 0]
        slot = torch.from_numpy(bt[i, sel // ps].astype(np.int64) * ps + sel % ps)
        ro, rl = oracle.sparse_attn(sub["q"][i:i + 1], kc[slot], vc[slot],
                                    np.arange(sel.size, dtype=np.int32)[None], [0], sm_of(spec.d))
        assert_attn_close(out[b:b + 1].float().cpu().numpy(), ro, lse[b:b + 1].cpu().numpy(), rl,
                          f"{name} seq {b}")
    # planted needles (noisy copies of the new query): a sanity metric, not a
    # parity criterion -- the GPU recalls as many as the oracle's own selection
    hits_g, hits_o = 0, 0
    for i, b in enumerate(seqs):
        pos = set(inp["needle_pos"][b].tolist())
        hits_g += len(pos & set(idx_s[i].tolist()))
        hits_o += len(pos & set(ref["idx"][i].tolist()))
    assert abs(hits_g - hits_o) <= max(2, hits_o // 100), (hits_g, hits_o)


@pytest.mark.parametrize("name", ["p16k_hq128"])
def test_prefill_host_matches_device(name):
    """dsa_prefill_host (inputs and outputs in page-locked host memory, moved
    pass by pass alongside the computation) returns exactly what dsa_prefill
    returns on device-resident inputs: same kernels, same passes."""
    spec = dsa_synth.prefill_spec(name)
    inp = dsa_synth.make_prefill(spec, device="cuda")
    out_d, lse_d, idx_d = dsa.dsa_prefill(inp, spec.k, sm_of(spec.d))
    torch.cuda.synchronize()
    keys = ("q_idx", "q_scale", "k_idx", "k_scale", "w", "q", "k", "v")
    host = {key: inp[key].cpu().pin_memory() for key in keys}
    out_h = torch.empty(out_d.shape, dtype=out_d.dtype).pin_memory()
    lse_h = torch.empty(lse_d.shape, dtype=lse_d.dtype).pin_memory()
    idx_h = torch.empty(idx_d.shape, dtype=idx_d.dtype).pin_memory()
    dsa.dsa_prefill_host(host, spec.k, out_h, sm_of(spec.d), lse=lse_h, idx_out=idx_h)
    torch.cuda.synchronize()
    assert torch.equal(idx_h, idx_d.cpu())
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(lse_h, lse_d.cpu())
