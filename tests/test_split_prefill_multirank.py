"""The rank orchestration of the single-sequence prefill split
(split_prefill: the zigzag row partition, the key-side message and its one
all-gather), run as gloo ranks on the host.  Each rank holds only its two
chunks' per-token inputs; the per-rank prefill of a row range is played by a
CPU stand-in built on the oracle (its indexer, selection and attention for
the listed rows, reading only this rank's query rows and the gathered key
side).  The union of the ranks' outputs must equal the oracle's prefill of
the whole sequence, and the gathered key side must equal the original bytes."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SM = 0.125
K_SEL = 24


class OracleOps:
    """CPU stand-in for the per-rank prefill of rows [row_begin, row_begin + n)."""

    def prefill_rows(self, rows, keys, row_begin, k_sel, sm_scale):
        from oracle import oracle
        n = rows["q_idx"].shape[0]
        T = keys["k_idx"].shape[0]
        full = {}
        for f in ("q_idx", "q_scale", "w", "q"):          # query side: only this range is filled
            x = rows[f]
            buf = torch.zeros((T,) + tuple(x.shape[1:]), dtype=x.dtype)
            buf[row_begin:row_begin + n] = x
            full[f] = buf
        full.update(keys)
        res = oracle.prefill(full, k_sel, sm_scale, np.arange(row_begin, row_begin + n))
        return res["out"], res["lse"], res["idx"]


def _rank_main(rank, world, port, root):
    import sys
    sys.path.insert(0, root)
    import torch.distributed as dist
    import dsa_synth
    from oracle import oracle
    from long_context_fp8_b200 import split_prefill

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        spec = dsa_synth.PrefillSpec("split_prefill_cpu", L=301, H_I=8, d_I=128, k=K_SEL, H_q=8, d=128,
                                     fp8=True, n_needles=4, seed=5)
        inp = dsa_synth.make_prefill(spec)                 # the same problem on every rank
        T = spec.L
        chunks = []
        for b, e in split_prefill.rank_rows(T, world, rank):
            chunks.append({f: inp[f][b:e].clone() for f in split_prefill.QUERY_FIELDS + split_prefill.KEY_FIELDS})
        keys = split_prefill.gather_keys(chunks, T)
        for f in split_prefill.KEY_FIELDS:                 # the exchange is exact
            assert torch.equal(keys[f].view(torch.uint8), inp[f].contiguous().view(torch.uint8)), f
        res = split_prefill.split_prefill(chunks, T, spec.k, sm_scale=SM, ops=OracleOps())
        ref = oracle.prefill(inp, spec.k, SM, np.arange(T))
        covered = []
        for (b, e), (out, lse, idx) in zip(split_prefill.rank_rows(T, world, rank), res):
            np.testing.assert_array_equal(idx, ref["idx"][b:e])
            np.testing.assert_array_equal(out, ref["out"][b:e])
            np.testing.assert_array_equal(lse, ref["lse"][b:e])
            covered.extend(range(b, e))
        # the ranks' rows cover every row exactly once
        mine = torch.zeros(T, dtype=torch.int64)
        mine[torch.tensor(covered, dtype=torch.int64)] += 1
        dist.all_reduce(mine)
        assert torch.equal(mine, torch.ones(T, dtype=torch.int64))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_prefill_gloo(world):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    mp.spawn(_rank_main, args=(world, _free_port(), root), nprocs=world, join=True)


def test_zigzag_chunks_cover_every_row_once_and_balance_the_work():
    from long_context_fp8_b200 import split_prefill
    for T in (1, 7, 301, 131072, 131075):
        for G in (1, 2, 3, 4, 8):
            rows = [r for g in range(G) for r in split_prefill.rank_rows(T, G, g)]
            cov = np.zeros(T, np.int64)
            for b, e in rows:
                cov[b:e] += 1
            assert np.all(cov == 1), (T, G)
            if T >= 1024:
                # causal work of a rank: sum over its rows of (t + 1)
                work = [sum((e * (e + 1) - b * (b + 1)) // 2 for b, e in split_prefill.rank_rows(T, G, g))
                        for g in range(G)]
                assert max(work) / min(work) < 1.01, (T, G, work)


def test_key_message_layout_is_16_byte_aligned():
    from long_context_fp8_b200 import split_prefill
    for c_max in (1, 3, 100, 16384):
        off, slot = split_prefill.key_layout(c_max, 128, 128)
        assert all(v % 16 == 0 for v in off.values()) and slot % 16 == 0
        assert off["k_scale"] >= c_max * 128 and off["k"] >= off["k_scale"] + 4 * c_max
        assert off["v"] >= off["k"] + 2 * c_max * 128 and slot >= off["v"] + 2 * c_max * 128
