"""The multi-rank bookkeeping of bench.py, run as two gloo ranks on the host.

Under torchrun every rank runs its own independent problem (weak scaling, no
data-path collective); the job's step time is the max over ranks and the
whole-job rate is world_size x the per-rank units over that time.  These
tests run that logic on CPU with world_size 2.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, root):
    import sys
    sys.path.insert(0, root)
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import dsa_synth
    import torch.distributed as dist

    ws, r, _ = bench.dist_setup(backend="gloo")
    try:
        assert (ws, r) == (world, rank)
        assert dist.get_backend() == "gloo"

        # The max over ranks of a per-rank step time.
        per_rank_ms = [12.5, 31.25, 7.0][:world]
        m = bench.max_over_ranks(per_rank_ms[rank], ws)
        assert m == max(per_rank_ms)

        # Whole-job rate: every rank's units over the slowest rank's time.
        T = 1024
        rate = bench.whole_job_rate(ws, T, m)
        assert rate == pytest.approx(world * T / (max(per_rank_ms) * 1e-3), rel=1e-12)

        # Each rank's problem: same shapes, its own seed; rank 0 keeps the
        # single-GPU workload unchanged.
        base = dsa_synth.prefill_spec("tiny")
        spec = bench.replica_spec(base, rank)
        if rank == 0:
            assert spec == base
        inp = dsa_synth.make_prefill(spec, device="cpu")
        shapes = {k: tuple(v.shape) for k, v in inp.items() if torch.is_tensor(v)}
        digest = torch.tensor([float(inp["q"].double().sum()), float(inp["k_idx"].double().sum())],
                              dtype=torch.float64)
        gathered = [torch.zeros_like(digest) for _ in range(ws)]
        dist.all_gather(gathered, digest)
        for other in range(ws):
            if other != rank:
                assert not torch.equal(gathered[other], digest), "ranks drew the same problem"
        all_shapes = [None] * ws
        dist.all_gather_object(all_shapes, shapes)
        assert all(s == shapes for s in all_shapes)

        # Decode replicas: same rule.
        dbase = dsa_synth.decode_spec("dec64x64k")
        dspec = bench.replica_spec(dbase, rank)
        assert dspec.B == dbase.B and dspec.context_lens == dbase.context_lens
        assert (dspec.seed == dbase.seed) == (rank == 0)

        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_bench_ranks_gloo(world):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    mp.spawn(_rank_main, args=(world, _free_port(), root), nprocs=world, join=True)


def test_whole_job_rate_single_rank():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1, 131072, 125.0) == pytest.approx(131072 / 0.125)
