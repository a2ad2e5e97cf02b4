"""Multi-rank host logic on CPU, with gloo ranks:

* the benchmark: every rank learns the slowest rank's step time, the
  whole-job throughput counts every rank's tokens, and the reference arm runs
  on rank 0 only (head-sharded replicas have no data-path collective);
* the sequence-sharded forward's one exchange: rank r receives the sum of
  the states of ranks 0 .. r-1 (the carry into its slice)."""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = 2.0 + 3.0 * rank                    # rank 1 is the slow one
        value, ms_max = bench.aggregate_throughput(ms, 131072, world, "cpu")
        out[rank] = (value, ms_max, bench.max_over_ranks(-rank, world, "cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        value, ms_max, neg = res[rank]
        assert ms_max == 5.0
        assert value == pytest.approx(2 * 131072 / 5e-3)
        assert neg == 0.0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    value, ms = bench.aggregate_throughput(4.0, 1000, 1, "cpu")
    assert ms == 4.0 and value == pytest.approx(1000 / 4e-3)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "long131k_bf16"
        steps = 1
        warmup = 0
        ref_step_budget = 0.5

    assert bench.run_reference(Args, 1, 2) == 0     # rank 1: no work, no output
    assert capsys.readouterr().out == ""


def _prefix_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch

        from kernelized_linear_attention_kata_b200.sequence_parallel import \
            exclusive_prefix_over_ranks
        # rank r's "state": distinct powers of two, so every partial sum is exact
        # and identifies exactly which ranks were summed
        local = torch.full((3, 5), float(2 ** rank), dtype=torch.float32)
        local[0, 0] = float(rank + 1) * 1000.0
        out[rank] = exclusive_prefix_over_ranks(local).tolist()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_shards_receive_the_exclusive_prefix(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_prefix_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        got = res[rank]
        want_fill = float(sum(2 ** r for r in range(rank)))
        want_corner = float(sum((r + 1) * 1000 for r in range(rank)))
        assert got[0][0] == want_corner
        assert all(x == want_fill for row in got for x in row[1:])
        assert all(row[0] == want_fill for row in got[1:])
