"""Multi-rank host logic on CPU, with gloo ranks:

* the benchmark: every rank learns the slowest rank's step time, the
  whole-job throughput counts every rank's tokens, and the reference arm runs
  on rank 0 only (head-sharded replicas have no data-path collective);
* the sequence-sharded forward's one exchange: rank r receives the sum of
  the states of ranks 0 .. r-1 (the carry into its slice);
* the sequence-sharded forward end to end (slice, state, exchange,
  carry-in), with the library's two calls stood in for by the fp64 oracle:
  the ranks' outputs are the whole sequence's."""

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


def _sp_forward_main(rank, world, port, feature, out):
    """One rank of the sequence-sharded forward, with the library's two calls
    replaced in this process by fp64 oracle stand-ins of the same signature:
    what runs is the host logic (slice, state, exchange, carry-in)."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        import torch

        import oracle as O
        from kernelized_linear_attention_kata_b200 import api
        from kernelized_linear_attention_kata_b200 import sequence_parallel as SP

        def oracle_state(k, v, C, feature="psd"):
            B, H, _, _ = k.shape
            D = O.state_dim(k.shape[3], feature)
            S = torch.zeros((B, H, D, v.shape[3]), dtype=torch.float64)
            z = torch.zeros((B, H, D), dtype=torch.float64)
            for b in range(B):
                for h in range(H):
                    Sn, zn = O.final_state(k[b, h].numpy(), v[b, h].numpy(), feature)
                    S[b, h], z[b, h] = torch.from_numpy(Sn), torch.from_numpy(zn)
            return S, z

        def oracle_forward(q, k, v, o, C, feature="psd", S_out=None, z_out=None, S0=None, z0=None,
                           **_):
            for b in range(q.shape[0]):
                for h in range(q.shape[1]):
                    y, S, z = O.forward_chunked(q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(), C,
                                                feature, S0=S0[b, h].numpy(), z0=z0[b, h].numpy(),
                                                return_state=True)
                    o[b, h] = torch.from_numpy(y)
                    if S_out is not None:
                        S_out[b, h], z_out[b, h] = torch.from_numpy(S), torch.from_numpy(z)
            return o

        api.chunked_state = oracle_state
        api.kata_fwd_chunked = oracle_forward
        r = np.random.default_rng(21)                     # the same sequence on every rank
        B, H, T, d_k, d_v = 1, 2, 40 * world, 4, 3
        unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)  # noqa: E731
        q = unit(r.standard_normal((B, H, T, d_k)))
        k = unit(r.standard_normal((B, H, T, d_k)))
        v = r.standard_normal((B, H, T, d_v))
        sl = slice(rank * 40, (rank + 1) * 40)
        qs, ks, vs = (torch.from_numpy(np.ascontiguousarray(x[:, :, sl])) for x in (q, k, v))
        o, S, z = SP.fwd_chunked_sequence_parallel(qs, ks, vs, 16, feature, return_state=True)
        out[rank] = (o.numpy(), S.numpy(), z.numpy(), (q, k, v))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,feature", [(2, "psd"), (3, "psd"), (2, "first_order")])
def test_sequence_sharded_forward_equals_the_whole_sequence(world, feature):
    """Slices of 40 tokens (two full chunks of 16 and a ragged one) on each
    rank: the ranks' outputs, in rank order, are the whole sequence's, and the
    last rank's state is the whole sequence's state."""
    import numpy as np

    import oracle as O

    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_sp_forward_main, args=(world, port, feature, out), nprocs=world, join=True)
        res = dict(out)
    q, k, v = res[0][3]
    y = np.concatenate([res[r][0] for r in range(world)], axis=2)
    ref = O.per_head(O.forward_brute_force, q, k, v, feature)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)
    for h in range(q.shape[1]):
        S_ref, z_ref = O.final_state(k[0, h], v[0, h], feature)
        assert np.allclose(res[world - 1][1][0, h], S_ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(res[world - 1][2][0, h], z_ref, rtol=1e-12, atol=1e-12)


def _bench_lines(argv, env=None):
    import json
    import subprocess
    e = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        e.pop(k, None)
    e.update(env or {})
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv], env=e,
                       capture_output=True, text=True, timeout=300)
    lines = [json.loads(l) for l in p.stdout.splitlines() if l.startswith("{")]
    return p.returncode, lines, p.stderr


def test_bench_starts_its_own_ranks():
    """`bench.py --gpus 2` without a launcher in the environment re-runs itself
    as two ranks under torch.distributed.run; rank 0 alone prints the line,
    with n_gpus = 2 (reference arm: the CPU oracle, so no GPU is needed)."""
    rc, lines, err = _bench_lines(["--gpus", "2", "--impl", "reference", "--steps", "1",
                                   "--warmup", "0", "--workload", "tiny_f32",
                                   "--ref-step-budget", "0.2"])
    assert rc == 0, err[-2000:]
    assert len(lines) == 1, lines
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_bench_rejects_a_rank_count_the_launcher_did_not_start():
    rc, lines, err = _bench_lines(["--gpus", "3", "--impl", "reference", "--steps", "1",
                                   "--warmup", "0", "--workload", "tiny_f32"],
                                  env={"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert rc != 0 and not lines
    assert "--gpus 3" in err
