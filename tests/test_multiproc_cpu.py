"""The multi-rank (N > 1) host path of bench.py on CPU: two processes with the
gloo backend, rendezvous on 127.0.0.1.  The GPU machine runs one GPU per call, so
these are the tests of the rank logic."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    class A:
        gpus = world
    w, r, _ = bench.dist_setup(A())
    try:
        bench.barrier(w)
        m = bench.max_over_ranks(1.5 + r, w)
        # rank r "took" 1 + r seconds for 10 steps of 100 units each
        rate = bench.aggregate_rate(w, 10, 100, 1.0 + r)
        out_q.put((r, m, rate))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_rate_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for r, m, rate in res:
        assert m == 2.5                             # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 10 * 100 / 2.0)   # all units over the slowest rank


def test_rank_seeds_differ():
    seeds = {bench.rank_seed(1001, r) for r in range(8)}
    assert len(seeds) == 8


def test_reference_arm_under_torchrun():
    """`--impl reference` launched as the driver launches multi-GPU runs: rank 0
    alone prints one JSON line, the other rank exits 0 without work."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def _seqpar_worker(rank, world, port, out_q):
    """One rank of the sequence-sharded forward protocol over gloo, with the
    oracle doing each segment's scan (this test checks the exchange: which
    rank runs what, gather order, carry-in selection)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from selective_state_space_50_b200 import seqpar
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = np.random.default_rng(5)
        batch, dim, N, L = 2, 3, 4, 60
        u, delta, z = r.standard_normal((3, batch, dim, L))
        A = -np.exp(r.standard_normal((dim, N)))
        B, C = r.standard_normal((2, batch, N, L))
        D = r.uniform(0.5, 1.5, dim)
        bias = r.uniform(-1, 1, dim)
        Ls = L // world
        sl = slice(rank * Ls, (rank + 1) * Ls)
        calls = []

        def run_segment(h0):
            calls.append(h0 is not None)
            out, last = oracle.fwd(u[..., sl], delta[..., sl], A, B[..., sl], C[..., sl], D,
                                   z[..., sl], bias, True, h0=None if h0 is None else h0.numpy())
            return out, torch.from_numpy(last), torch.from_numpy(oracle.delta_sums(delta[..., sl], bias))

        def gather(x):   # the helper the CUDA path uses, here over gloo
            return seqpar.all_gather_stacked(x)

        def combine(ds, es):
            return torch.from_numpy(oracle.combine_carries(A, ds.numpy(), es.numpy()))

        out, last = seqpar.forward_rank(rank, run_segment, gather, combine)
        want, wlast = oracle.fwd(u, delta, A, B, C, D, z, bias, True)
        ok_out = np.allclose(out, want[..., sl], rtol=1e-11, atol=1e-12)
        ok_last = rank != world - 1 or np.allclose(last.numpy(), wlast, rtol=1e-11, atol=1e-12)
        out_q.put((rank, bool(ok_out), bool(ok_last), calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharded_forward_protocol_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seqpar_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ok_out, ok_last, calls in res:
        assert ok_out and ok_last, rank
        # pass 1 from zeros everywhere; pass 2 from the carry-in on ranks > 0 only
        assert calls == ([False] if rank == 0 else [False, True])


def _dp_worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    from selective_state_space_50_b200 import dp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = {"dA": torch.full((6, 4), float(rank + 1)), "dD": torch.arange(6.0) * (rank + 1),
             "ddelta_bias": None, "du": torch.full((2, 6, 8), float(rank))}
        dp.allreduce_param_grads(g)
        tot = sum(r + 1 for r in range(world))
        ok = (torch.equal(g["dA"], torch.full((6, 4), float(tot)))
              and torch.equal(g["dD"], torch.arange(6.0) * tot)
              and g["ddelta_bias"] is None
              and torch.equal(g["du"], torch.full((2, 6, 8), float(rank))))   # activation grads untouched
        out_q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_data_parallel_param_grad_allreduce_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(ok for _, ok in res)
