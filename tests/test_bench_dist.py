"""The benchmark's multi-process plumbing on CPU: two gloo ranks set up the process
group, meet at the barrier and agree on the max over ranks (the N-GPU bench times
every rank and reports the slowest); the reference arm does its work on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup(world, backend="gloo")
    try:
        bench.barrier(w)
        m = bench.max_over_ranks(1.5 + 10.0 * r, w)
        args = type("A", (), {"steps": 1, "warmup": 0})()
        ref = bench.run_reference(args, r, w) if r != 0 else "skipped"
        out.put((r, w, local, m, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_reference_runs_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[:3] for g in got] == [(0, 2, 0), (1, 2, 1)]
    assert all(g[3] == pytest.approx(11.5) for g in got)
    assert got[1][4] is None                     # rank 1 of the reference arm does no work


def test_chunk_roofline_helpers():
    """FLOP count of the chunk-attention sub-benchmark and the fp16 tensor peak it is
    compared with (host logic only)."""
    import bench
    # Qwen3-32B-shaped layer: 32 sequences x 16 queries x 64 heads x 8192 positions, 512 FLOPs each
    assert bench.chunk_flops(32, 16, 64, 8192) == 512 * 32 * 16 * 64 * 8192 == 137438953472
    peak, kind = bench._f16_tensor_peak()
    assert peak > 1000.0 and "fp16" in kind
