"""bench.py's N > 1 path on CPU: two gloo ranks (127.0.0.1) take the same
collective steps as the GPU ranks -- barrier, max over ranks of the step time --
serve batches of the same shape with their own seeds, and report the
whole-job throughput from the slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import dsa_inputs as di
        bench.barrier(world)
        my_ms = 2.0 + rank                      # rank 1 is the slower one
        worst = bench.max_over_ranks(my_ms, world)
        spec = bench.rank_spec(di.config("decode128k"), rank, world)
        value = bench.aggregate_throughput(spec.T, worst, world)
        out[rank] = (worst, spec.seed, spec.T, tuple(spec.kv_lens), value)
        bench.barrier(world)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_shard_the_batches():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0, 0], codes
        r0, r1 = out[0], out[1]
    # both ranks see the slowest rank's step time
    assert r0[0] == r1[0] == 3.0
    # same batch shape (tokens per rank), different seeds: weak scaling with no exchange
    assert r0[2] == r1[2] == 64 and r0[1] != r1[1]
    # the seed changes the generated inputs but not the lengths of the configuration
    assert r0[3] == r1[3]
    # whole-job throughput = all ranks' tokens over the slowest rank's time
    assert r0[4] == pytest.approx(2 * 64 / 3e-3)
