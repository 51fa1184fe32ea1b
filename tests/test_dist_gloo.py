"""The multi-rank path of bench.py on CPU with the gloo backend (world size 2): ranks run
independent replicas, the step time is the max over ranks and the throughput aggregates all
ranks' tokens (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    bench._dist = dist
    try:
        local_ms = 10.0 * (rank + 1)            # rank 1 is the slow one
        ms, value = bench.replica_throughput(local_ms, steps=5, tokens_per_rank=1000, world=world)
        bench.barrier()
        out[rank] = (ms, value)
    finally:
        bench._dist = None
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_replica_timing_is_max_over_ranks_and_tokens_add_up():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        # both ranks need the same port: pick it once
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
            assert p.exitcode == 0
        res = dict(out)
    assert set(res) == {0, 1}
    for ms, value in res.values():
        assert ms == pytest.approx(20.0 / 5)                    # slowest rank, per step
        assert value == pytest.approx(2 * 1000 / (4.0e-3))      # both ranks' tokens
