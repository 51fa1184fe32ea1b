"""Multi-rank paths on CPU with the gloo backend (world sizes 2 and 4): bench.py's replicas (the
step time is the max over ranks and the throughput aggregates all ranks' tokens; weak scaling,
no data-path collective), the exchange of the context-parallel In-Place forward, and what a
rank sees when a peer fails before the exchange (an error from the collective within the
process group's timeout, not a hang)."""
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
@pytest.mark.parametrize("world", [2, 4])
def test_replica_timing_is_max_over_ranks_and_tokens_add_up(world):
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
    assert set(res) == set(range(world))
    for ms, value in res.values():
        assert ms == pytest.approx(10.0 * world / 5)                       # slowest rank, per step
        assert value == pytest.approx(world * 1000 / (ms * 1e-3))          # every rank's tokens



class _OracleOps:
    """CPU stand-ins of the library calls of inplace_cp_fwd, written on the oracle, so the
    exchange (all-gather and the exclusive prefix) is tested without a GPU."""

    @staticmethod
    def delta(T, d_ff, d_model, lr, Z, Vhat, dW, workspace, workspace_bytes):
        import numpy as np
        import torch
        import oracle
        W0 = np.zeros((d_model, d_ff))
        # one chunk from zero: lr Vhat^T Z (float64 arrays straight to the oracle)
        _, WF = oracle.inplace_fwd(Z.numpy(), Vhat.numpy(), W0, C=T, lr=lr)
        dW.copy_(torch.from_numpy(WF))

    @staticmethod
    def add(dst, src):
        dst.add_(src)

    @staticmethod
    def fwd(T, d_ff, d_model, C, lr, Z, Vhat, W, O, workspace, workspace_bytes):
        import torch
        import oracle
        o, wf = oracle.inplace_fwd(Z.numpy(), Vhat.numpy(), W.numpy(), C=C, lr=lr)
        O.copy_(torch.from_numpy(o))
        W.copy_(torch.from_numpy(wf))


def _cp_rank(rank, world, port, out):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import weight_sequence_layers_b200 as ttt
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(70)
        T, d_ff, d_model, C, lr = 8 * world, 6, 5, 4, 0.1
        Z = rng.standard_normal((T, d_ff))
        Vh = rng.standard_normal((T, d_model))
        W0 = rng.standard_normal((d_model, d_ff))
        n = T // world
        sl = slice(rank * n, (rank + 1) * n)
        W = torch.from_numpy(W0.copy())
        O = torch.empty((n, d_model), dtype=torch.float64)
        ttt.inplace_cp_fwd(n, d_ff, d_model, C, lr, torch.from_numpy(Z[sl].copy()),
                           torch.from_numpy(Vh[sl].copy()), W, O, None, 0, ops=_OracleOps)
        out[rank] = (O.numpy().tolist(), W.numpy().tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
@pytest.mark.parametrize("world", [2, 4])
def test_inplace_context_parallel_scan_equals_one_sequence(world):
    import numpy as np

    import oracle
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_cp_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
            assert p.exitcode == 0
        res = dict(out)
    rng = np.random.default_rng(70)
    T, d_ff, d_model, C, lr = 8 * world, 6, 5, 4, 0.1
    Z = rng.standard_normal((T, d_ff))
    Vh = rng.standard_normal((T, d_model))
    W0 = rng.standard_normal((d_model, d_ff))
    O, WF = oracle.inplace_fwd(Z, Vh, W0, C=C, lr=lr)
    got = np.concatenate([np.array(res[r][0]) for r in range(world)])
    np.testing.assert_allclose(got, O, atol=1e-12)
    np.testing.assert_allclose(np.array(res[world - 1][1]), WF, atol=1e-12)


def _cp_rank_with_failed_peer(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import weight_sequence_layers_b200 as ttt
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == world - 1:
        os._exit(3)  # this rank fails between steps, before the exchange
    n, d_ff, d_model, C = 4, 6, 5, 4
    W = torch.zeros((d_model, d_ff), dtype=torch.float64)
    O = torch.empty((n, d_model), dtype=torch.float64)
    try:
        ttt.inplace_cp_fwd(n, d_ff, d_model, C, 0.1, torch.ones((n, d_ff), dtype=torch.float64),
                           torch.ones((n, d_model), dtype=torch.float64), W, O, None, 0,
                           ops=_OracleOps)
        out[rank] = "returned"
    except Exception as e:  # the collective reports the lost peer
        out[rank] = "raised " + type(e).__name__
    os._exit(0)


@pytest.mark.timeout(120)
def test_context_parallel_exchange_fails_loudly_when_a_peer_is_gone():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_cp_rank_with_failed_peer, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 3]
    assert res.get(0, "").startswith("raised"), res
