"""Multi-process host logic on CPU (gloo, world size 2): batch sharding needs no exchange (the
oracle on each rank's rows reproduces the whole batch), and timing reduces to the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_23_b200.dist import barrier, max_over_ranks, shard_rows


def test_shard_rows_partition():
    for total in (0, 1, 7, 8, 9, 256):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (b0, e0), (b1, _) in zip(spans, spans[1:]):
                assert e0 == b1
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(8, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload
        w = workload("tiny_f32", batch=5, dim=6, seqlen=40, dstate=4)
        x = {k: to_f64(v) for k, v in make_inputs(w, seed=3, with_h0=True).items()}
        b0, b1 = shard_rows(w.batch, world, rank)
        sl = lambda k: x[k][b0:b1]
        mine = oracle.scan_fwd(sl("u"), sl("delta"), x["A"], sl("B"), sl("C"), D=x["D"], z=sl("z"),
                               dt_bias=x["dt_bias"], h0=sl("h0"), nthreads=1)
        gathered = [None] * world
        dist.all_gather_object(gathered, (b0, b1, mine["out"], mine["hL"]))
        barrier()
        t = max_over_ranks(1.5 + rank)
        q.put((rank, t, gathered if rank == 0 else None))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_without_exchange_and_time_is_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [2.5, 2.5]          # max over ranks, seen by every rank
    gathered = res[0][2]
    import oracle
    from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload
    w = workload("tiny_f32", batch=5, dim=6, seqlen=40, dstate=4)
    x = {k: to_f64(v) for k, v in make_inputs(w, seed=3, with_h0=True).items()}
    full = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                           dt_bias=x["dt_bias"], h0=x["h0"], nthreads=1)
    out = np.concatenate([g[2] for g in gathered], 0)
    hL = np.concatenate([g[3] for g in gathered], 0)
    assert [g[:2] for g in gathered] == [(0, 3), (3, 5)]
    np.testing.assert_array_equal(out, full["out"])
    np.testing.assert_array_equal(hL, full["hL"])


def test_max_over_ranks_single_process():
    assert max_over_ranks(3.25) == 3.25
