"""Multi-process host logic on CPU (gloo, world size 2): batch sharding needs no exchange in the
forward (the oracle on each rank's rows reproduces the whole batch), the backward's parameter
gradients are the all-reduced sums of the ranks' partial gradients, and timing reduces to the
max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_23_b200.dist import (allreduce_bc_grads, allreduce_param_grads, barrier,
                                                 max_over_ranks, seq_split_scan_fwd, shard_channels,
                                                 shard_rows)


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


BWD_SHAPE = dict(batch=5, dim=6, seqlen=37, dstate=4)


def _bwd_inputs():
    from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload
    w = workload("tiny_f32", **BWD_SHAPE)
    return {k: to_f64(v) for k, v in make_inputs(w, seed=5, with_h0=True, with_dout=True).items()}


def _bwd(oracle, x, b0, b1):
    sl = lambda k: x[k][b0:b1]
    return oracle.scan_bwd(sl("u"), sl("delta"), x["A"], sl("B"), sl("C"), sl("dout"), D=x["D"],
                           z=sl("z"), dt_bias=x["dt_bias"], h0=sl("h0"), nthreads=1)


def _bwd_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        x = _bwd_inputs()
        b0, b1 = shard_rows(BWD_SHAPE["batch"], world, rank)
        g = _bwd(oracle, x, b0, b1)
        part = {k: torch.from_numpy(np.ascontiguousarray(g[k])) for k in ("dA", "dD", "ddt_bias")}
        before = {k: v.clone() for k, v in part.items()}
        allreduce_param_grads(part)
        rows = {k: g[k] for k in ("du", "ddelta", "dz", "dB", "dC", "dh0")}
        q.put((rank, (b0, b1), {k: v.numpy() for k, v in part.items()},
               {k: v.numpy() for k, v in before.items()}, rows))
    finally:
        dist.destroy_process_group()


def test_two_ranks_backward_param_grads_allreduced():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda r: r[0])
    import oracle
    x = _bwd_inputs()
    full = _bwd(oracle, x, 0, BWD_SHAPE["batch"])
    for k in ("dA", "dD", "ddt_bias"):
        # every rank holds the whole-batch gradient, and it is the sum of the two partials
        for r in res:
            np.testing.assert_allclose(r[2][k], full[k], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(res[0][2][k], res[1][2][k])
        np.testing.assert_array_equal(res[0][2][k], res[0][3][k] + res[1][3][k])
        # a rank's partial alone is not the whole-batch gradient
        assert not np.allclose(res[0][3][k], full[k])
    # the row gradients need no exchange: each rank's rows are the whole batch's rows
    for k in ("du", "ddelta", "dz", "dB", "dC", "dh0"):
        got = np.concatenate([r[4][k] for r in res], 0)
        np.testing.assert_array_equal(got, full[k])


def test_shard_channels_partition():
    for dim in (0, 5, 16, 40, 80, 2048):
        for world in (1, 2, 3, 8):
            for align in (1, 16, 64):
                spans = [shard_channels(dim, world, r, align) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == dim
                for (b0, e0), (b1, _) in zip(spans, spans[1:]):
                    assert e0 == b1
                for b, e in spans:   # every span starts on a block boundary
                    assert b % align == 0 or b == dim
                blocks = [-(-(e - b) // align) for b, e in spans]
                assert max(blocks) - min(blocks) <= 1
    with pytest.raises(ValueError):
        shard_channels(16, 2, 2)


CH_SHAPE = dict(batch=3, dim=10, seqlen=29, dstate=4)


def _ch_inputs():
    from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload
    w = workload("tiny_f32", **CH_SHAPE)
    return {k: to_f64(v) for k, v in make_inputs(w, seed=6, with_h0=True, with_dout=True).items()}


def _bwd_channels(oracle, x, d0, d1):
    c = lambda k: x[k][:, d0:d1]
    return oracle.scan_bwd(c("u"), c("delta"), x["A"][d0:d1], x["B"], x["C"], c("dout"),
                           D=x["D"][d0:d1], z=c("z"), dt_bias=x["dt_bias"][d0:d1], h0=c("h0"),
                           nthreads=1)


def _bwd_channels_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        x = _ch_inputs()
        d0, d1 = shard_channels(CH_SHAPE["dim"], world, rank, align=4)
        g = _bwd_channels(oracle, x, d0, d1)
        bc = {k: torch.from_numpy(np.ascontiguousarray(g[k])) for k in ("dB", "dC")}
        before = {k: v.clone() for k, v in bc.items()}
        allreduce_bc_grads(bc)
        own = {k: g[k] for k in ("du", "ddelta", "dz", "dh0", "dA", "dD", "ddt_bias")}
        q.put((rank, (d0, d1), {k: v.numpy() for k, v in bc.items()},
               {k: v.numpy() for k, v in before.items()}, own))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_channel_sharded_backward_allreduces_dB_dC(world):
    """Channels split over gloo ranks (the fp64 oracle as each rank's backward): dB, dC summed
    over the ranks equal the whole layer's; every per-channel gradient needs no exchange."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bwd_channels_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda r: r[0])
    import oracle
    x = _ch_inputs()
    full = _bwd_channels(oracle, x, 0, CH_SHAPE["dim"])
    for k in ("dB", "dC"):
        for r in res:
            np.testing.assert_allclose(r[2][k], full[k], rtol=1e-12, atol=1e-12)
        assert not np.allclose(res[0][3][k], full[k])   # one rank's channels alone are not
    for k in ("du", "ddelta", "dz", "dh0", "dA", "dD", "ddt_bias"):
        got = np.concatenate([r[4][k] for r in res], 1 if k in ("du", "ddelta", "dz", "dh0") else 0)
        np.testing.assert_array_equal(got, full[k])


def test_allreduce_bc_grads_sums_16_bit_in_f32_without_group_is_identity():
    g = {"dB": torch.ones(2, 3, dtype=torch.bfloat16), "dC": None}
    out = allreduce_bc_grads(g)
    assert out is g and torch.equal(g["dB"], torch.ones(2, 3, dtype=torch.bfloat16))


def test_allreduce_param_grads_without_group_is_identity():
    g = {"dA": torch.ones(3, 2), "dD": None}
    out = allreduce_param_grads(g)
    assert out is g and torch.equal(g["dA"], torch.ones(3, 2)) and g["dD"] is None


# ------------------------------------------------------------------ sequence split
SEQ_SHAPE = dict(batch=2, dim=5, seqlen=53, dstate=4)
# one decay rate per channel with the larger state of the Mamba-2 setting
SEQ_SHAPE_SCALAR = dict(batch=1, dim=3, seqlen=41, dstate=32)


def _seq_inputs(scalar=False):
    from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload
    w = workload("tiny_f32", **(SEQ_SHAPE_SCALAR if scalar else SEQ_SHAPE))
    return {k: to_f64(v) for k, v in make_inputs(w, seed=8, with_h0=True, scalar_a=scalar).items()}


def _full_a(A, N):
    """A as [dim][N] for the oracle: a per-channel rate [dim] repeated over the states."""
    return np.repeat(A[:, None], N, axis=1) if A.ndim == 1 else A


def _oracle_ops():
    """Stand-ins for the library's summary, chain and scan calls, built on the fp64 oracle, so
    that the exchange and composition logic runs on CPU ranks (A [dim][N], or [dim] for one
    decay rate per channel)."""
    import oracle

    def summary(u, delta, A, B, C, dt_bias, softplus):
        Af = _full_a(A.numpy(), B.shape[-2])
        hend = oracle.scan_fwd(u.numpy(), delta.numpy(), Af, B.numpy(), C.numpy(),
                               dt_bias=dt_bias.numpy(), delta_softplus=softplus, nthreads=1)["hL"]
        v = delta.numpy() + dt_bias.numpy()[None, :, None]
        dsum = (np.logaddexp(0.0, v) if softplus else v).sum(axis=2)
        return torch.from_numpy(hend), torch.from_numpy(dsum)

    def chain(hend_all, dsum_all, A, h0):
        h = np.zeros(hend_all.shape[1:]) if h0 is None else h0.numpy().copy()
        hin = np.empty(hend_all.shape)
        for r in range(hend_all.shape[0]):
            hin[r] = h
            Af = _full_a(A.numpy(), hend_all.shape[-1])
            h = np.exp(Af[None] * dsum_all[r].numpy()[..., None]) * h + hend_all[r].numpy()
        return torch.from_numpy(hin)

    def scan(u, delta, A, B, C, D, z, dt_bias, softplus, h0, return_final_state):
        r = oracle.scan_fwd(u.numpy(), delta.numpy(), _full_a(A.numpy(), B.shape[-2]), B.numpy(),
                            C.numpy(), D=D.numpy(), z=z.numpy(), dt_bias=dt_bias.numpy(),
                            delta_softplus=softplus, h0=h0.numpy(), nthreads=1)
        return r["out"], r["hL"]

    return {"summary": summary, "chain": chain, "scan": scan}


def _seq_worker(rank, world, port, q, scalar=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from selective_state_space_23_b200.dist import seq_split_scan_fwd
        x = _seq_inputs(scalar)
        L = (SEQ_SHAPE_SCALAR if scalar else SEQ_SHAPE)["seqlen"]
        t0, t1 = shard_rows(L, world, rank)   # this rank's time segment
        seg = lambda k: torch.from_numpy(np.ascontiguousarray(x[k][..., t0:t1]))
        full = lambda k: torch.from_numpy(x[k])
        out, hL = seq_split_scan_fwd(seg("u"), seg("delta"), full("A"), seg("B"), seg("C"),
                                     D=full("D"), z=seg("z"), dt_bias=full("dt_bias"),
                                     h0=full("h0"), return_final_state=True, scalar_a=scalar,
                                     ops=_oracle_ops())
        q.put((rank, (t0, t1), out, hL))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,scalar", [(2, False), (3, False), (3, True)])
def test_sequence_split_over_ranks_matches_full_sequence(world, scalar):
    """Each rank scans its time segment from the state that the all-gathered segment summaries
    chain to; the concatenated outputs and the last rank's final state are the full sequence's
    (also with one decay rate per channel and 32 states)."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_seq_worker, args=(r, world, port, q, scalar))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda r: r[0])
    import oracle
    x = _seq_inputs(scalar)
    x["A"] = _full_a(x["A"], x["B"].shape[-2])
    full = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                           dt_bias=x["dt_bias"], h0=x["h0"], nthreads=1)
    assert res[0][1][0] == 0 and res[-1][1][1] == (SEQ_SHAPE_SCALAR if scalar else SEQ_SHAPE)["seqlen"]
    out = np.concatenate([r[2] for r in res], axis=2)
    np.testing.assert_allclose(out, full["out"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[-1][3], full["hL"], rtol=1e-10, atol=1e-12)
    # the first segment alone, without the chain, is exact; later ones need their entering state
    first = oracle.scan_fwd(x["u"][..., :res[1][1][0]], x["delta"][..., :res[1][1][0]], x["A"],
                            x["B"][..., :res[1][1][0]], x["C"][..., :res[1][1][0]], D=x["D"],
                            z=x["z"][..., :res[1][1][0]], dt_bias=x["dt_bias"], h0=x["h0"],
                            nthreads=1)
    np.testing.assert_array_equal(res[0][2], first["out"])
