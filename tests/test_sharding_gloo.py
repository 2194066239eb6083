"""Multi-process (gloo, world size 2, CPU) tests of the sharded run's host
logic: batch partition, and max-over-ranks timing."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_93_b200.sharding import batch_shard, max_over_ranks


@pytest.mark.parametrize("B,world", [(8, 2), (7, 2), (3, 4), (1, 3), (0, 2)])
def test_batch_shard_partitions_exactly(B, world):
    owned = []
    for r in range(world):
        s, e = batch_shard(B, world, r)
        assert 0 <= s <= e <= B
        owned += list(range(s, e))
    assert owned == list(range(B))
    sizes = [batch_shard(B, world, r)[1] - batch_shard(B, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_batch_shard_rejects_bad_rank():
    with pytest.raises(ValueError):
        batch_shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input

        inp = make_chunk_inputs(5, 40, 2, 8, 6, torch.float32, "scalar", True, seed=21)
        s, e = batch_shard(5, world, rank)
        sl = {k: v[s:e] for k, v in inp.items()}
        o, S_T = oracle.gdr_fwd(to_numpy_input(sl["q"]), to_numpy_input(sl["k"]),
                                to_numpy_input(sl["v"]), sl["g"].numpy(), sl["beta"].numpy(),
                                sl["S0"].double().numpy(), nthreads=1)
        # gather variable-size shards on every rank
        parts = [None] * world
        dist.all_gather_object(parts, (s, e, o, S_T))
        # max over ranks of a per-rank "time"
        m = max_over_ranks([1.0 + rank, 10.0 - rank])
        if rank == 0:
            out.put((parts, m))
    finally:
        dist.destroy_process_group()


def test_sharded_run_equals_unsharded_gloo():
    import oracle
    from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts, m = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = make_chunk_inputs(5, 40, 2, 8, 6, torch.float32, "scalar", True, seed=21)
    o, S_T = oracle.gdr_fwd(to_numpy_input(inp["q"]), to_numpy_input(inp["k"]),
                            to_numpy_input(inp["v"]), inp["g"].numpy(), inp["beta"].numpy(),
                            inp["S0"].double().numpy(), nthreads=1)
    o_sh = np.concatenate([p[2] for p in sorted(parts, key=lambda x: x[0])], axis=0)
    S_sh = np.concatenate([p[3] for p in sorted(parts, key=lambda x: x[0])], axis=0)
    assert np.array_equal(o_sh, o) and np.array_equal(S_sh, S_T)
    assert m == [2.0, 10.0]


def _bwd_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input

        inp = make_chunk_inputs(5, 30, 2, 8, 8, torch.float32, "channel", True, seed=22)
        dout = torch.randn(5, 30, 2, 8, generator=torch.Generator().manual_seed(23))
        s, e = batch_shard(5, world, rank)
        sl = {k: v[s:e] for k, v in inp.items()}
        g = oracle.gdr_bwd(to_numpy_input(sl["q"]), to_numpy_input(sl["k"]),
                           to_numpy_input(sl["v"]), sl["g"].numpy(), sl["beta"].numpy(),
                           dout[s:e].double().numpy(), sl["S0"].double().numpy(),
                           gate="channel", nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (s, e, g))
        if rank == 0:
            out.put(parts)
    finally:
        dist.destroy_process_group()


def test_sharded_backward_equals_unsharded_gloo():
    """The backward shards over the batch like the forward: every (b, h) is
    independent, so per-rank gradients concatenate to the unsharded ones."""
    import oracle
    from gated_delta_rule_93_b200.inputs import make_chunk_inputs, to_numpy_input

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = make_chunk_inputs(5, 30, 2, 8, 8, torch.float32, "channel", True, seed=22)
    dout = torch.randn(5, 30, 2, 8, generator=torch.Generator().manual_seed(23))
    full = oracle.gdr_bwd(to_numpy_input(inp["q"]), to_numpy_input(inp["k"]),
                          to_numpy_input(inp["v"]), inp["g"].numpy(), inp["beta"].numpy(),
                          dout.double().numpy(), inp["S0"].double().numpy(), gate="channel",
                          nthreads=1)
    parts = sorted(parts, key=lambda x: x[0])
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS0"):
        got = np.concatenate([p[2][name] for p in parts], axis=0)
        assert np.array_equal(got, full[name]), name
