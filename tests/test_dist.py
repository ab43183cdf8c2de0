"""The multi-GPU path is data parallel with no exchange on the data path
(replicas): every rank runs its own block of tokens through its own copy of
the layer.  These CPU tests run that decomposition with world size 2 over
gloo: each rank computes its shard with the oracle, the shards are gathered,
and the result must equal the single-process batch bit for bit (tokens are
independent in a MoE layer).  They also check the max-over-ranks reduction
that bench.py applies to device-timed durations."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, n_tok, q):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import synth
        from tests.helpers import oracle_expert

        cfg = synth.config("tiny")
        x = synth.tokens(cfg, n_tok)
        shard = list(bench.rank_token_shard(n_tok, rank, world))
        experts = {e: oracle_expert(cfg, 0, e) for e in range(cfg["n_experts"])}
        shared = [oracle_expert(cfg, 0, 0, shared=True)]
        out, idx, _ = oracle.moe_layer(cfg, synth.router_w(cfg), synth.bias(cfg), experts, shared, x[shard])
        # gather variable-size shards: pad to the largest shard
        m = (n_tok + world - 1) // world
        buf = np.zeros((m, cfg["hidden"]), np.float32)
        buf[:len(shard)] = out
        parts = [torch.zeros(m, cfg["hidden"]) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(buf))
        t = bench.max_over_ranks(1.5 + rank)
        if rank == 0:
            full = np.concatenate([parts[r].numpy()[:len(bench.rank_token_shard(n_tok, r, world))]
                                   for r in range(world)])
            q.put((full, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_tok", [8, 7])
def test_replicas_equal_single_batch(ora, syn, n_tok):
    import oracle
    from tests.helpers import oracle_expert
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n_tok, q)) for r in range(world)]
    for p in procs:
        p.start()
    full, t = q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    cfg = syn.config("tiny")
    x = syn.tokens(cfg, n_tok)
    experts = {e: oracle_expert(cfg, 0, e) for e in range(cfg["n_experts"])}
    shared = [oracle_expert(cfg, 0, 0, shared=True)]
    want, _, _ = oracle.moe_layer(cfg, syn.router_w(cfg), syn.bias(cfg), experts, shared, x)
    assert np.array_equal(full, want)
    assert t == 2.5  # max over ranks of 1.5 + rank


def test_token_shards_partition_the_batch():
    import bench
    for n in (0, 1, 7, 8, 2048):
        for w in (1, 2, 3, 8):
            ids = [i for r in range(w) for i in bench.rank_token_shard(n, r, w)]
            assert ids == list(range(n))
    assert bench.max_over_ranks(3.25) == 3.25  # no process group: identity
