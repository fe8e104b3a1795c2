"""Replica (data-parallel) host logic with two gloo ranks on the CPU.

The layer shards as replicas: each rank runs its own copy on its own tokens and
only the timing is reduced (max over ranks).  Checked here without a GPU:
the bench's per-rank inputs (one set of weights, distinct token batches), the max-over-ranks reduction the bench uses,
and that per-rank shards of a batch reproduce the full batch (tokens are
independent, so replicas need no exchange).
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import synth
        # the bench's per-rank inputs: the same weights on every rank, distinct tokens
        wl, copies = bench.build_inputs("tiny_fp32", rank, 1)
        (layers, x), = copies
        gathered = [torch.zeros(wl.T, wl.H) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(x.astype(np.float32)))
        wr = [torch.zeros(wl.E, wl.H) for _ in range(world)]
        dist.all_gather(wr, torch.from_numpy(layers[0].w_router.astype(np.float32)))
        # the slowest rank sets the time
        t = bench.max_over_ranks(10.0 + rank, dist)
        # shards of one batch, routed on their own rank, equal the full batch
        inp = synth.make("tiny_fp32")
        L = inp.layers[0]
        o = oracle.Oracle(oracle.LayerWeights(**L.arrays(), top_k=wl.k))
        shard = np.array_split(np.arange(inp.x.shape[0]), world)[rank]
        y_shard, _, _, _ = o.forward(inp.x[shard])
        parts = [torch.zeros(len(s), wl.H, dtype=torch.float64)
                 for s in np.array_split(np.arange(inp.x.shape[0]), world)]
        dist.all_gather(parts, torch.from_numpy(y_shard))
        if rank == 0:
            y_full, _, _, _ = o.forward(inp.x)
            out.put(dict(distinct=not torch.equal(gathered[0], gathered[1]), t=t,
                         same_weights=torch.equal(wr[0], wr[1]),
                         same=bool(np.array_equal(torch.cat(parts).numpy(), y_full))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=240)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert res["distinct"] and res["same_weights"]
    assert res["t"] == 11.0
    assert res["same"]
