"""Multi-process host logic of the benchmark (gloo, world size 2, CPU).

Each rank decodes its own batch of independent sequences (no collective on the
data path); timings are reduced with a max over ranks and the reported value is
the whole job's throughput.  Checked here without a GPU: the shards differ, the
union of the shards' oracle outputs is what each rank computes on its own, and
the max reduction and aggregation are right.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from workloads import make_workload, preset

        spec = bench.shard_spec(preset("tiny_mixed_d64_L512"), rank, world)
        w = make_workload(spec)
        # this rank's decode step on the oracle (what the GPU computes for this shard)
        ref = oracle.decode_step(w.q.double().numpy(), w.k.double().numpy(), w.v.double().numpy(), w.offsets.tolist(),
                                 w.roles.tolist(), w.scale, idom=w.idom.numpy(),
                                 n_fac_per_seq=w.n_fac_per_seq.tolist(), sink=spec.sink, window=spec.window)
        out = np.stack([ref[(0, g)]["out"][0] for g in range(4)])
        # a rank-dependent fake timing: the slower rank sets the step time
        ms = [1.0 + rank, 2.0 + 3 * rank]
        red = bench.max_over_ranks(ms, world, torch.device("cpu"))
        gathered = [torch.zeros(4 * 64, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(out.reshape(-1)))
        q.put((rank, spec.seed, red, int(w.lengths.sum()), [g.numpy() for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_independent_batches_and_reduce_max():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    seeds = [r[1] for r in res]
    assert seeds[0] != seeds[1]                       # independent sequences per rank
    for r in res:
        assert r[2] == [2.0, 5.0]                     # element-wise max over ranks
    outs0, outs1 = res[0][4], res[1][4]
    assert np.array_equal(outs0[0], outs1[0]) and np.array_equal(outs0[1], outs1[1])
    assert not np.allclose(outs0[0], outs0[1])        # the two shards really differ

    import sys

    sys.path.insert(0, ROOT)
    import bench

    # whole-job throughput: both ranks' tokens in the slowest rank's step time
    assert bench.aggregate_throughput(res[0][3], world, 2.0) == res[0][3] * 2 / 2e-3
