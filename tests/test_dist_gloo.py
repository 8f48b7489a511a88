"""Multi-process host logic on the CPU (gloo, world size 2): the max over ranks
used for timings, and channel sharding of the operator's rows -- each rank
computes its channel range alone (here with the oracle) and the shards
reassemble to the unsharded result with no exchange on the data path."""
import os
import socket
import tempfile

import numpy as np


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import oracle
    from fft_long_convolution_02_b200 import dist as hd
    from fft_long_convolution_02_b200 import inputs as I
    hd.init("gloo", 60.0)
    m = hd.max_over_ranks(1.5 * (rank + 1))
    p = I.WORKLOADS["tiny"].with_(B=2, C=7, L=256, seed=7001)
    c0, c1 = hd.channel_shard(p.C, world, rank)
    rows = np.array([b * p.C + c for b in range(p.B) for c in range(c0, c1)], dtype=np.int64)
    data = I.make_all(p)
    y = (oracle.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], B=p.B, C=p.C, order=p.order,
                              shape=p.shape, rows=rows, method=1) if len(rows) else np.zeros((0, p.L)))
    np.save(os.path.join(outdir, f"r{rank}.npy"), y.reshape(p.B, c1 - c0, p.L))
    np.save(os.path.join(outdir, f"m{rank}.npy"), np.array([m, c0, c1]))
    hd.barrier()
    dist.destroy_process_group()


def test_channel_shard_partitions():
    from fft_long_convolution_02_b200 import dist as hd
    for C in (1, 2, 7, 256, 768):
        for world in (1, 2, 3, 8):
            ranges = [hd.channel_shard(C, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == C
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_shard_and_reduce():
    import torch.multiprocessing as mp

    import oracle
    from fft_long_convolution_02_b200 import inputs as I
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d), nprocs=world, join=True, start_method="spawn")
        meta = [np.load(os.path.join(d, f"m{r}.npy")) for r in range(world)]
        assert all(m[0] == 1.5 * world for m in meta)          # max over ranks seen by every rank
        shards = [np.load(os.path.join(d, f"r{r}.npy")) for r in range(world)]
    p = I.WORKLOADS["tiny"].with_(B=2, C=7, L=256, seed=7001)
    y_sharded = np.concatenate(shards, axis=1)
    data = I.make_all(p)
    y_full = oracle.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], B=p.B, C=p.C, order=p.order,
                                  shape=p.shape, method=1).reshape(p.B, p.C, p.L)
    assert np.array_equal(y_sharded, y_full)
