"""The N > 1 path on CPU: two gloo ranks, each with its own replica of a
workload (no data exchange), timing reduced as the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_long_sequence_attn_b200 import replicas
from sparse_long_sequence_attn_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ws, rk, _ = replicas.dist_env()
        assert (ws, rk) == (world, rank)
        w = wl.WORKLOADS["tiny"]
        q, k, v = wl.make_inputs(w, seed=replicas.replica_seed(w.seed, rank))
        import oracle

        out, lse = oracle.dilated_attn_fp64(q, k, v, w.patterns, w.causal)
        np.save(os.path.join(outdir, f"out{rank}.npy"), out)
        fake_time = 1.0 + rank * 0.5
        mx = replicas.max_over_ranks(fake_time)
        np.save(os.path.join(outdir, f"max{rank}.npy"), np.array([mx]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_replicas(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    o0 = np.load(tmp_path / "out0.npy")
    o1 = np.load(tmp_path / "out1.npy")
    assert o0.shape == o1.shape and not np.allclose(o0, o1)  # different replicas
    # rank 0's replica is exactly the single-process workload
    import oracle

    w = wl.WORKLOADS["tiny"]
    ref, _ = oracle.dilated_attn_fp64(*wl.make_inputs(w), w.patterns, w.causal)
    assert np.array_equal(o0, ref)
    for r in range(world):
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == 1.5  # max over ranks


def test_weak_scaling_rate_and_single_process_identity():
    assert replicas.max_over_ranks(3.25) == 3.25
    assert replicas.weak_scaling_rate(32768, 4, 0.5) == pytest.approx(262144.0)
    assert replicas.replica_seed(10, 0) == 10 and replicas.replica_seed(10, 1) != 10
