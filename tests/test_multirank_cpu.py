"""The N > 1 host logic of bench.py over gloo ranks on the CPU: ranks read their identity
from the torchrun environment, the step time is the maximum over ranks, barriers pass."""
import os
import socket

import numpy as np
import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    d = bench.Dist(torch, backend="gloo", device="cpu").init()
    try:
        d.barrier()
        m = d.max(1.5 + rank * 2.25)          # every rank reports a different time
        d.barrier()
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array([d.rank, d.world, m]))
    finally:
        d.close()


@pytest.mark.parametrize("world", [2, 3])
def test_dist_max_over_ranks(repo_tmp, world):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(world, _free_port(), repo_tmp), nprocs=world,
                       start_method="spawn")
    for r in range(world):
        rank, w, m = np.load(os.path.join(repo_tmp, f"r{r}.npy"))
        assert (rank, w) == (r, world)
        assert m == 1.5 + (world - 1) * 2.25
