"""Sharding by sequence over ranks (host planning, CPU): token balance of the partition, and
a 2-rank gloo run in which each rank prefills only its sequences (the oracle playing the
prefill) and the gathered outputs equal the whole batch's, sequence by sequence."""
import os
import socket

import numpy as np
import pytest

import gdn_inputs as gi
from linear_attention_recurrence_05_b200.partition import balance_sequences, rank_pack, split_rows


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_balance_is_a_partition_within_the_bound(world):
    lengths = [int(x) for x in gi.varlen_lengths(4)]      # 32 log-uniform lengths, 1K..64K
    parts = balance_sequences(lengths, world)
    assert sorted(i for p in parts for i in p) == list(range(len(lengths)))
    assert all(p == sorted(p) for p in parts)
    loads = [sum(lengths[i] for i in p) for p in parts]
    assert max(loads) <= sum(lengths) / world + max(lengths)
    # no better assignment of the heaviest rank's smallest sequence to the lightest rank exists
    # that the greedy rule would have missed: moving it would not lower the maximum
    if world > 1:
        hi, lo = int(np.argmax(loads)), int(np.argmin(loads))
        s = min(lengths[i] for i in parts[hi])
        assert max(loads[hi] - s, loads[lo] + s) >= max(loads) or len(parts[hi]) == 1


def test_balance_small_cases():
    assert balance_sequences([5, 1, 1, 1, 1, 1], 2) == [[0], [1, 2, 3, 4, 5]]
    assert balance_sequences([3, 3, 2, 2, 2], 2) == [[0, 2, 4], [1, 3]]
    assert balance_sequences([], 3) == [[], [], []]


def test_split_rows_and_pack():
    assert [list(r) for r in split_rows(10, 3)] == [[0, 1, 2, 3], [4, 5, 6], [7, 8, 9]]
    assert sum(len(r) for r in split_rows(256, 8)) == 256
    spans, cu = rank_pack([4, 0, 3, 5], [0, 2, 3])
    assert spans == [(0, 4), (4, 7), (7, 12)] and cu == [0, 4, 7, 12]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPE = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
LENGTHS = [90, 0, 17, 130, 64, 3, 71]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = gi.make_prefill_inputs(SHAPE, LENGTHS, gi.BF16, seed=61, with_initial_state=True,
                                     with_conv_state=True)
        mine = balance_sequences(LENGTHS, world)[rank]
        spans, cu = rank_pack(LENGTHS, mine)
        rows = np.concatenate([np.arange(a, b) for a, b in spans]) if spans else np.zeros(0, int)
        sub = gi.PrefillInputs(SHAPE, inp.dtype, inp.q[rows], inp.k[rows], inp.v[rows], inp.w_q, inp.w_k,
                               inp.w_v, inp.alpha[rows], inp.beta[rows], np.asarray(cu, np.int32),
                               inp.initial_state[mine], inp.conv_state[mine])
        y, fin, _ = oracle.prefill(sub, n_threads=1)
        got = [None] * world
        dist.all_gather_object(got, (mine, [y[a:b] for a, b in zip(cu[:-1], cu[1:])], fin))
        if rank == 0:
            per_seq = {}
            for idx, ys, fs in got:
                for j, i in enumerate(idx):
                    per_seq[i] = (ys[j], fs[j])
            np.save(os.path.join(out_dir, "y.npy"), np.concatenate([per_seq[i][0] for i in range(len(LENGTHS))]))
            np.save(os.path.join(out_dir, "f.npy"), np.stack([per_seq[i][1] for i in range(len(LENGTHS))]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_equal_whole_batch(repo_tmp):
    import torch.multiprocessing as mp
    import oracle
    mp.start_processes(_rank_main, args=(2, _free_port(), repo_tmp), nprocs=2, start_method="spawn")
    inp = gi.make_prefill_inputs(SHAPE, LENGTHS, gi.BF16, seed=61, with_initial_state=True,
                                 with_conv_state=True)
    yo, fo, _ = oracle.prefill(inp)
    assert np.array_equal(np.load(os.path.join(repo_tmp, "y.npy")), yo)
    assert np.array_equal(np.load(os.path.join(repo_tmp, "f.npy")), fo)
