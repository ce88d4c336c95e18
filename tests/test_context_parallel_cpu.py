"""Context-parallel prefill (spans of one sequence) on the CPU: the oracle plays the prefill,
so the span maps, their prefix combination and the conv history carried between spans are
checked exactly (fp64) against the oracle over the whole sequence; ranks are gloo processes."""
import os
import socket

import numpy as np
import pytest
import torch

import gdn_inputs as gi
import oracle
from linear_attention_recurrence_05_b200 import GdnConfig
from linear_attention_recurrence_05_b200.context_parallel import cp_prefill, cp_prefill_spans

SHAPE = gi.GdnShape(n_qk_heads=2, n_v_heads=6)


def oracle_prefill(q, k, v, w_q, w_k, w_v, alpha, beta, cu, *, cfg, initial_state=None,
                   conv_state_in=None, **_):
    """The fp64 oracle behind gdn_prefill's signature (torch tensors in and out, fp64)."""
    n = lambda t: None if t is None else t.detach().cpu().double().numpy()
    y, fin, cso = oracle.gdn_prefill_f64(n(q), n(k), n(v), n(w_q), n(w_k), n(w_v), n(alpha), n(beta),
                                         cu.cpu().numpy(), n_qk_heads=cfg.n_qk_heads,
                                         n_v_heads=cfg.n_v_heads, initial_state=n(initial_state),
                                         conv_state=n(conv_state_in), n_threads=1)
    return torch.from_numpy(y), torch.from_numpy(fin), torch.from_numpy(cso)


def oracle_combine(M, B, S0):
    """The fp64 oracle behind affine_combine's signature."""
    from oracle.affine import affine_prefix
    return torch.from_numpy(affine_prefix(M.double().numpy(), B.double().numpy(), S0.double().numpy()))


def _case(T, seed):
    inp = gi.make_prefill_inputs(SHAPE, [T], gi.F32, seed=seed, with_initial_state=True,
                                 with_conv_state=True)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float()
    full = [t(inp.q), t(inp.k), t(inp.v), t(inp.alpha), t(inp.beta)]
    w = [t(inp.w_q), t(inp.w_k), t(inp.w_v)]
    return inp, full, w


def _split(full, bounds):
    return [[x[a:b] for x in full] for a, b in zip(bounds[:-1], bounds[1:])]


@pytest.mark.parametrize("bounds", [[0, 100, 230], [0, 5, 64, 65, 230], [0, 3, 230]])
def test_spans_equal_whole_sequence(bounds):
    inp, full, w = _case(230, 51)
    cfg = GdnConfig(2, 6)
    ys, fin = cp_prefill_spans(_split(full, bounds), w, cfg=cfg,
                               initial_state=torch.from_numpy(inp.initial_state[0]).float(),
                               conv_state=torch.from_numpy(inp.conv_state[0]).float(), prefill=oracle_prefill,
                               combine=oracle_combine)
    yo, fo, _ = oracle.prefill(inp)
    np.testing.assert_allclose(torch.cat(ys).numpy(), yo, rtol=0, atol=1e-9 * np.abs(yo).max())
    np.testing.assert_allclose(fin.numpy(), fo[0], rtol=0, atol=1e-9 * np.abs(fo).max())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, bounds, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp, full, w = _case(230, 51)
        q, k, v, a, b = _split(full, bounds)[rank]
        y, fin = cp_prefill(q, k, v, w, a, b, cfg=GdnConfig(2, 6), prefill=oracle_prefill, combine=oracle_combine,
                            initial_state=torch.from_numpy(inp.initial_state[0]).float() if rank == 0 else None,
                            conv_state=torch.from_numpy(inp.conv_state[0]).float() if rank == 0 else None)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
        np.save(os.path.join(out_dir, f"f{rank}.npy"), fin.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [[0, 120, 230], [0, 40, 41 + 60, 230]])
def test_ranks_equal_whole_sequence(repo_tmp, bounds):
    """One span per gloo rank; the last rank's final state is the sequence's."""
    import torch.multiprocessing as mp
    world = len(bounds) - 1
    mp.start_processes(_rank_main, args=(world, _free_port(), bounds, repo_tmp), nprocs=world,
                       start_method="spawn")
    inp, _, _ = _case(230, 51)
    yo, fo, _ = oracle.prefill(inp)
    y = np.concatenate([np.load(os.path.join(repo_tmp, f"y{r}.npy")) for r in range(world)])
    np.testing.assert_allclose(y, yo, rtol=0, atol=1e-9 * np.abs(yo).max())
    np.testing.assert_allclose(np.load(os.path.join(repo_tmp, f"f{world - 1}.npy")), fo[0], rtol=0,
                               atol=1e-9 * np.abs(fo).max())


def test_affine_prefix_closed_forms():
    """The combination's own pins: identity maps add up the offsets; zero offsets multiply the
    maps in span order (M[p] ... M[0] S0), which a transposed product would not give."""
    from oracle.affine import affine_prefix
    rng = np.random.default_rng(3)
    P, H, d = 4, 2, 5
    B = rng.standard_normal((P, H, d, d))
    S0 = rng.standard_normal((H, d, d))
    I = np.broadcast_to(np.eye(d), (P, H, d, d))
    S = affine_prefix(I, B, S0)
    for p in range(P + 1):
        np.testing.assert_allclose(S[p], S0 + B[:p].sum(axis=0), atol=1e-12)
    M = rng.standard_normal((P, H, d, d))
    S = affine_prefix(M, np.zeros_like(B), S0)
    for h in range(H):
        X = S0[h]
        for p in range(P):
            X = M[p, h] @ X
            np.testing.assert_allclose(S[p + 1, h], X, atol=1e-10)
    assert np.array_equal(affine_prefix(M[:0], B[:0], S0), S0[None])
