"""The seeded input recipe shared by the oracle and the CUDA path (gdn_inputs.py): its bf16
rounding, its distributions and the workload table, checked against library routines and
the stated configurations."""
import math

import numpy as np
import pytest

import gdn_inputs as gi

torch = pytest.importorskip("torch")


def test_bf16_rounding_matches_torch_and_ties_go_to_even():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 100000),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3.3895314e38, 3.4e38, -3.4e38,
                  np.inf, -np.inf, 0.0, -0.0, 1e-40, -1e-40], dtype=np.float32)]).astype(np.float32)
    ours = gi.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # halfway cases: 1 + 2^-8 lies between 1 (even) and 1 + 2^-7 (odd); 1 + 3 * 2^-8 between
    # 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert gi.bf16_bits_to_f32(gi.f32_to_bf16_bits(np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8]))).tolist() == \
        [1.0, 1 + 2 ** -6]
    assert gi.f32_to_bf16_bits(np.float32([np.nan]))[0] == 0x7FC0
    # widening is exact
    assert np.array_equal(gi.stored_to_f64(ours, gi.BF16), gi.bf16_bits_to_f32(ours).astype(np.float64))


def _alpha_mean(c):
    from scipy import integrate
    f = lambda x: math.exp(-c * math.log1p(math.exp(x))) * math.exp(-x * x / 2) / math.sqrt(2 * math.pi)
    return integrate.quad(f, -40, 40)[0]


@pytest.mark.parametrize("c,stated", [(0.1, 0.924), (0.025, 0.980)])
def test_alpha_distribution(c, stated):
    """alpha = exp(-c softplus(x)), x ~ N(0, 1): the sample mean agrees with the integral,
    which is the mean the workload table states (0.924, and 0.98 for the long context)."""
    exact = _alpha_mean(c)
    assert abs(exact - stated) < 5e-4
    a = gi.draw_alpha(np.random.default_rng(11), 1_000_000, c)
    assert 0.0 < a.min() and a.max() <= 1.0
    assert abs(a.mean() - exact) < 6 * a.std() / 1000.0


def test_beta_distribution():
    b = gi.draw_beta(np.random.default_rng(12), 1_000_000)
    assert 0.0 < b.min() and b.max() < 1.0
    assert abs(b.mean() - 0.5) < 6 * b.std() / 1000.0
    # sigmoid of a standard normal: P(beta < sigmoid(1)) = Phi(1)
    assert abs(np.mean(b < 1 / (1 + math.exp(-1))) - 0.841345) < 3e-3


def test_workload_table_matches_the_configurations():
    W = gi.WORKLOADS
    assert (W[0]["dtype"], W[0]["lengths"], W[0]["shape"].n_qk_heads, W[0]["shape"].n_v_heads) == (gi.F32, [512], 2, 6)
    for i in (1, 2, 3, 4):
        assert (W[i]["shape"].n_qk_heads, W[i]["shape"].n_v_heads, W[i]["dtype"]) == (16, 48, gi.BF16)
    assert W[1]["lengths"] == [8192] and W[1]["c"] == 0.1
    assert W[2]["lengths"] == [262144] and W[2]["c"] == 0.025
    assert (W[3]["batch"], W[3]["steps"], W[3]["warm_tokens"]) == (256, 1024, 4096)
    assert (W[4]["n_seqs"], W[4]["len_lo"], W[4]["len_hi"], W[4]["warm_tokens"]) == (32, 1024, 65536, 2048)
    L = gi.varlen_lengths(4)
    assert len(L) == 32 and L.min() >= 1024 and L.max() <= 65536
    assert int(L.sum()) == 602887
    # log-uniform: the logs spread over [ln 1024, ln 65536]; their mean is near the midpoint
    assert abs(np.log(L).mean() - (math.log(1024) + math.log(65536)) / 2) < 4 * 1.2 / math.sqrt(32)


def test_layer_workload_draws():
    inp = gi.make_workload(1)
    assert inp.q.shape == (8192, 16, 128) and inp.v.shape == (8192, 48, 128)
    assert inp.q.dtype == np.uint16 and inp.alpha.shape == (8192, 48)
    for name in ("q", "k", "v"):
        x = gi.stored_to_f64(getattr(inp, name), gi.BF16)
        assert abs(x.mean()) < 5 / math.sqrt(x.size) and abs(x.std() - 1.0) < 2e-3
    for w in (inp.w_q, inp.w_k, inp.w_v):
        assert w.dtype == np.float32 and w.shape[1] == 4 and abs(w.std() - 0.5) < 0.02
    assert np.array_equal(inp.cu_seqlens, [0, 8192])
    # one spawned stream per tensor: q and k differ, and the same seed repeats exactly
    assert not np.array_equal(inp.q, inp.k)
    again = gi.make_workload(1)
    assert all(np.array_equal(getattr(inp, f), getattr(again, f)) for f in ("q", "k", "v", "alpha", "beta", "w_v"))


def test_decode_steps_have_their_own_streams():
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    a0 = gi.make_decode_step(shape, 4, 0, gi.BF16, 7)
    a1 = gi.make_decode_step(shape, 4, 1, gi.BF16, 7)
    both = gi.make_decode_inputs(shape, 4, 2, gi.BF16, 7)
    assert not np.array_equal(a0.q, a1.q)
    assert np.array_equal(both.q[0], a0.q[0]) and np.array_equal(both.v[1], a1.v[0])
    # any subset of warm-up rows draws the same rows
    sub = gi.warmup_prefill_inputs(4, [5])
    pair = gi.warmup_prefill_inputs(4, [2, 5])
    assert np.array_equal(sub.q, pair.q[2048:])
