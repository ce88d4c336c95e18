"""gdn_decode_step (CUDA, through the C ABI) against the fp64 oracle, step by step."""
import numpy as np
import pytest

import gdn_inputs as gi
import oracle
from gdn_testutil import rel_err, to_dev, to_host_f64, tol

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_attention_recurrence_05_b200 as gdn
    return gdn


def _weights_dev(w, dtype):
    return [to_dev(x, dtype) for x in w]


def _run_steps(lib, shape, dtype, dec, w, state, conv, slots=None, n_rows=None, act=0):
    """Run every step of ``dec`` on the GPU; returns per-step outputs [steps, B, Hv, dv]."""
    cfg = lib.GdnConfig(shape.n_qk_heads, shape.n_v_heads, conv_activation=act)
    wd = _weights_dev(w, dtype)
    ys = []
    for s in range(dec.q.shape[0]):
        y = lib.gdn_decode_step(to_dev(dec.q[s], dtype), to_dev(dec.k[s], dtype),
                                to_dev(dec.v[s], dtype), *wd, to_dev(dec.alpha[s], dtype),
                                to_dev(dec.beta[s], dtype), state, conv, state_slots=slots, cfg=cfg)
        ys.append(to_host_f64(y))
    torch.cuda.synchronize()
    return np.stack(ys)


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
def test_small_batch_every_step(lib, dtype):
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    B, steps = 5, 24
    w = gi.make_conv_weights(shape, 91)
    dec = gi.make_decode_inputs(shape, B, steps, dtype, seed=92)
    rng = np.random.default_rng(93)
    S0 = (0.05 * rng.standard_normal((B, 12, 128, 128))).astype(np.float32)
    cs0 = gi.quantize(rng.standard_normal((B, 3, shape.channels)).astype(np.float32), dtype)
    state = torch.from_numpy(S0.copy()).cuda()
    conv = to_dev(cs0, dtype)
    ys = _run_steps(lib, shape, dtype, dec, w, state, conv)
    yo, So, co = oracle.decode_steps(shape, dtype, dec, w, S0, cs0)
    assert rel_err(ys, yo) <= tol(dtype)
    assert rel_err(to_host_f64(state), So) <= tol(dtype)
    assert np.array_equal(to_host_f64(conv), co)


def test_state_slots_and_skipped_rows(lib):
    """Rows map to state rows through state_slots; a slot of -1 leaves every state row
    untouched and writes zeros for that row."""
    dtype = gi.BF16
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    B, R = 4, 7
    slots = np.array([5, -1, 0, 3], np.int32)
    w = gi.make_conv_weights(shape, 94)
    dec = gi.make_decode_inputs(shape, B, 3, dtype, seed=95)
    rng = np.random.default_rng(96)
    S0 = (0.05 * rng.standard_normal((R, 6, 128, 128))).astype(np.float32)
    cs0 = gi.quantize(rng.standard_normal((R, 3, shape.channels)).astype(np.float32), dtype)
    state = torch.from_numpy(S0.copy()).cuda()
    conv = to_dev(cs0, dtype)
    ys = _run_steps(lib, shape, dtype, dec, w, state, conv,
                    slots=torch.from_numpy(slots).cuda())
    live = [0, 2, 3]
    # the oracle sees the live rows with their slots' starting states
    S_live = S0[slots[live]]
    cs_live = cs0[slots[live]]
    sub = gi.DecodeInputs(*(getattr(dec, f)[:, live] for f in ("q", "k", "v", "alpha", "beta")))
    yo, So, co = oracle.decode_steps(shape, dtype, sub, w, S_live, cs_live)
    assert rel_err(ys[:, live], yo) <= tol(dtype)
    assert np.all(ys[:, 1] == 0.0)
    St = to_host_f64(state)
    assert rel_err(St[slots[live]], So) <= tol(dtype)
    untouched = [r for r in range(R) if r not in slots[live]]
    assert np.array_equal(St[untouched], S0[untouched].astype(np.float64))
    ct = to_host_f64(conv)
    assert np.array_equal(ct[slots[live]], co)
    assert np.array_equal(ct[untouched], gi.stored_to_f64(cs0[untouched], dtype))


def test_decode_without_conv_state(lib):
    """A null conv state means zero history and nothing written."""
    dtype = gi.F32
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    w = gi.make_conv_weights(shape, 97)
    dec = gi.make_decode_inputs(shape, 3, 1, dtype, seed=98)
    state = torch.zeros((3, 6, 128, 128), device="cuda")
    ys = _run_steps(lib, shape, dtype, dec, w, state, None)
    yo, So, _ = oracle.decode_steps(shape, dtype, dec, w, np.zeros((3, 6, 128, 128)),
                                    np.zeros((3, 3, shape.channels), np.float32))
    assert rel_err(ys, yo) <= tol(dtype)
    assert rel_err(to_host_f64(state), So) <= tol(dtype)


@pytest.mark.slow
def test_workload3_full_batch_sampled(lib):
    """256 rows x 1024 steps at the pages' shape.  All rows run on the GPU; rows
    [0, 77, 200, 255] x V heads [0, 1, 2, 23, 47] are compared at every step and at the
    end.  Their starting states are the oracle's final states of the seeded 4096-token
    warm-up prefill (other pairs start from zero and are not compared)."""
    w3 = gi.WORKLOADS[3]
    shape, dtype, B, steps = w3["shape"], w3["dtype"], w3["batch"], w3["steps"]
    rows = [0, 77, 200, 255]
    heads = [0, 1, 2, 23, 47]
    w = gi.workload_weights(3)
    warm = gi.warmup_prefill_inputs(3, rows)
    _, wf, wc = oracle.prefill(warm, heads=heads)
    S0 = np.zeros((B, 48, 128, 128), np.float32)
    for i, r in enumerate(rows):
        S0[r, heads] = wf[i, heads].astype(np.float32)
    cs0 = np.zeros((B, 3, shape.channels), np.uint16)
    cs0[rows] = gi.quantize(wc.astype(np.float32), dtype)
    state = torch.from_numpy(S0).cuda()
    conv = to_dev(cs0, dtype)
    cfg = lib.GdnConfig(16, 48)
    wd = _weights_dev(w, dtype)
    ys_gpu = torch.empty((steps, len(rows), 48, 128), dtype=torch.float32, device="cuda")
    rows_t = torch.tensor(rows, device="cuda")
    sub_parts = []
    for s in range(steps):
        d = gi.decode_workload_step(s)
        y = lib.gdn_decode_step(to_dev(d.q[0], dtype), to_dev(d.k[0], dtype), to_dev(d.v[0], dtype),
                                *wd, to_dev(d.alpha[0], dtype), to_dev(d.beta[0], dtype), state,
                                conv, cfg=cfg)
        ys_gpu[s] = y.index_select(0, rows_t).float()
        sub_parts.append(gi.DecodeInputs(*(getattr(d, f)[:, rows]
                                           for f in ("q", "k", "v", "alpha", "beta"))))
    torch.cuda.synchronize()
    sub = gi.DecodeInputs(*(np.concatenate([getattr(p, f) for p in sub_parts])
                            for f in ("q", "k", "v", "alpha", "beta")))
    yo, So, _ = oracle.decode_steps(shape, dtype, sub, w, S0[rows], cs0[rows], heads=heads)
    yg = ys_gpu.double().cpu().numpy()
    assert rel_err(yg[:, :, heads], yo[:, :, heads]) <= tol(dtype)
    St = state[rows_t].double().cpu().numpy()
    assert rel_err(St[:, heads], So[:, heads]) <= tol(dtype)


def _multi_inputs(dec, dtype):
    """DecodeInputs are [steps, B, ...]; the multi-token call takes [B, n, ...]."""
    return [to_dev(np.ascontiguousarray(np.swapaxes(getattr(dec, f), 0, 1)), dtype)
            for f in ("q", "k", "v", "alpha", "beta")]


@pytest.mark.parametrize("dtype,n", [(gi.BF16, 1), (gi.BF16, 3), (gi.BF16, 4), (gi.BF16, 8), (gi.F32, 4)])
def test_multi_token_with_checkpoints(lib, dtype, n):
    """gdn_decode_multi over n tokens per row equals n single-token oracle steps: y of every
    token, the state and conv state after the last one, and the checkpoints after each."""
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    B = 5
    w = gi.make_conv_weights(shape, 101)
    dec = gi.make_decode_inputs(shape, B, n, dtype, seed=102 + n)
    rng = np.random.default_rng(103)
    S0 = (0.05 * rng.standard_normal((B, 12, 128, 128))).astype(np.float32)
    cs0 = gi.quantize(rng.standard_normal((B, 3, shape.channels)).astype(np.float32), dtype)
    state = torch.from_numpy(S0.copy()).cuda()
    conv = to_dev(cs0, dtype)
    ck = torch.full((B, n, 12, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    cck = torch.zeros((B, n, 3, shape.channels), dtype=conv.dtype, device="cuda")
    q, k, v, a, b = _multi_inputs(dec, dtype)
    y = lib.gdn_decode_multi(q, k, v, *_weights_dev(w, dtype), a, b, state, conv, state_ckpt=ck, conv_ckpt=cck,
                             cfg=lib.GdnConfig(4, 12))
    torch.cuda.synchronize()
    yo, So, co = oracle.decode_steps(shape, dtype, dec, w, S0, cs0)
    assert rel_err(np.swapaxes(to_host_f64(y), 0, 1), yo) <= tol(dtype)
    assert rel_err(to_host_f64(state), So) <= tol(dtype)
    assert np.array_equal(to_host_f64(conv), co)
    for j in range(n):   # checkpoint j = the oracle after j + 1 tokens
        _, Sj, cj = oracle.decode_steps(shape, dtype, dec, w, S0, cs0, steps=j + 1)
        assert rel_err(to_host_f64(ck[:, j]), Sj) <= tol(dtype)
        assert np.array_equal(to_host_f64(cck[:, j]), cj)


def test_multi_token_slots_and_skipped_rows(lib):
    """state_slots map rows to state rows; a slot of -1 writes zero outputs and touches no
    state row; no conv state (zero history) and no checkpoints."""
    dtype = gi.BF16
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    B, R, n = 4, 6, 3
    slots = np.array([4, -1, 1, 2], np.int32)
    w = gi.make_conv_weights(shape, 104)
    dec = gi.make_decode_inputs(shape, B, n, dtype, seed=105)
    rng = np.random.default_rng(106)
    S0 = (0.05 * rng.standard_normal((R, 6, 128, 128))).astype(np.float32)
    state = torch.from_numpy(S0.copy()).cuda()
    q, k, v, a, b = _multi_inputs(dec, dtype)
    y = to_host_f64(lib.gdn_decode_multi(q, k, v, *_weights_dev(w, dtype), a, b, state, None,
                                         state_slots=torch.from_numpy(slots).cuda(), cfg=lib.GdnConfig(2, 6)))
    torch.cuda.synchronize()
    live = [0, 2, 3]
    sub = gi.DecodeInputs(*(getattr(dec, f)[:, live] for f in ("q", "k", "v", "alpha", "beta")))
    cs_zero = np.zeros((len(live), 3, shape.channels), np.float32)
    yo, So, _ = oracle.decode_steps(shape, dtype, sub, w, S0[slots[live]], cs_zero)
    assert rel_err(np.swapaxes(y[live], 0, 1), yo) <= tol(dtype)
    assert np.all(y[1] == 0)
    Sg = to_host_f64(state)
    assert rel_err(Sg[slots[live]], So) <= tol(dtype)
    untouched = [r for r in range(R) if r not in slots[live]]
    assert np.array_equal(Sg[untouched], S0[untouched].astype(np.float64))


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
def test_conv_silu_single_and_multi_token(lib, dtype):
    """The optional SiLU on the ShortConv outputs in both decode kernels, against oracle steps
    with the same option."""
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    B, steps = 3, 4
    w = gi.make_conv_weights(shape, 111)
    dec = gi.make_decode_inputs(shape, B, steps, dtype, seed=112)
    rng = np.random.default_rng(113)
    S0 = (0.05 * rng.standard_normal((B, 12, 128, 128))).astype(np.float32)
    cs0 = gi.quantize(rng.standard_normal((B, 3, shape.channels)).astype(np.float32), dtype)
    yo, So, co = oracle.decode_steps(shape, dtype, dec, w, S0, cs0, conv_silu=True)
    state = torch.from_numpy(S0.copy()).cuda()
    conv = to_dev(cs0, dtype)
    ys = _run_steps(lib, shape, dtype, dec, w, state, conv, act=1)
    assert rel_err(ys, yo) <= tol(dtype)
    assert rel_err(to_host_f64(state), So) <= tol(dtype)
    assert np.array_equal(to_host_f64(conv), co)
    state = torch.from_numpy(S0.copy()).cuda()
    conv = to_dev(cs0, dtype)
    q, k, v, a, b = _multi_inputs(dec, dtype)
    y = lib.gdn_decode_multi(q, k, v, *_weights_dev(w, dtype), a, b, state, conv,
                             cfg=lib.GdnConfig(4, 12, conv_activation=1))
    torch.cuda.synchronize()
    assert rel_err(np.swapaxes(to_host_f64(y), 0, 1), yo) <= tol(dtype)
    assert rel_err(to_host_f64(state), So) <= tol(dtype)
