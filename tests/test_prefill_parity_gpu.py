"""gdn_prefill (CUDA, through the C ABI) against the fp64 oracle on the same seeded inputs.

Bound: max|y_gpu - y_oracle| / rms(y_oracle) <= 2e-2 for bf16 storage and <= 1e-4 for
fp32 storage, and the same bound on final states against rms(S_oracle).
"""
import numpy as np
import pytest

import gdn_inputs as gi
import oracle
from gdn_testutil import prefill_args, prefill_dev, rel_err, to_host_f64, tol

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_attention_recurrence_05_b200 as gdn
    return gdn


def _check(inp, lib, heads=None, with_conv=True, label="", silu=False):
    y, fin, cso = prefill_dev(inp, lib, with_conv_out=with_conv, conv_activation=int(silu))
    torch.cuda.synchronize()
    yo, fo, co = oracle.prefill(inp, heads=heads, conv_silu=silu)
    sel = slice(None) if heads is None else list(heads)
    ey = rel_err(to_host_f64(y)[:, sel], yo[:, sel])
    es = rel_err(to_host_f64(fin)[:, sel], fo[:, sel])
    t = tol(inp.dtype)
    assert ey <= t, f"{label} output error {ey:.3e} > {t}"
    assert es <= t, f"{label} final-state error {es:.3e} > {t}"
    if with_conv:
        got = to_host_f64(cso)
        ref = co if inp.conv_state is None or inp.dtype == gi.F32 else co
        assert np.array_equal(got, ref), f"{label} conv state differs"
    return ey, es


def test_workload0_tiny_fp32(lib):
    inp = gi.make_workload(0)
    _check(inp, lib, label="workload0")


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
def test_ragged_varlen_with_states(lib, dtype):
    """Chunk edges and partial chunks: lengths around 64, an empty sequence, and both
    initial states and conv states."""
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    inp = gi.make_prefill_inputs(shape, [1, 63, 64, 65, 0, 130, 200, 2], dtype, seed=77,
                                 with_initial_state=True, with_conv_state=True)
    _check(inp, lib, label=f"ragged-{dtype}")


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
@pytest.mark.parametrize("with_init", [True, False])
def test_no_tokens_at_all(lib, dtype, with_init):
    """Every sequence empty (total_tokens = 0): y has no rows, each final state is its
    initial state (zero without one) and the conv states pass through, all bit for bit."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    inp = gi.make_prefill_inputs(shape, [0, 0, 0], dtype, seed=5, with_initial_state=with_init,
                                 with_conv_state=True)
    y, fin, cso = prefill_dev(inp, lib, with_conv_out=True)
    torch.cuda.synchronize()
    yo, fo, co = oracle.prefill(inp)
    assert tuple(y.shape) == (0, 6, 128) and yo.shape == (0, 6, 128)
    assert np.array_equal(to_host_f64(fin), fo)
    assert np.array_equal(to_host_f64(cso), co)


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
def test_conv_silu(lib, dtype):
    """The optional SiLU on the ShortConv outputs (gdn_config.conv_activation = SiLU) against
    the oracle with the same option: ragged lengths, initial and conv states."""
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    inp = gi.make_prefill_inputs(shape, [1, 64, 65, 0, 200, 3], dtype, seed=87,
                                 with_initial_state=True, with_conv_state=True)
    _check(inp, lib, label=f"silu-{dtype}", silu=True)


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
def test_pages_heads_short(lib, dtype):
    shape = gi.PAGES_SHAPE
    inp = gi.make_prefill_inputs(shape, [300], dtype, seed=78)
    _check(inp, lib, label=f"h16x48-{dtype}")


def test_beta_above_one(lib):
    """beta in (1, 1.9): each token's map alpha (I - beta k k^T) still contracts, and chunk
    prep's T_beta = (I + A)^-1 diag(beta), stored as fp16, reaches entries near beta (|T_beta|
    <= 1 for beta in [0, 1]); several chunks and a partial one (gated delta rule, page
    "ARCHITECTURE PREVIEW / FIELD NOTES", section 03; the equations admit any beta).  Keys are
    the usual random ones: with identical keys and beta > 1 the chunked form loses ~6e-2 with
    TF32 operands throughout (the alternating terms of T_beta V cancel), fp16 or not."""
    shape = gi.GdnShape(n_qk_heads=1, n_v_heads=3)
    T = 150
    inp = gi.make_prefill_inputs(shape, [T], gi.BF16, seed=91)
    inp.beta = gi.quantize(np.random.default_rng(6).uniform(1.0, 1.9, (T, 3)).astype(np.float32), gi.BF16)
    _check(inp, lib, label="beta-above-one")


@pytest.mark.parametrize("dtype", [gi.BF16, gi.F32])
def test_strong_decay_resets_and_degenerate_beta(lib, dtype):
    """Gates at their edges: strong decay (alpha ~ e^-1.6 per token, so a chunk's total decay
    passes e^-80 and chunk prep forms exp(g_t - g_i) directly instead of as gamma_t / gamma_i),
    exact resets (alpha = 0, which the kernels take as e^-80), runs of alpha = 1, and beta = 0
    (no write) and beta = 1 rows; ragged lengths over several chunks, initial and conv states
    (gated delta rule, page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03)."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    lengths = [300, 129, 64]
    inp = gi.make_prefill_inputs(shape, lengths, dtype, seed=97, with_initial_state=True, with_conv_state=True)
    T = inp.total_tokens
    rng = np.random.default_rng(98)
    x = rng.standard_normal((T, 6))
    alpha = np.exp(-2.0 * np.logaddexp(0.0, x))          # strong decay
    alpha[rng.random((T, 6)) < 0.03] = 0.0                  # resets
    alpha[100:140] = 1.0                                    # no decay at all
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, 6))))
    beta[rng.random((T, 6)) < 0.1] = 0.0
    beta[rng.random((T, 6)) < 0.1] = 1.0
    inp.alpha = gi.quantize(alpha.astype(np.float32), dtype)
    inp.beta = gi.quantize(beta.astype(np.float32), dtype)
    _check(inp, lib, label=f"edge-gates-{dtype}")


@pytest.mark.parametrize("heads", [(2, 2), (2, 4), (1, 4), (2, 10)])
def test_head_ratios(lib, heads):
    """V heads per QK head other than 3: the chunk-prep pass then serves 1 or 2 V heads per CTA
    (ratios 1, 2, 4, 5), and the V -> QK head map changes; ragged lengths, initial and conv
    states."""
    shape = gi.GdnShape(n_qk_heads=heads[0], n_v_heads=heads[1])
    inp = gi.make_prefill_inputs(shape, [130, 1, 64, 200], gi.BF16, seed=83 + heads[1],
                                 with_initial_state=True, with_conv_state=True)
    _check(inp, lib, label=f"h{heads[0]}x{heads[1]}")


def test_pipelined_chunk_ranges(lib):
    """Few (sequence, head) chains and many chunks run as a pipeline over chunk ranges (the
    state carried from range to range): sequences that start, end and lie wholly inside a
    range, an empty one, initial states; with a final-state buffer, without one (the state is
    carried in the workspace) and with the final state aliasing the initial state."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    # 6,137 tokens in 5 sequences (5 x 6 heads = 30 chains): 3 ranges of 32 chunks per sequence
    inp = gi.make_prefill_inputs(shape, [2500, 0, 1400, 2200, 37], gi.BF16, seed=91,
                                 with_initial_state=True, with_conv_state=True)
    ey, es = _check(inp, lib, label="pipelined")
    from gdn_testutil import to_dev
    d = inp.dtype
    args = [to_dev(x, d) for x in (inp.q, inp.k, inp.v, inp.w_q, inp.w_k, inp.w_v, inp.alpha, inp.beta)]
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    cfg = lib.GdnConfig(2, 6)
    st = torch.from_numpy(inp.initial_state).cuda()
    cs = to_dev(inp.conv_state, d)
    y_nofin, fin_none, _ = lib.gdn_prefill(*args, cu, cfg=cfg, initial_state=st.clone(),
                                           return_final_state=False, conv_state_in=cs)
    alias = st.clone()
    y_alias, fin_alias, _ = lib.gdn_prefill(*args, cu, cfg=cfg, initial_state=alias, final_state=alias,
                                            conv_state_in=cs)
    # the conv state updated in place: every range's conv pass (on the second stream) and
    # every chain must read the old one
    cs_alias = cs.clone()
    y_csal, _, _ = lib.gdn_prefill(*args, cu, cfg=cfg, initial_state=st.clone(), conv_state_in=cs_alias,
                                   conv_state_out=cs_alias)
    torch.cuda.synchronize()
    assert fin_none is None
    yo, fo, co = oracle.prefill(inp)
    assert rel_err(to_host_f64(y_nofin), yo) <= tol(d)
    assert rel_err(to_host_f64(y_alias), yo) <= tol(d)
    assert rel_err(to_host_f64(fin_alias), fo) <= tol(d)
    assert rel_err(to_host_f64(y_csal), yo) <= tol(d)
    assert np.array_equal(to_host_f64(cs_alias), co)


def test_state_aliasing(lib):
    """final_state may alias initial_state and conv_state_out may alias conv_state_in."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    inp = gi.make_prefill_inputs(shape, [70, 5, 0], gi.BF16, seed=79, with_initial_state=True,
                                 with_conv_state=True)
    from gdn_testutil import to_dev
    d = inp.dtype
    st = torch.from_numpy(inp.initial_state).cuda()
    cs = to_dev(inp.conv_state, d)
    cfg = lib.GdnConfig(2, 6)
    y, _, _ = lib.gdn_prefill(
        to_dev(inp.q, d), to_dev(inp.k, d), to_dev(inp.v, d), to_dev(inp.w_q, d), to_dev(inp.w_k, d),
        to_dev(inp.w_v, d), to_dev(inp.alpha, d), to_dev(inp.beta, d),
        torch.from_numpy(inp.cu_seqlens).cuda(), cfg=cfg, initial_state=st, final_state=st,
        conv_state_in=cs, conv_state_out=cs)
    torch.cuda.synchronize()
    yo, fo, co = oracle.prefill(inp)
    assert rel_err(to_host_f64(y), yo) <= tol(d)
    assert rel_err(to_host_f64(st), fo) <= tol(d)
    assert np.array_equal(to_host_f64(cs), co)


def test_split_equals_whole_on_gpu(lib):
    """Prefill of [0:T1] then [T1:T] from the returned states matches the oracle on [0:T]."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    inp = gi.make_prefill_inputs(shape, [300], gi.BF16, seed=80)
    yo, fo, _ = oracle.prefill(inp)
    T1 = 137
    a = gi.make_prefill_inputs(shape, [T1], gi.BF16, seed=80)
    b = gi.make_prefill_inputs(shape, [300 - T1], gi.BF16, seed=80)
    for name in ("q", "k", "v", "alpha", "beta"):
        setattr(a, name, getattr(inp, name)[:T1])
        setattr(b, name, getattr(inp, name)[T1:])
    ya, fa, ca = prefill_dev(a, lib, with_conv_out=True)
    yb, fb, _ = lib.gdn_prefill(*[t for t in prefill_args(b, lib)], cfg=lib.GdnConfig(2, 6),
                                initial_state=fa, conv_state_in=ca)
    torch.cuda.synchronize()
    y = np.concatenate([to_host_f64(ya), to_host_f64(yb)])
    assert rel_err(y, yo) <= tol(gi.BF16)
    assert rel_err(to_host_f64(fb), fo) <= tol(gi.BF16)


def test_workload1_full_sampled_heads(lib):
    """T = 8192, 16 QK / 48 V heads, bf16: every token of five sampled V heads."""
    inp = gi.make_workload(1)
    _check(inp, lib, heads=[0, 1, 2, 25, 47], with_conv=False, label="workload1")


def test_repeated_launches_deterministic(lib):
    """The T = 8192 layer (16/48 heads, 4 chunk ranges pipelined over two streams) run 12
    times back to back on the same inputs and workspace, as a benchmark does: every run's y
    and final state bit-equal to the first run's and finite (the kernels have no data-dependent
    order, so any difference would be a race between the ranges, the streams or the roles of
    the chain; a bounded wait that gave up would show as NaN)."""
    from gdn_testutil import prefill_args
    inp = gi.make_workload(1)
    args = prefill_args(inp, lib)
    cfg = lib.GdnConfig(inp.shape.n_qk_heads, inp.shape.n_v_heads)
    T = inp.total_tokens
    ws = torch.empty(lib.prefill_workspace_size(cfg, torch.bfloat16, T, 1, T), dtype=torch.uint8, device="cuda")
    ys, fins = [], []
    for _ in range(12):
        y, fin, _ = lib.gdn_prefill(*args, cfg=cfg, workspace=ws, max_seqlen=T)
        ys.append(y)
        fins.append(fin)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(ys[0]).all()) and bool(torch.isfinite(fins[0]).all())
    for y, fin in zip(ys[1:], fins[1:]):
        assert torch.equal(y, ys[0]) and torch.equal(fin, fins[0])


@pytest.mark.slow
def test_workload2_full_sampled_heads(lib):
    """T = 262,144 (mean alpha ~ 0.98), bf16: every token of two sampled V heads."""
    inp = gi.make_workload(2)
    _check(inp, lib, heads=[4, 46], with_conv=False, label="workload2")


@pytest.mark.slow
def test_workload4_varlen_prefix_states(lib):
    """32 packed sequences (log-uniform 1K..64K) with nonzero initial states: the states of
    the sampled (sequence, V head) pairs are the oracle's final states of a seeded 2048-token
    prefill through the same layer; other pairs start from zero and are not compared."""
    inp = gi.make_workload(4)
    n = inp.n_seqs
    heads = [3, 30]
    warm = gi.warmup_prefill_inputs(4, range(n))
    _, wf, wc = oracle.prefill(warm, heads=heads)
    init = np.zeros((n, 48, 128, 128), np.float32)
    init[:, heads] = wf[:, heads].astype(np.float32)
    inp.initial_state = init
    inp.conv_state = gi.quantize(wc.astype(np.float32), gi.BF16)
    _check(inp, lib, heads=heads, with_conv=False, label="workload4")


def test_bf16_output(lib):
    """out_dtype = bf16: same bound plus each entry's own bf16 rounding."""
    from gdn_testutil import rel_err_bf16_out, to_dev
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    inp = gi.make_prefill_inputs(shape, [200, 65], gi.BF16, seed=81, with_initial_state=True)
    y, fin, _ = lib.gdn_prefill(*prefill_args(inp, lib), cfg=lib.GdnConfig(4, 12),
                                initial_state=torch.from_numpy(inp.initial_state).cuda(),
                                out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert y.dtype == torch.bfloat16
    yo, fo, _ = oracle.prefill(inp)
    assert rel_err_bf16_out(to_host_f64(y), yo) <= tol(gi.BF16)
    assert rel_err(to_host_f64(fin), fo) <= tol(gi.BF16)


def test_context_parallel_spans(lib):
    """One sequence in 3 spans through libgdn (span maps M, B from two prefills each, prefix
    combination, re-run from the true entering state): y and the final state match the oracle
    over the whole sequence (initial state and conv state given)."""
    from gdn_testutil import to_dev
    from linear_attention_recurrence_05_b200.context_parallel import cp_prefill_spans
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    inp = gi.make_prefill_inputs(shape, [700], gi.BF16, seed=97, with_initial_state=True,
                                 with_conv_state=True)
    d = inp.dtype
    full = [to_dev(x, d) for x in (inp.q, inp.k, inp.v, inp.alpha, inp.beta)]
    w = [to_dev(x, d) for x in (inp.w_q, inp.w_k, inp.w_v)]
    bounds = [0, 250, 253, 700]
    spans = [[x[a:b] for x in full] for a, b in zip(bounds[:-1], bounds[1:])]
    ys, fin = cp_prefill_spans(spans, w, cfg=lib.GdnConfig(2, 6),
                               initial_state=torch.from_numpy(inp.initial_state[0]).cuda(),
                               conv_state=to_dev(inp.conv_state[0], d))
    torch.cuda.synchronize()
    yo, fo, _ = oracle.prefill(inp)
    assert rel_err(to_host_f64(torch.cat(ys)), yo) <= tol(d)
    assert rel_err(to_host_f64(fin), fo[0]) <= tol(d)


def _trace_count(lib, fn, kernel):
    tr = lib.LaunchTrace(capacity=4096)
    with tr:
        out = fn()
    torch.cuda.synchronize()
    return out, sum(1 for n, _ in tr.records() if n == kernel)


@pytest.mark.parametrize("with_final", [True, False])
def test_short_ranges_from_small_workspace(lib, with_final):
    """A workspace smaller than the preferred one makes the chunk ranges shorter: this ragged
    problem (an empty sequence, sequences shorter than a chunk, initial and conv states) then
    runs as 11 ranges of one chunk per sequence, its states carried in the final-state buffer
    or in the workspace.  Same bound against the oracle, and bit for bit the default run (one
    range over every chunk)."""
    from gdn_testutil import to_dev
    shape = gi.GdnShape(n_qk_heads=4, n_v_heads=12)
    inp = gi.make_prefill_inputs(shape, [1, 700, 64, 0, 500, 3], gi.BF16, seed=77,
                                 with_initial_state=True, with_conv_state=True)
    d = inp.dtype
    cfg = lib.GdnConfig(4, 12)
    args = prefill_args(inp, lib)
    st = torch.from_numpy(inp.initial_state).cuda()
    cs = to_dev(inp.conv_state, d)
    T, n = inp.total_tokens, inp.n_seqs
    pref = lib.prefill_workspace_size(cfg, torch.bfloat16, T, n, 700)
    slot = 4 * (65536 + 32768) + 12 * (32768 + 3 * 16384 + 640)
    small = 2 * n * slot + n * 12 * 65536 + (1 << 16)   # two buffers of one chunk per sequence
    assert small < pref
    ws = torch.empty(small, dtype=torch.uint8, device="cuda")
    (y, fin, _), launches = _trace_count(lib, lambda: lib.gdn_prefill(
        *args, cfg=cfg, initial_state=st, conv_state_in=cs, workspace=ws, max_seqlen=700,
        return_final_state=with_final), "prefill_tc")
    assert launches == 11
    y_ref, fin_ref, _ = lib.gdn_prefill(*args, cfg=cfg, initial_state=st, conv_state_in=cs, max_seqlen=700)
    torch.cuda.synchronize()
    yo, fo, _ = oracle.prefill(inp)
    assert rel_err(to_host_f64(y), yo) <= tol(d)
    assert np.array_equal(to_host_f64(y), to_host_f64(y_ref))
    if with_final:
        assert rel_err(to_host_f64(fin), fo) <= tol(d)
        assert np.array_equal(to_host_f64(fin), to_host_f64(fin_ref))


def test_sequence_longer_than_max_seqlen(lib):
    """A sequence longer than the max_seqlen bound: with ranges of one chunk per sequence
    (small workspace) the tokens past the bound's last range and that sequence's final state
    are NaN; the other sequence, within the bound, is computed as usual."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6)
    inp = gi.make_prefill_inputs(shape, [300, 1000], gi.BF16, seed=85, with_initial_state=True)
    cfg = lib.GdnConfig(2, 6)
    slot = 2 * (65536 + 32768) + 6 * (32768 + 3 * 16384 + 640)
    ws = torch.empty(2 * 2 * slot + 2 * 6 * 65536 + (1 << 14), dtype=torch.uint8, device="cuda")
    y, fin, _ = lib.gdn_prefill(*prefill_args(inp, lib), cfg=cfg, workspace=ws, max_seqlen=300,
                                initial_state=torch.from_numpy(inp.initial_state).cuda())
    torch.cuda.synchronize()
    yo, fo, _ = oracle.prefill(inp)
    yh, fh = to_host_f64(y), to_host_f64(fin)
    assert rel_err(yh[:300], yo[:300]) <= tol(gi.BF16)
    assert rel_err(fh[0], fo[0]) <= tol(gi.BF16)
    covered = 300 + 5 * 64          # the bound's 5 chunks of sequence 1
    assert rel_err(yh[300:covered], yo[300:covered]) <= tol(gi.BF16)
    assert np.isnan(yh[covered:]).all() and np.isnan(fh[1]).all()
