"""gdn_output_gate (CUDA, through the C ABI) against the fp64 output-tail oracle."""
import numpy as np
import pytest

import gdn_inputs as gi
from gdn_testutil import to_dev, to_host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_attention_recurrence_05_b200 as gdn
    return gdn


def _inputs(T, Hv, ydt, zdt, seed):
    rng = np.random.default_rng(seed)
    y = gi.quantize((0.3 * rng.standard_normal((T, Hv, 128))).astype(np.float32), ydt)
    z = gi.quantize((2.0 * rng.standard_normal((T, Hv, 128))).astype(np.float32), zdt)
    w = (1.0 + 0.2 * rng.standard_normal(128)).astype(np.float32)
    return y, z, w


@pytest.mark.parametrize("ydt,zdt,odt", [(gi.F32, gi.BF16, gi.F32), (gi.BF16, gi.BF16, gi.BF16),
                                         (gi.F32, gi.F32, gi.BF16), (gi.BF16, gi.F32, gi.F32)])
def test_output_gate_matches_oracle(lib, ydt, zdt, odt):
    from oracle.output_gate import output_gate
    y, z, w = _inputs(1000, 6, ydt, zdt, 11)
    yd, zd = to_dev(y, ydt), to_dev(z, zdt)
    out = lib.gdn_output_gate(yd, zd, torch.from_numpy(w).cuda(), eps=1e-6,
                              out_dtype=torch.bfloat16 if odt == gi.BF16 else torch.float32)
    torch.cuda.synchronize()
    ref = output_gate(gi.stored_to_f64(y, ydt), gi.stored_to_f64(z, zdt), w, 1e-6)
    got = to_host_f64(out)
    rms = np.sqrt(np.mean(ref ** 2))
    if odt == gi.BF16:
        # the rounding of a bf16 output is relative (half an ulp: 2^-9), and gated values reach
        # ~20 x their rms, so the bound is per element: 2^-8 |ref| (rounding plus fp32 math)
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * rms)
    else:
        assert np.max(np.abs(got - ref)) / rms <= 1e-5


def test_output_gate_in_place_and_zero_rows(lib):
    """out = y in place; an all-zero row gives zeros (eps keeps the scale finite)."""
    from oracle.output_gate import output_gate
    y, z, w = _inputs(257, 48, gi.F32, gi.BF16, 12)
    y[5] = 0.0
    yd = to_dev(y, gi.F32)
    lib.gdn_output_gate(yd, to_dev(z, gi.BF16), torch.from_numpy(w).cuda(), eps=1e-6, out=yd)
    torch.cuda.synchronize()
    ref = output_gate(y, gi.stored_to_f64(z, gi.BF16), w, 1e-6)
    got = to_host_f64(yd)
    assert np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref ** 2)) <= 1e-5
    assert np.all(got[5] == 0)


@pytest.mark.parametrize("dtype,zdt,odt,lengths", [
    (gi.BF16, gi.BF16, gi.F32, [1, 63, 64, 65, 0, 130, 2]),
    (gi.BF16, gi.F32, gi.BF16, [200, 77]),
    (gi.BF16, gi.BF16, gi.F32, [3000]),          # several chunk ranges
    (gi.F32, gi.BF16, gi.F32, [130, 64, 5]),     # fp32 path: y in out, then the tail in place
])
def test_prefill_gated_matches_oracle(lib, dtype, zdt, odt, lengths):
    """gdn_prefill_gated (the tail fused into the chain's store of y) against
    oracle/output_gate.py applied to the oracle's y, and against libgdn's unfused composition
    (gdn_prefill, then gdn_output_gate on its fp32 y)."""
    import oracle
    from oracle.output_gate import output_gate
    from gdn_testutil import prefill_args, rel_err, tol
    shape = gi.GdnShape(n_qk_heads=2 if lengths == [3000] else 4, n_v_heads=6 if lengths == [3000] else 12)
    inp = gi.make_prefill_inputs(shape, lengths, dtype, seed=211, with_initial_state=True,
                                 with_conv_state=True)
    T, Hv = inp.total_tokens, shape.n_v_heads
    rng = np.random.default_rng(212)
    z = gi.quantize((2.0 * rng.standard_normal((T, Hv, 128))).astype(np.float32), zdt)
    w = (1.0 + 0.2 * rng.standard_normal(128)).astype(np.float32)
    cfg = lib.GdnConfig(shape.n_qk_heads, Hv)
    args = prefill_args(inp, lib)
    st = torch.from_numpy(inp.initial_state).cuda()
    cs = to_dev(inp.conv_state, dtype)
    zd, wd = to_dev(z, zdt), torch.from_numpy(w).cuda()
    odt_t = torch.bfloat16 if odt == gi.BF16 else torch.float32
    o, fin, _ = lib.gdn_prefill(*args, cfg=cfg, initial_state=st, conv_state_in=cs, out_dtype=odt_t,
                                gate=(zd, wd, 1e-6), max_seqlen=max(lengths))
    y, _, _ = lib.gdn_prefill(*args, cfg=cfg, initial_state=st, conv_state_in=cs, max_seqlen=max(lengths))
    o2 = lib.gdn_output_gate(y, zd, wd, eps=1e-6, out_dtype=torch.float32)
    torch.cuda.synchronize()
    got = to_host_f64(o)
    yo, fo, _ = oracle.prefill(inp)
    ref = output_gate(yo, gi.stored_to_f64(z, zdt), w, 1e-6)
    # y is within tol * rms(y) of the oracle per element; the row normalisation divides that
    # by the row's own rms, and the gate scales it by |w SiLU(z)| (x 3 for the norm's own change).
    # The fused path takes SiLU from the hardware tanh, SiLU(z) = z/2 (1 + tanh(z/2)), whose
    # relative error bound 2^-10.987 leaves |z| 2^-12 on SiLU: 2^-11 |z| |w| |y / rms(y row)|
    # more (2x margin), the only term left where SiLU(z) -> 0.
    t = tol(dtype)
    zf = gi.stored_to_f64(z, zdt)
    row_rms = np.sqrt(np.mean(yo ** 2, axis=-1, keepdims=True))
    gate = np.abs(w * zf / (1.0 + np.exp(-zf)))
    silu_term = 2.0 ** -11 * np.abs(zf) * np.abs(w) * np.abs(yo) / row_rms
    bound = (3 * t * np.sqrt(np.mean(yo ** 2)) / row_rms * gate + 1e-6 * np.sqrt(np.mean(ref ** 2))
             + silu_term * (1 + 3 * t))
    if odt == gi.BF16:
        bound = bound + 2.0 ** -8 * np.abs(ref)
    assert np.all(np.abs(got - ref) <= bound)
    assert rel_err(to_host_f64(fin), fo) <= t
    # the fused tail against the unfused composition on the same y: fp32 arithmetic apart from
    # the fused path's tanh-based SiLU (bound above, from the GPU's own y)
    o2h = to_host_f64(o2)
    yh = to_host_f64(y)
    yn = yh / np.sqrt(np.mean(yh ** 2, axis=-1, keepdims=True) + 1e-6)
    b2 = 2.0 ** -11 * np.abs(zf) * np.abs(w) * np.abs(yn) + 1e-5 * np.sqrt(np.mean(o2h ** 2))
    if odt == gi.BF16:
        b2 = b2 + 2.0 ** -8 * np.abs(o2h)
    assert np.all(np.abs(got - o2h) <= b2)
