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
