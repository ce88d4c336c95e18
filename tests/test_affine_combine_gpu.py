"""gdn_affine_combine (CUDA, through the C ABI) against the fp64 oracle of the span-state
combination: S_in[0] = S0, S_in[p+1] = M[p] S_in[p] + B[p] per V head."""
import numpy as np
import pytest

from gdn_testutil import rel_err

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_attention_recurrence_05_b200 as gdn
    return gdn


def _maps(rng, P, Hv, d=128):
    # products of per-token maps alpha (I - beta k k^T) are contractions: random orthogonal
    # matrices scaled below 1 stand in for them; offsets of state size
    q, _ = np.linalg.qr(rng.standard_normal((P, Hv, d, d)))
    M = (0.6 + 0.3 * rng.random((P, Hv, 1, 1))) * q
    B = 0.2 * rng.standard_normal((P, Hv, d, d))
    return M.astype(np.float32), B.astype(np.float32)


@pytest.mark.parametrize("P,Hv,with_s0", [(1, 48, True), (3, 6, False), (7, 48, True), (0, 4, True)])
def test_affine_combine_matches_oracle(lib, P, Hv, with_s0):
    from oracle.affine import affine_prefix
    rng = np.random.default_rng(100 + P)
    M, B = _maps(rng, P, Hv)
    S0 = (0.3 * rng.standard_normal((Hv, 128, 128))).astype(np.float32) if with_s0 else None
    dev = lambda a: None if a is None else torch.from_numpy(a).cuda()
    out = lib.affine_combine(dev(M), dev(B), dev(S0), cfg=lib.GdnConfig(1, Hv))
    torch.cuda.synchronize()
    ref = affine_prefix(M, B, S0)
    got = out.cpu().double().numpy()
    assert got.shape == ref.shape
    assert np.array_equal(got[0], ref[0])          # S0 (or zero) copied exactly
    for p in range(1, P + 1):
        assert rel_err(got[p], ref[p]) <= 1e-5, p
