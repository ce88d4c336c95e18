"""Pins of the fp64 oracle against what the page and the mathematics fix (CPU only).

The pages print no worked numeric example of the Gated DeltaNet, so the oracle
(four-equation form, page "ARCHITECTURE PREVIEW / FIELD NOTES" section 03) is held
to independent statements of the same definition:
  * the page's expanded one-step form, S_t = alpha(I - beta k k^T) S + beta k v^T,
    evaluated exactly in rationals (golden fixture) and in numpy;
  * brute-force transition products on tiny inputs;
  * closed forms: beta = 0 is pure decay; alpha = beta = 1 with orthonormal keys
    recalls every written value exactly; a repeated identical write changes nothing;
  * the chunked (WY/UT) form that the CUDA path implements equals the sequential one;
  * split == whole, packed == separate, T one-token steps == one T-token call;
  * the ShortConv equals numpy's convolution, and L2 normalisation gives unit norm;
  * V heads of one QK group with identical inputs give identical outputs.
A final test plants each mistake of a list into the oracle (compile-time switch)
and checks that these pins catch it.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import gdn_inputs as gi
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------- helpers
def identity_weights(channels, W=4):
    w = np.zeros((channels, W))
    w[:, W - 1] = 1.0
    return w


def unit_rows(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def run_core(Q, K, V, a, b, S0=None, mutant=0):
    """Oracle on one (QK head, V head) pair with an identity conv and eps = 0,
    so that q^ = Q and k^ = K exactly when Q, K have unit rows.  Q,K [T,dk], V [T,dv]."""
    T, dk = K.shape
    dv = V.shape[1]
    y, fin, _ = oracle.gdn_prefill_f64(
        Q[:, None, :], K[:, None, :], V[:, None, :], identity_weights(dk), identity_weights(dk),
        identity_weights(dv), np.asarray(a, float)[:, None], np.asarray(b, float)[:, None],
        np.array([0, T], np.int32), n_qk_heads=1, n_v_heads=1,
        initial_state=None if S0 is None else S0[None, None], l2_eps=0.0, mutant=mutant)
    return y[:, 0, :], fin[0, 0]


def one_step_np(Q, K, V, a, b, S0):
    """The page's expanded one-step form, coded on its own with an explicit d_k x d_k matrix."""
    dk = K.shape[1]
    S = S0.copy()
    Y = []
    for t in range(K.shape[0]):
        M = a[t] * (np.eye(dk) - b[t] * np.outer(K[t], K[t]))
        S = M @ S + b[t] * np.outer(K[t], V[t])
        Y.append(S.T @ Q[t])
    return np.array(Y), S


def transition_brute(Q, K, V, a, b, S0):
    """S_t = P_t...P_1 S_0 + sum_i P_t...P_{i+1} beta_i k_i v_i^T with P_s = a_s(I - b_s k_s k_s^T),
    each S_t rebuilt from scratch from the products (no recurrence on S)."""
    T, dk = K.shape
    P = [a[s] * (np.eye(dk) - b[s] * np.outer(K[s], K[s])) for s in range(T)]

    def prod(lo, hi):  # P_hi ... P_lo (inclusive), identity if empty
        M = np.eye(dk)
        for s in range(lo, hi + 1):
            M = P[s] @ M
        return M

    Y, S_t = [], None
    for t in range(T):
        S_t = prod(0, t) @ S0
        for i in range(t + 1):
            S_t = S_t + prod(i + 1, t) @ (b[i] * np.outer(K[i], V[i]))
        Y.append(S_t.T @ Q[t])
    return np.array(Y), S_t


def chunked_np(Q, K, V, a, b, S0, C):
    """Chunked (WY/UT) form of the gated delta rule, fp64.

    Within a chunk, gamma_t = prod_{s<=t} alpha_s and u_t = beta_t (v_t - alpha_t S_{t-1}^T k_t).
    Unrolling the recurrence gives (I + A) u = diag(beta) V - diag(beta gamma) K S_0 with
    A_ti = beta_t (gamma_t/gamma_i) k_t.k_i for i < t, so u = U - W S_0,
    U = T diag(beta) V, W = T diag(beta gamma) K, T = (I + A)^-1, and then
    S_C = gamma_C S_0 + sum_i (gamma_C/gamma_i) k_i u_i^T,
    y_t = gamma_t S_0^T q_t + sum_{i<=t} (gamma_t/gamma_i)(k_i.q_t) u_i.
    """
    T_len = K.shape[0]
    S = S0.copy()
    Y = np.zeros((T_len, V.shape[1]))
    for c0 in range(0, T_len, C):
        c1 = min(T_len, c0 + C)
        Kc, Vc, Qc = K[c0:c1], V[c0:c1], Q[c0:c1]
        g = np.cumsum(np.log(a[c0:c1]))
        gam = np.exp(g)
        bc = b[c0:c1]
        n = c1 - c0
        Gam = np.exp(g[:, None] - g[None, :])
        A = np.tril(bc[:, None] * (Kc @ Kc.T) * Gam, -1)
        Tinv = np.linalg.inv(np.eye(n) + A)
        W = Tinv @ ((bc * gam)[:, None] * Kc)
        U = Tinv @ (bc[:, None] * Vc)
        u = U - W @ S
        Pm = np.tril((Qc @ Kc.T) * Gam)
        Y[c0:c1] = gam[:, None] * (Qc @ S) + Pm @ u
        S = gam[-1] * S + ((gam[-1] / gam)[:, None] * Kc).T @ u
    return Y, S


def rel(x, ref):
    return float(np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300))


def rand_core(seed, T, dk, dv, c=0.1, s0_std=0.3):
    rng = np.random.default_rng(seed)
    Q, K = unit_rows(rng, (T, dk)), unit_rows(rng, (T, dk))
    V = rng.standard_normal((T, dv))
    a = np.exp(-c * np.logaddexp(0, rng.standard_normal(T)))
    b = 1 / (1 + np.exp(-rng.standard_normal(T)))
    S0 = s0_std * rng.standard_normal((dk, dv))
    return Q, K, V, a, b, S0


# ----------------------------------------------------------------------------- pins
def test_golden_exact_rational():
    """The four-equation oracle equals an exact rational evaluation of the one-step form."""
    doc = json.load(open(os.path.join(GOLDEN, "gdn_tiny_exact.json")))
    fr = lambda s: float(Fraction(s))  # noqa: E731
    inp = doc["inputs"]
    K = np.array([[fr(x) for x in r] for r in inp["k"]])
    Q = np.array([[fr(x) for x in r] for r in inp["q"]])
    V = np.array([[fr(x) for x in r] for r in inp["v"]])
    a = np.array([fr(x) for x in inp["alpha"]])
    b = np.array([fr(x) for x in inp["beta"]])
    S0 = np.array([[fr(x) for x in r] for r in inp["S0"]])
    y, S = run_core(Q, K, V, a, b, S0)
    yg = np.array([[fr(x) for x in r] for r in doc["y"]])
    Sg = np.array([[fr(x) for x in r] for r in doc["S_T"]])
    assert np.max(np.abs(y - yg)) < 1e-13
    assert np.max(np.abs(S - Sg)) < 1e-13


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_matches_one_step_form(seed):
    Q, K, V, a, b, S0 = rand_core(seed, T=40, dk=16, dv=12)
    y, S = run_core(Q, K, V, a, b, S0)
    y1, S1 = one_step_np(Q, K, V, a, b, S0)
    assert rel(y, y1) < 1e-12 and rel(S, S1) < 1e-12


@pytest.mark.parametrize("dk,dv,T", [(4, 4, 6), (8, 5, 8), (6, 8, 7)])
def test_brute_force_transition_products(dk, dv, T):
    Q, K, V, a, b, S0 = rand_core(10 + T, T, dk, dv)
    y, S = run_core(Q, K, V, a, b, S0)
    yb, Sb = transition_brute(Q, K, V, a, b, S0)
    assert rel(y, yb) < 1e-12 and rel(S, Sb) < 1e-12


def test_beta_zero_is_pure_decay():
    Q, K, V, a, b, S0 = rand_core(7, T=50, dk=16, dv=16)
    b = np.zeros_like(b)
    y, S = run_core(Q, K, V, a, b, S0)
    gam = np.cumprod(a)
    assert rel(S, gam[-1] * S0) < 1e-13
    assert rel(y, gam[:, None] * (Q @ S0)) < 1e-13


@pytest.mark.parametrize("with_s0", [False, True])
def test_orthonormal_keys_exact_recall(with_s0):
    """alpha = beta = 1 and orthonormal keys: S_t^T k_i = v_i for every i <= t."""
    rng = np.random.default_rng(5)
    dk, dv, T = 32, 24, 32
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    K = Qm.T[:T]                                   # orthonormal rows
    V = rng.standard_normal((T, dv))
    # q_t reads back an earlier key, so y_t must be that key's value
    src = np.array([rng.integers(0, t + 1) for t in range(T)])
    Q = K[src]
    S0 = rng.standard_normal((dk, dv)) if with_s0 else np.zeros((dk, dv))
    y, S = run_core(Q, K, V, np.ones(T), np.ones(T), S0)
    assert np.max(np.abs(S.T @ K.T - V.T)) < 1e-12
    assert np.max(np.abs(y - V[src])) < 1e-12


def test_idempotent_write():
    rng = np.random.default_rng(9)
    dk, dv = 16, 8
    k = unit_rows(rng, (1, dk))
    v = rng.standard_normal((1, dv))
    S0 = rng.standard_normal((dk, dv))
    K2, V2 = np.vstack([k, k]), np.vstack([v, v])
    _, S_once = run_core(K2[:1], K2[:1], V2[:1], np.ones(1), np.ones(1), S0)
    _, S_twice = run_core(K2, K2, V2, np.ones(2), np.ones(2), S0)
    assert np.max(np.abs(S_once - S_twice)) < 1e-13


@pytest.mark.parametrize("C", [1, 16, 64])
@pytest.mark.parametrize("T", [64, 100, 200])
def test_chunked_equals_sequential(C, T):
    Q, K, V, a, b, S0 = rand_core(100 + T + C, T, dk=32, dv=24)
    y, S = run_core(Q, K, V, a, b, S0)
    yc, Sc = chunked_np(Q, K, V, a, b, S0, C)
    assert rel(y, yc) < 1e-10 and rel(S, Sc) < 1e-10


def test_linear_in_values():
    """With a zero initial state and fixed q, k, alpha, beta, y is linear in the raw values
    (conv and recurrence are both linear in v)."""
    shape = gi.GdnShape(n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16)
    p = gi.make_prefill_inputs(shape, [37], gi.F32, seed=11)
    v2 = gi.make_prefill_inputs(shape, [37], gi.F32, seed=12).v.astype(np.float64)
    v1 = p.v.astype(np.float64)

    def run(v):
        return oracle.gdn_prefill_f64(p.q, p.k, v, p.w_q, p.w_k, p.w_v, p.alpha, p.beta,
                                      p.cu_seqlens, n_qk_heads=1, n_v_heads=2)[0]
    assert rel(run(2.0 * v1 - 3.0 * v2), 2 * run(v1) - 3 * run(v2)) < 1e-12


# ----------------------------------------------------------------------------- conv + L2
def test_conv_matches_numpy_convolve_and_unit_norm():
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=4, d_k=8, d_v=8)
    p = gi.make_prefill_inputs(shape, [5, 0, 9, 2], gi.F32, seed=3, with_conv_state=True)
    qh, kh, vh = oracle.gdn_conv_l2_f64(p.q, p.k, p.v, p.w_q, p.w_k, p.w_v, p.cu_seqlens,
                                        n_qk_heads=2, n_v_heads=4, conv_state=p.conv_state,
                                        l2_eps=0.0, q_scale=0.5)
    cs = p.conv_state.astype(np.float64)
    H, dk = 2, 8
    for b in range(p.n_seqs):
        t0, t1 = p.cu_seqlens[b], p.cu_seqlens[b + 1]
        for name, x, w, out, off, norm in (("q", p.q, p.w_q, qh, 0, 0.5), ("k", p.k, p.w_k, kh, H * dk, 1.0),
                                          ("v", p.v, p.w_v, vh, 2 * H * dk, None)):
            xs = x[t0:t1].reshape(t1 - t0, x.shape[1] * x.shape[2]).astype(np.float64)
            hist = cs[b, :, off:off + xs.shape[1]]
            full = np.vstack([hist, xs])                 # history rows first
            ref = np.zeros_like(xs)
            for c in range(xs.shape[1]):
                conv = np.convolve(full[:, c], w[c, ::-1].astype(np.float64))
                ref[:, c] = conv[3:3 + (t1 - t0)]        # outputs aligned with the sequence rows
            ref = ref.reshape(x[t0:t1].shape)
            if norm is not None:
                ref = norm * ref / np.linalg.norm(ref, axis=-1, keepdims=True)
                if t1 > t0:
                    assert np.allclose(np.linalg.norm(out[t0:t1], axis=-1), norm, atol=1e-13)
            assert np.max(np.abs(out[t0:t1] - ref), initial=0.0) < 1e-12, name


def test_identity_conv_without_history():
    shape = gi.GdnShape(n_qk_heads=1, n_v_heads=1, d_k=8, d_v=8)
    p = gi.make_prefill_inputs(shape, [6], gi.F32, seed=4)
    w = identity_weights(8)
    qh, kh, vh = oracle.gdn_conv_l2_f64(p.q, p.k, p.v, w, w, w, p.cu_seqlens, n_qk_heads=1,
                                        n_v_heads=1, l2_eps=0.0)
    assert np.max(np.abs(vh - p.v)) == 0.0
    qn = p.q / np.linalg.norm(p.q.astype(np.float64), axis=-1, keepdims=True)
    assert np.max(np.abs(qh - qn)) < 1e-15


def test_conv_state_out_is_last_raw_rows():
    shape = gi.GdnShape(n_qk_heads=1, n_v_heads=2, d_k=4, d_v=4)
    p = gi.make_prefill_inputs(shape, [0, 1, 2, 3, 7], gi.F32, seed=8, with_conv_state=True)
    _, _, cso = oracle.prefill(p)
    raw = np.concatenate([p.q.reshape(p.total_tokens, -1), p.k.reshape(p.total_tokens, -1),
                          p.v.reshape(p.total_tokens, -1)], axis=1).astype(np.float64)
    for b in range(p.n_seqs):
        t0, t1 = p.cu_seqlens[b], p.cu_seqlens[b + 1]
        rows = np.vstack([p.conv_state[b].astype(np.float64), raw[t0:t1]])
        assert np.array_equal(cso[b], rows[-3:])


# ----------------------------------------------------------------------------- composition
def test_split_equals_whole():
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6, d_k=16, d_v=16)
    p = gi.make_prefill_inputs(shape, [90], gi.F32, seed=21, with_initial_state=True,
                               with_conv_state=True)
    y, fin, cso = oracle.prefill(p)
    T1 = 37
    first = gi.make_prefill_inputs(shape, [90], gi.F32, seed=21, with_initial_state=True,
                                   with_conv_state=True)
    for name in ("q", "k", "v", "alpha", "beta"):
        setattr(first, name, getattr(p, name)[:T1])
    first.cu_seqlens = np.array([0, T1], np.int32)
    y1, fin1, cs1 = oracle.prefill(first)
    second = gi.make_prefill_inputs(shape, [90], gi.F32, seed=21)
    for name in ("q", "k", "v", "alpha", "beta"):
        setattr(second, name, getattr(p, name)[T1:])
    second.cu_seqlens = np.array([0, 90 - T1], np.int32)
    y2, fin2, cs2 = oracle.prefill(second, initial_state=fin1, conv_state=cs1)
    assert rel(np.concatenate([y1, y2]), y) < 1e-12
    assert rel(fin2, fin) < 1e-12
    assert np.array_equal(cs2, cso)


def test_packed_equals_separate():
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=4, d_k=16, d_v=8)
    lens = [13, 0, 1, 40, 3]
    p = gi.make_prefill_inputs(shape, lens, gi.F32, seed=31, with_initial_state=True,
                               with_conv_state=True)
    y, fin, cso = oracle.prefill(p)
    for b, L in enumerate(lens):
        t0, t1 = p.cu_seqlens[b], p.cu_seqlens[b + 1]
        s = gi.make_prefill_inputs(shape, [L], gi.F32, seed=31)
        for name in ("q", "k", "v", "alpha", "beta"):
            setattr(s, name, getattr(p, name)[t0:t1])
        s.w_q, s.w_k, s.w_v = p.w_q, p.w_k, p.w_v
        ys, fs, cs = oracle.prefill(s, initial_state=p.initial_state[b:b + 1],
                                    conv_state=p.conv_state[b:b + 1].astype(np.float64))
        assert np.max(np.abs(ys - y[t0:t1]), initial=0.0) < 1e-12
        assert np.max(np.abs(fs[0] - fin[b])) < 1e-12
        assert np.array_equal(cs[0], cso[b])
    # a zero-length sequence returns its initial state and conv state unchanged
    assert np.array_equal(fin[1], p.initial_state[1].astype(np.float64))
    assert np.array_equal(cso[1], p.conv_state[1].astype(np.float64))


def test_decode_steps_equal_prefill():
    shape = gi.GdnShape(n_qk_heads=1, n_v_heads=3, d_k=8, d_v=8)
    B, T = 3, 10
    w = gi.make_conv_weights(shape, 41)
    dec = gi.make_decode_inputs(shape, B, T, gi.F32, seed=42)
    rng = np.random.default_rng(43)
    S0 = 0.1 * rng.standard_normal((B, 3, 8, 8))
    cs0 = rng.standard_normal((B, 3, shape.channels)).astype(np.float32)
    ys, S, cs = oracle.decode_steps(shape, gi.F32, dec, w, S0, cs0)
    for b in range(B):
        y, fin, cso = oracle.gdn_prefill_f64(
            dec.q[:, b], dec.k[:, b], dec.v[:, b], *w, dec.alpha[:, b], dec.beta[:, b],
            np.array([0, T], np.int32), n_qk_heads=1, n_v_heads=3, initial_state=S0[b:b + 1],
            conv_state=cs0[b:b + 1])
        assert rel(ys[:, b], y) < 1e-12
        assert rel(S[b], fin[0]) < 1e-12
        assert np.array_equal(cs[b], cso[0])


def test_head_mapping_contiguous_groups():
    """V heads g*G .. g*G+G-1 read QK head g: identical v/alpha/beta within a group give
    identical outputs, and permuting V heads inside a group permutes the outputs."""
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6, d_k=8, d_v=8)
    p = gi.make_prefill_inputs(shape, [20], gi.F32, seed=51)
    for g in range(2):
        for h in range(3 * g + 1, 3 * g + 3):
            p.v[:, h] = p.v[:, 3 * g]
            p.alpha[:, h] = p.alpha[:, 3 * g]
            p.beta[:, h] = p.beta[:, 3 * g]
            p.w_v[h * 8:(h + 1) * 8] = p.w_v[3 * g * 8:(3 * g + 1) * 8]
    y, _, _ = oracle.prefill(p)
    for g in range(2):
        for h in range(3 * g + 1, 3 * g + 3):
            assert np.array_equal(y[:, h], y[:, 3 * g])
    assert not np.allclose(y[:, 0], y[:, 3])
    # permutation within group 1
    p2 = gi.make_prefill_inputs(shape, [20], gi.F32, seed=52)
    ya, _, _ = oracle.prefill(p2)
    perm = [0, 1, 2, 5, 3, 4]
    p2.v = p2.v[:, perm].copy()
    p2.alpha = p2.alpha[:, perm].copy()
    p2.beta = p2.beta[:, perm].copy()
    p2.w_v = p2.w_v.reshape(6, 8, 4)[perm].reshape(48, 4).copy()
    yb, _, _ = oracle.prefill(p2)
    assert np.array_equal(yb, ya[:, perm])


# ----------------------------------------------------------------------------- planted mistakes
def _full_pipeline_brute(p, q_scale=1.0, silu=False):
    """Whole mixer rebuilt from library routines: np.convolve, scipy's logistic function for
    the optional SiLU, np.linalg.norm and the transition-product brute force (one
    (seq, V head) at a time)."""
    from scipy.special import expit
    H, Hv = p.shape.n_qk_heads, p.shape.n_v_heads
    dk, dv = p.shape.d_k, p.shape.d_v
    G = Hv // H
    T = p.total_tokens
    out = np.zeros((T, Hv, dv))
    fins = np.zeros((p.n_seqs, Hv, dk, dv))
    for b in range(p.n_seqs):
        t0, t1 = p.cu_seqlens[b], p.cu_seqlens[b + 1]

        def conv(x, w):
            xs = x[t0:t1].reshape(t1 - t0, x.shape[1] * x.shape[2]).astype(np.float64)
            full = np.vstack([np.zeros((3, xs.shape[1])), xs])
            r = np.stack([np.convolve(full[:, c], w[c, ::-1].astype(np.float64))[3:3 + t1 - t0]
                          for c in range(xs.shape[1])], axis=1)
            return r.reshape(x[t0:t1].shape)
        qc, kc, vc = conv(p.q, p.w_q), conv(p.k, p.w_k), conv(p.v, p.w_v)
        if silu:
            qc, kc, vc = qc * expit(qc), kc * expit(kc), vc * expit(vc)
        qn = q_scale * qc / np.sqrt((qc ** 2).sum(-1, keepdims=True) + 1e-6)
        kn = kc / np.sqrt((kc ** 2).sum(-1, keepdims=True) + 1e-6)
        for h in range(Hv):
            g = h // G
            a = p.alpha[t0:t1, h].astype(np.float64)
            bb = p.beta[t0:t1, h].astype(np.float64)
            y, S = transition_brute(qn[:, g], kn[:, g], vc[:, h], a, bb, np.zeros((dk, dv)))
            out[t0:t1, h] = y
            fins[b, h] = S
    return out, fins


@pytest.mark.parametrize("silu", [False, True])
def test_brute_pipeline_matches_oracle(silu):
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6, d_k=6, d_v=5)
    p = gi.make_prefill_inputs(shape, [7, 3], gi.F32, seed=61)
    y, fin, _ = oracle.prefill(p, conv_silu=silu)
    yb, fb = _full_pipeline_brute(p, silu=silu)
    assert rel(y, yb) < 1e-11 and rel(fin, fb) < 1e-11
    if silu:   # the activation changes the result
        y0, _, _ = oracle.prefill(p)
        assert rel(y, y0) > 1e-2


def test_conv_silu_closed_forms():
    """With the identity conv ([0, 0, 0, 1] taps) the conv output of each channel is the raw
    value x, so q^ is SiLU(x) normalised: SiLU(0) = 0, SiLU(ln 3) = (3/4) ln 3 and
    SiLU(-ln 3) = -(1/4) ln 3 (the logistic function at ln 3 is 3/4); v is SiLU(x) itself."""
    shape = gi.GdnShape(n_qk_heads=1, n_v_heads=1, d_k=4, d_v=4)
    ln3 = np.log(3.0)
    x = np.array([[[0.0, ln3, -ln3, 2.0]]])
    w = identity_weights(4)
    qh, kh, vh = oracle.gdn_conv_l2_f64(x, x, x, w, w, w, np.array([0, 1], np.int32), n_qk_heads=1,
                                        n_v_heads=1, l2_eps=0.0, conv_silu=True)
    s = np.array([0.0, 0.75 * ln3, -0.25 * ln3, 2.0 / (1.0 + np.exp(-2.0))])
    np.testing.assert_allclose(vh[0, 0], s, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(qh[0, 0], s / np.linalg.norm(s), rtol=1e-14)
    np.testing.assert_allclose(kh[0, 0], s / np.linalg.norm(s), rtol=1e-14)


MUTANTS = {1: "error uses the undecayed state", 2: "output reads the state before the write",
           3: "state transposed", 4: "conv taps reversed", 5: "interleaved V->QK head mapping",
           6: "beta dropped from the write", 7: "conv SiLU after the L2 normalisation"}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutant):
    shape = gi.GdnShape(n_qk_heads=2, n_v_heads=6, d_k=6, d_v=6)
    p = gi.make_prefill_inputs(shape, [7, 3], gi.F32, seed=61)
    oracle.build(mutant)
    silu = mutant == 7   # that mistake lives in the optional activation
    y, fin, _ = oracle.prefill(p, mutant=mutant, conv_silu=silu)
    yb, fb = _full_pipeline_brute(p, silu=silu)
    assert rel(y, yb) > 1e-3 or rel(fin, fb) > 1e-3, MUTANTS[mutant]


# ----------------------------------------------------------------- output tail (gated RMSNorm)
def test_output_gate_closed_forms():
    """One-hot y: the RMS over 128 channels is 1/sqrt(128), so o_0 = sqrt(128 / (1 + 128 eps))
    w_0 SiLU(z_0) and every other channel is 0; SiLU at 0, ln 3 and -ln 3 is 0, (3/4) ln 3 and
    -(1/4) ln 3 (sigmoid(ln 3) = 3/4)."""
    from oracle.output_gate import output_gate
    eps = 1e-6
    y = np.zeros((3, 2, 128))
    y[..., 0] = 1.0
    ln3 = np.log(3.0)
    z = np.zeros((3, 2, 128))
    z[0, :, 0], z[1, :, 0], z[2, :, 0] = 0.0, ln3, -ln3
    w = np.linspace(0.5, 1.5, 128)
    o = output_gate(y, z, w, eps)
    amp = np.sqrt(128.0 / (1.0 + 128.0 * eps)) * w[0]
    np.testing.assert_allclose(o[0, :, 0], 0.0, atol=0)
    np.testing.assert_allclose(o[1, :, 0], amp * 0.75 * ln3, rtol=1e-14)
    np.testing.assert_allclose(o[2, :, 0], -amp * 0.25 * ln3, rtol=1e-14)
    assert np.all(o[..., 1:] == 0)


def test_output_gate_invariances():
    """With eps = 0 the normalisation removes any positive scale of y and is odd in y; the
    norm is per (token, head): scaling one head leaves the others unchanged."""
    from oracle.output_gate import output_gate
    rng = np.random.default_rng(7)
    y = rng.standard_normal((5, 3, 128))
    z = rng.standard_normal((5, 3, 128))
    w = rng.standard_normal(128)
    o = output_gate(y, z, w, 0.0)
    np.testing.assert_allclose(output_gate(7.5 * y, z, w, 0.0), o, rtol=1e-13)
    np.testing.assert_allclose(output_gate(-y, z, w, 0.0), -o, rtol=1e-13)
    y2 = y.copy()
    y2[:, 1] *= 100.0
    o2 = output_gate(y2, z, w, 0.0)
    np.testing.assert_allclose(o2[:, [0, 2]], o[:, [0, 2]], rtol=1e-13)


def test_output_gate_brute_force():
    """Element by element in plain Python (math module) on a tiny case."""
    import math
    from oracle.output_gate import output_gate
    rng = np.random.default_rng(8)
    y = rng.standard_normal((2, 2, 128))
    z = 3.0 * rng.standard_normal((2, 2, 128))
    w = rng.standard_normal(128)
    eps = 1e-3
    o = output_gate(y, z, w, eps)
    for t in range(2):
        for h in range(2):
            s = 0.0
            for i in range(128):
                s += y[t, h, i] ** 2
            inv = 1.0 / math.sqrt(s / 128.0 + eps)
            for i in range(128):
                g = z[t, h, i] / (1.0 + math.exp(-z[t, h, i]))
                assert abs(o[t, h, i] - y[t, h, i] * inv * w[i] * g) <= 1e-12 * (1 + abs(o[t, h, i]))
