"""Pins of the QSA indexer oracle against what the page and the mathematics fix (CPU only).

Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03, QSA indexer figure (BLOCK SCORE,
CAUSAL SPARSE SET) and the five-step list under "QSA".  The page prints no worked numbers,
so the oracle is held to statements other than its own code:
  * closed forms: bf16 rounding of chosen values; RMSNorm of constant rows; the mean of a
    block with eps = 1 (which a sum would miss); the rotation of basis vectors, which fixes
    the pairing (d, d + 32), the sign, the frequency theta^(-d/32) and that dims 64..127
    stay; a block's encoding at position r b;
  * rotation invariants: norms kept, scores depend only on position differences (so
    shifting queries and blocks together by whole blocks changes nothing);
  * brute force: scores by plain loops; the selected set maximises the summed score over
    all k-subsets (distinct scores); equal scores resolved toward the lower index;
  * ReLU(x) + ReLU(-x) = |x| per head, which holds only if ReLU comes before the head sum;
  * the token set with an unlimited budget is exactly the causal prefix 0..i, each token
    once, for every i (fixes the completeness rule and the tail together).
``test_planted_mistakes`` swaps one plausible mistake at a time into the oracle and checks
that these pins catch each one.
"""
import itertools
import math

import numpy as np
import pytest

import gdn_inputs as gi
from oracle import qsa_indexer as qi


# ----------------------------------------------------------------------------- pins
def pin_bf16_round():
    cases = [(1.0 + 2.0 ** -8, 1.0),                       # halfway: to even (1.0)
             (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),        # halfway: to even (1 + 2/128)
             (1.0 + 2.0 ** -8 + 2.0 ** -20, 1.0 + 2.0 ** -7),
             (-3.0 - 2.0 ** -7, -3.0),
             (0.0, 0.0)]
    for x, want in cases:
        assert qi.bf16_round(x) == want, (x, qi.bf16_round(x), want)
    # fp32-representable values: same result as the input module's bit-level rounding
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(4096) * np.exp(rng.uniform(-20, 20, 4096))).astype(np.float32)
    ref = gi.bf16_bits_to_f32(gi.f32_to_bf16_bits(x)).astype(np.float64)
    assert np.array_equal(qi.bf16_round(x.astype(np.float64)), ref)


def pin_rms_norm():
    w = np.linspace(0.5, 2.0, 128)
    for c, eps in ((3.0, 0.0), (2.0, 1.0), (-0.5, 1e-6)):
        got = qi.rms_norm(np.full(128, c), w, eps)
        assert np.allclose(got, c / math.sqrt(c * c + eps) * w, rtol=1e-15, atol=0)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128))
    y = qi.rms_norm(x, np.ones(128), 0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-14)      # unit mean square
    assert np.allclose(qi.rms_norm(7.5 * x, np.ones(128), 0.0), y, rtol=1e-14)


def pin_block_mean():
    # rows 1, 2, 3, 6 in every dim: mean 3 -> 3 / sqrt(9 + 1) with eps = 1, block 0 (no rotation)
    k = np.repeat(np.array([1.0, 2.0, 3.0, 6.0])[:, None], 128, axis=1)
    got = qi.block_keys(k, np.ones(128), eps=1.0, theta=10000.0)
    assert got.shape == (1, 128)
    assert np.allclose(got[0], 3.0 / math.sqrt(10.0), rtol=1e-15)
    # a trailing incomplete block is not formed
    assert qi.block_keys(np.ones((7, 128)), np.ones(128)).shape == (1, 128)


def pin_rope_basis():
    theta = 10000.0
    for d in (0, 5, 16, 31):
        f = theta ** (-d / 32.0)
        for p in (1, 3, 100, 12345):
            e = np.zeros(128)
            e[d] = 1.0
            got = qi.rope_partial(e, p, theta)
            want = np.zeros(128)
            want[d], want[d + 32] = math.cos(p * f), math.sin(p * f)
            assert np.allclose(got, want, atol=1e-12), (d, p)
            e2 = np.zeros(128)
            e2[d + 32] = 1.0
            want2 = np.zeros(128)
            want2[d], want2[d + 32] = -math.sin(p * f), math.cos(p * f)
            assert np.allclose(qi.rope_partial(e2, p, theta), want2, atol=1e-12), (d, p)
    # frequency of pair 16 at theta = 1e4 is 1/100: position 100 turns it by one radian
    e = np.zeros(128)
    e[16] = 1.0
    got = qi.rope_partial(e, 100, 1e4)
    assert abs(got[16] - math.cos(1.0)) < 1e-12 and abs(got[48] - math.sin(1.0)) < 1e-12
    # dims 64..127 never move; position 0 is the identity
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128)
    assert np.array_equal(qi.rope_partial(x, 777, theta)[64:], x[64:])
    assert np.allclose(qi.rope_partial(x, 0, theta), x, atol=0)


def pin_rope_invariants():
    rng = np.random.default_rng(4)
    x, y = rng.standard_normal((2, 128))
    theta = 5e5
    for p, s, shift in ((10, 3, 400), (0, 1000, 4), (65535, 17, 1 << 19)):
        a = qi.rope_partial(x, p, theta) @ qi.rope_partial(y, s, theta)
        b = qi.rope_partial(x, p + shift, theta) @ qi.rope_partial(y, s + shift, theta)
        assert abs(a - b) < 1e-8 * (1 + abs(a))
        assert abs(np.linalg.norm(qi.rope_partial(x, p, theta)) - np.linalg.norm(x)) < 1e-12


def pin_block_position():
    # every token's key = e_0, w = 1, eps = 0: pooled e_0 -> sqrt(128) e_0 -> rotated at 4 j
    T = 24
    k = np.zeros((T, 128))
    k[:, 0] = 1.0
    got = qi.block_keys(k, np.ones(128), eps=0.0, theta=10000.0)
    for j in range(T // 4):
        want = np.zeros(128)
        want[0], want[32] = math.cos(4 * j), math.sin(4 * j)
        assert np.allclose(got[j], math.sqrt(128) * want, atol=1e-12), j
    # the same with the tokens starting at position 8: block j sits at 8 + 4 j
    got8 = qi.block_keys(k, np.ones(128), eps=0.0, theta=10000.0, pos0=8)
    assert np.allclose(got8[0], got[2], atol=1e-12)


def _brute_scores(qh, kbar, pos):
    n, nb = qh.shape[0], kbar.shape[0]
    out = [[0.0] * nb for _ in range(n)]
    for r in range(n):
        for b in range(nb):
            if 4 * b + 3 > pos[r]:
                out[r][b] = -math.inf
                continue
            tot = 0.0
            for h in range(4):
                dot = 0.0
                for d in range(128):
                    dot += qh[r, h, d] * kbar[b, d]
                tot += dot if dot > 0 else 0.0
            out[r][b] = tot
    return np.array(out)


def pin_scores_brute():
    rng = np.random.default_rng(5)
    qh = rng.standard_normal((7, 4, 128))
    kbar = rng.standard_normal((6, 128))
    pos = np.array([0, 2, 3, 4, 7, 18, 30])
    got = qi.block_scores(qh, kbar, pos)
    want = _brute_scores(qh, kbar, pos)
    assert np.array_equal(np.isinf(got), np.isinf(want))
    fin = np.isfinite(want)
    assert np.allclose(got[fin], want[fin], rtol=1e-12, atol=1e-12)
    # the cache size caps the visible blocks
    capped = qi.block_scores(qh, kbar, pos, n_blocks=2)
    assert np.all(np.isinf(capped[:, 2:]))


def pin_relu_per_head():
    rng = np.random.default_rng(6)
    qh = rng.standard_normal((3, 4, 128))
    kbar = rng.standard_normal((5, 128))
    pos = np.array([100, 100, 100])
    s = qi.block_scores(qh, kbar, pos) + qi.block_scores(-qh, kbar, pos)
    want = np.abs(np.einsum("nhd,bd->nhb", qh, kbar)).sum(axis=1)
    assert np.allclose(s, want, rtol=1e-12)
    # the heads enter symmetrically
    perm = qi.block_scores(qh[:, [2, 0, 3, 1]], kbar, pos)
    assert np.allclose(perm, qi.block_scores(qh, kbar, pos), rtol=1e-12)


def pin_top_blocks():
    rng = np.random.default_rng(7)
    for trial in range(30):
        nb = int(rng.integers(1, 9))
        kb = int(rng.integers(1, 5))
        s = rng.permutation(nb).astype(np.float64) + rng.uniform(0, 0.5, nb)   # distinct
        ninf = int(rng.integers(0, nb))
        s[nb - ninf:] = -np.inf
        got = [int(b) for b in qi.top_blocks(s, kb) if b >= 0]
        fin = [b for b in range(nb) if np.isfinite(s[b])]
        m = min(kb, len(fin))
        best = max(itertools.combinations(fin, m), key=lambda c: sum(s[b] for b in c))
        assert sorted(best) == got, (s, kb, got)
        assert got == sorted(got)
    # equal scores: lower index first; all-equal row takes the first k
    assert list(qi.top_blocks([1.0, 2.0, 2.0, 2.0, 0.0], 2)) == [1, 2]
    assert list(qi.top_blocks([0.0] * 6, 3)) == [0, 1, 2]
    assert list(qi.top_blocks([5.0, -np.inf, -np.inf], 2)) == [0, -1]


def pin_token_set_prefix():
    # unlimited budget: the token set is exactly 0..i for every i
    rng = np.random.default_rng(8)
    nq = 60
    qh = rng.standard_normal((nq, 4, 128))
    kbar = rng.standard_normal((nq // 4 + 1, 128))
    pos = np.arange(nq)
    s = qi.block_scores(qh, kbar, pos)
    for i in range(nq):
        b = qi.top_blocks(s[i], 64)
        t = qi.token_set(b, i, 64)
        assert [int(x) for x in t if x >= 0] == list(range(i + 1)), i
    # limited budget: k full blocks + the tail, distinct, all <= i
    for i in (17, 31, 45, 59):
        b = qi.top_blocks(s[i], 3)
        t = [int(x) for x in qi.token_set(b, i, 3) if x >= 0]
        assert len(t) == len(set(t)) == 4 * 3 + (i + 1) % 4
        assert max(t) <= i and sorted(t) == t
        tail = (i + 1) % 4
        assert t[len(t) - tail:] == list(range(i + 1 - tail, i + 1))


def pin_shift_by_blocks():
    rng = np.random.default_rng(9)
    k = rng.standard_normal((64, 128))
    q = rng.standard_normal((10, 4, 128))
    wq, wk = rng.uniform(0.5, 1.5, (2, 128))
    pos = np.arange(54, 64)
    base = qi.block_scores(qi.query_heads(q, wq, pos), qi.block_keys(k, wk), pos)
    for d in (4, 4096):
        kb = qi.block_keys(k, wk, pos0=d)
        qh = qi.query_heads(q, wq, pos + d)
        # the same 16 blocks, now at block indices d/4 .. d/4 + 15; local numbering keeps 0..15
        got = np.maximum(np.einsum("nhd,bd->nhb", qh, kb), 0.0).sum(axis=1)
        assert np.allclose(got, np.where(np.isfinite(base), base, got), rtol=1e-9, atol=1e-9)


def pin_bf16_operands():
    rng = np.random.default_rng(10)
    k = rng.standard_normal((32, 128))
    q = rng.standard_normal((4, 4, 128))
    w = np.ones(128)
    for ex, bf in ((qi.block_keys(k, w), qi.block_keys(k, w, operands="bf16")),
                   (qi.query_heads(q, w, np.arange(4)), qi.query_heads(q, w, np.arange(4), operands="bf16"))):
        assert np.array_equal(qi.bf16_round(bf), bf)                      # representable
        assert np.all(np.abs(bf - ex) <= 2.0 ** -8 * np.abs(ex))              # half an ulp


PINS = [pin_bf16_round, pin_rms_norm, pin_block_mean, pin_rope_basis, pin_rope_invariants,
        pin_block_position, pin_scores_brute, pin_relu_per_head, pin_top_blocks,
        pin_token_set_prefix, pin_shift_by_blocks, pin_bf16_operands]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_end_to_end_small():
    """The composed reference agrees with its parts, row by row."""
    rng = np.random.default_rng(12)
    T = 90
    k = rng.standard_normal((T, 128))
    q = rng.standard_normal((T, 4, 128))
    wq, wk = rng.uniform(0.5, 1.5, (2, 128))
    pos = np.arange(T)
    kbar, s, b, t = qi.indexer(q, k, wq, wk, pos, k_b=5)
    assert kbar.shape == (T // 4, 128) and b.shape == (T, 5) and t.shape == (T, 23)
    for i in (0, 3, 4, 21, 22, 89):
        nv = (i + 1) // 4
        sel = [int(x) for x in b[i] if x >= 0]
        assert len(sel) == min(5, nv) and all(0 <= x < nv for x in sel)


# ----------------------------------------------------------------------------- mistakes
def _m_rope_adjacent(x, pos, theta):
    x = np.array(x, dtype=np.float64)
    f = theta ** (-np.arange(32, dtype=np.float64) / 32)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * f
    a, b = x[..., 0:64:2].copy(), x[..., 1:64:2].copy()
    x[..., 0:64:2] = a * np.cos(ang) - b * np.sin(ang)
    x[..., 1:64:2] = b * np.cos(ang) + a * np.sin(ang)
    return x


def _m_rope_sign(x, pos, theta):
    return _ORIG["rope_partial"](x, -np.asarray(pos, dtype=np.float64), theta)


def _m_rope_freq(x, pos, theta):
    return _ORIG["rope_partial"](x, pos, theta ** 2.0)          # theta^(-d/64)-style exponent


def _m_rope_last_dims(x, pos, theta):
    x = np.array(x, dtype=np.float64)
    r = _ORIG["rope_partial"](np.concatenate([x[..., 64:], x[..., :64]], -1), pos, theta)
    return np.concatenate([r[..., 64:], r[..., :64]], -1)


def _m_rms_eps_outside(x, w, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * w


def _m_block_keys_sum(k, w_k, eps=1e-6, theta=10000.0, pos0=0, operands="exact"):
    k = np.asarray(k, dtype=np.float64)
    nb = k.shape[0] // 4
    pooled = k[:nb * 4].reshape(nb, 4, 128).sum(axis=1)
    return qi.rope_partial(qi.rms_norm(pooled, w_k, eps), pos0 + 4 * np.arange(nb), theta)


def _m_block_keys_index_pos(k, w_k, eps=1e-6, theta=10000.0, pos0=0, operands="exact"):
    k = np.asarray(k, dtype=np.float64)
    nb = k.shape[0] // 4
    pooled = k[:nb * 4].reshape(nb, 4, 128).mean(axis=1)
    return qi.rope_partial(qi.rms_norm(pooled, w_k, eps), pos0 // 4 + np.arange(nb), theta)


def _m_scores_relu_after_sum(qh, kbar, pos, n_blocks=None):
    s = np.maximum(np.einsum("nhd,bd->nhb", qh, kbar).sum(axis=1), 0.0)
    for r, i in enumerate(np.asarray(pos)):
        s[r, qi.n_complete(i, n_blocks):] = -np.inf
    return s


def _m_complete_off_by_one(i, n_blocks=None):
    n = max(0, (int(i) + 2) // 4)
    return n if n_blocks is None else min(n, int(n_blocks))


def _m_top_ties_high(score_row, k_b=qi.K_B):
    s = np.asarray(score_row, dtype=np.float64)
    idx = np.flatnonzero(np.isfinite(s))
    order = idx[np.lexsort((-idx, -s[idx]))][:k_b]
    out = np.full(k_b, -1, dtype=np.int64)
    out[:len(order)] = np.sort(order)
    return out


def _m_tail_start(blocks, i, k_b=qi.K_B):
    sel = [int(b) for b in blocks if b >= 0]
    toks = [4 * b + t for b in sel for t in range(4)] + list(range(4 * (int(i) // 4), int(i) + 1))
    out = np.full(4 * k_b + 3, -1, dtype=np.int64)
    out[:len(toks)] = toks
    return out


def _m_bf16_truncate(x):
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.trunc(m * 256.0) / 256.0, e)


_ORIG = {n: getattr(qi, n) for n in ("rope_partial", "rms_norm", "block_keys", "block_scores",
                                     "n_complete", "top_blocks", "token_set", "bf16_round")}

MISTAKES = {
    "rope pairs adjacent dims": ("rope_partial", _m_rope_adjacent),
    "rope turns the other way": ("rope_partial", _m_rope_sign),
    "rope frequency exponent halved": ("rope_partial", _m_rope_freq),
    "rope on dims 64..127": ("rope_partial", _m_rope_last_dims),
    "rmsnorm eps outside the root": ("rms_norm", _m_rms_eps_outside),
    "block pooled by sum": ("block_keys", _m_block_keys_sum),
    "block rotated at its index": ("block_keys", _m_block_keys_index_pos),
    "ReLU after the head sum": ("block_scores", _m_scores_relu_after_sum),
    "completeness off by one": ("n_complete", _m_complete_off_by_one),
    "ties to the higher index": ("top_blocks", _m_top_ties_high),
    "tail starts at r floor(i / r)": ("token_set", _m_tail_start),
    "bf16 rounding truncates": ("bf16_round", _m_bf16_truncate),
}


@pytest.mark.parametrize("name", list(MISTAKES))
def test_planted_mistakes(name, monkeypatch):
    attr, bad = MISTAKES[name]
    monkeypatch.setattr(qi, attr, bad)
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches: {name}"


# ----------------------------------------------------------------------------- properties
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=200, deadline=None)
@given(st.lists(st.sampled_from([0.0, 0.5, 1.0, 2.0, 3.5, float("-inf")]), min_size=0, max_size=12),
       st.integers(min_value=1, max_value=6))
def test_top_blocks_property(scores, k):
    """Any row with ties: the selection holds min(k, finite) blocks, every selected score is
    >= every unselected finite score, and among equal scores at the cut the lowest indices win."""
    s = np.array(scores, dtype=np.float64)
    got = [int(b) for b in qi.top_blocks(s, k) if b >= 0]
    fin = [b for b in range(len(s)) if np.isfinite(s[b])]
    assert len(got) == min(k, len(fin)) and got == sorted(got) and set(got) <= set(fin)
    rest = [b for b in fin if b not in got]
    if got and rest:
        cut = min(s[b] for b in got)
        assert cut >= max(s[b] for b in rest)
        assert all(b > max(g for g in got if s[g] == cut) for b in rest if s[b] == cut)


@settings(max_examples=200, deadline=None)
@given(st.integers(min_value=0, max_value=400), st.integers(min_value=1, max_value=8))
def test_token_set_property(i, k):
    """For any position and budget: the token set is ascending, distinct, within 0..i, holds 4
    tokens per selected complete block plus the (i + 1) mod 4 tail tokens, and with the
    whole prefix selected it is exactly 0..i."""
    nv = qi.n_complete(i)
    blocks = np.full(k, -1)
    m = min(k, nv)
    blocks[:m] = np.arange(nv - m, nv)                 # the most recent blocks
    t = [int(x) for x in qi.token_set(blocks, i, k) if x >= 0]
    assert t == sorted(set(t)) and (not t or (t[0] >= 0 and t[-1] <= i))
    assert len(t) == 4 * m + (i + 1) % 4
    if m == nv:
        assert t == list(range(i + 1))
