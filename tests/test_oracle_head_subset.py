"""Pins of the oracle's head-subset mode (CPU only).

The full-size parity tests compute the oracle on a few sampled V heads: ``oracle.prefill``
then widens only the QK groups those heads read (their q/k heads, their conv weights and
the matching columns of the conv state) and maps each requested head to its place in the
sliced problem.  Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED DELTANET
equations): every V head evolves on its own from its QK head's q, k and its own v, alpha,
beta, so a subset must reproduce exactly what the whole layer computes for those heads.
These tests hold the subset mode to the whole-layer run, bit for bit, on a shape with
several QK groups, ragged sequences, initial states and conv states, and plant the slips
that a subset path could make to show that the comparison catches them.
"""
import numpy as np
import pytest

import gdn_inputs as gi
import oracle

SHAPE = gi.GdnShape(n_qk_heads=4, n_v_heads=12)          # 3 V heads per QK head
LENGTHS = [37, 0, 70, 5]
SUBSETS = [[7, 1, 10], [11], [0, 3, 6, 9], [5, 4], [2, 8, 3]]


@pytest.fixture(scope="module")
def problem(oracle_lib):
    inp = gi.make_prefill_inputs(SHAPE, LENGTHS, gi.BF16, seed=4321, with_initial_state=True,
                                 state_std=0.2, with_conv_state=True)
    full = oracle.prefill(inp)
    return inp, full


def _assert_subset_matches(inp, full, heads):
    y, fin, cs = oracle.prefill(inp, heads=heads)
    assert np.array_equal(y[:, heads], full[0][:, heads])
    assert np.array_equal(fin[:, heads], full[1][:, heads])
    others = [h for h in range(SHAPE.n_v_heads) if h not in heads]
    assert np.isnan(y[:, others]).all() and np.isnan(fin[:, others]).all()
    assert np.array_equal(cs, full[2])


@pytest.mark.parametrize("heads", SUBSETS)
def test_prefill_subset_equals_whole_layer(problem, heads):
    inp, full = problem
    _assert_subset_matches(inp, full, heads)


def test_prefill_subset_without_states(oracle_lib):
    inp = gi.make_prefill_inputs(SHAPE, [64, 1, 66], gi.BF16, seed=99)
    full = oracle.prefill(inp)
    for heads in SUBSETS:
        y, fin, _ = oracle.prefill(inp, heads=heads)
        assert np.array_equal(y[:, heads], full[0][:, heads])
        assert np.array_equal(fin[:, heads], full[1][:, heads])


def test_decode_subset_equals_all_heads(oracle_lib):
    B, steps = 3, 4
    dec = gi.make_decode_inputs(SHAPE, B, steps, gi.BF16, seed=555)
    w = gi.make_conv_weights(SHAPE, 555)
    rng = np.random.default_rng(7)
    state = 0.2 * rng.standard_normal((B, SHAPE.n_v_heads, 128, 128))
    conv = gi.quantize(rng.standard_normal((B, 3, SHAPE.channels)).astype(np.float32), gi.BF16)
    ys, st, cs = oracle.decode_steps(SHAPE, gi.BF16, dec, w, state, conv)
    for heads in SUBSETS:
        for rows in (None, [2, 0]):
            r = np.arange(B) if rows is None else np.asarray(rows)
            ys_h, st_h, cs_h = oracle.decode_steps(SHAPE, gi.BF16, dec, w, state, conv, rows=rows,
                                                   heads=heads)
            assert np.array_equal(ys_h[:, :, heads], ys[:, r][:, :, heads])
            assert np.array_equal(st_h[:, heads], st[r][:, heads])
            assert np.array_equal(cs_h, cs[r])


# ----------------------------------------------------------------------------- planted slips
def _cols_k_offset(shape, groups, vheads):
    """Slip: the k channels of the conv state taken one head too far."""
    dk, dv = shape.d_k, shape.d_v
    qkc = shape.n_qk_heads * dk
    qch = [g * dk + i for g in groups for i in range(dk)]
    vch = [h * dv + i for h in vheads for i in range(dv)]
    return qch + [(qkc + c + dk) % (2 * qkc) for c in qch] + [2 * qkc + c for c in vch]


def _cols_q_for_k(shape, groups, vheads):
    """Slip: the q history reused for k."""
    dk, dv = shape.d_k, shape.d_v
    qkc = shape.n_qk_heads * dk
    qch = [g * dk + i for g in groups for i in range(dk)]
    vch = [h * dv + i for h in vheads for i in range(dv)]
    return qch + qch + [2 * qkc + c for c in vch]


def _remap_in_group_only(shape, heads):
    """Slip: a requested head mapped by its place inside its group, forgetting the group's
    position among the sliced groups."""
    G = shape.n_v_heads // shape.n_qk_heads
    groups = sorted({int(h) // G for h in heads})
    vheads = [g * G + j for g in groups for j in range(G)]
    return groups, vheads, [int(h) % G for h in heads]


def _groups_by_modulo(shape, heads):
    """Slip: an interleaved head map (h mod Hqk) inside the subset path only."""
    G = shape.n_v_heads // shape.n_qk_heads
    groups = sorted({int(h) % shape.n_qk_heads for h in heads})
    vheads = [g * G + j for g in groups for j in range(G)]
    remap = [groups.index(int(h) % shape.n_qk_heads) * G + int(h) % G for h in heads]
    return groups, vheads, remap


@pytest.mark.parametrize("name,attr,slip", [
    ("k-channel offset in the conv-state columns", "_conv_state_columns", _cols_k_offset),
    ("q history used for k", "_conv_state_columns", _cols_q_for_k),
    ("remap ignores the group position", "_group_slices", _remap_in_group_only),
    ("groups chosen by h mod Hqk", "_group_slices", _groups_by_modulo),
])
def test_planted_subset_slips_are_caught(problem, monkeypatch, name, attr, slip):
    inp, full = problem
    monkeypatch.setattr(oracle, attr, slip)
    caught = 0
    for heads in SUBSETS:
        try:
            _assert_subset_matches(inp, full, heads)
        except AssertionError:
            caught += 1
    assert caught > 0, name
