"""Parity of the QSA indexer kernels with the fp64 oracle (GPU, through the C ABI).

Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03, QSA indexer figure.  The oracle
recomputes everything from the same seeded raw inputs in fp64, with the block keys and query
heads either exact ("exact" operands, the reference) or rounded to bf16 ("bf16" operands, the
precision the kernels chose for their MMA operands; used only for the tight checks below).

Bounds, from the arithmetic:
  * block keys: the kernel rounds an fp32 value, the oracle the exact one, to bf16, so an
    entry may differ by one bf16 unit in the last place (at most 2^-7 of its magnitude), and
    only where the fp32 value fell next to a rounding boundary (a small fraction).
  * scores: each operand the kernel multiplies is within half a bf16 unit (2^-8 of its
    magnitude) of the exact operand, and within one unit of the oracle's bf16 operand; the
    kernel accumulates in fp32.  Either way |I_kernel - I_oracle| <= 2^-7 A + 2^-16 A with
    A = sum_h sum_d |qh_hd| |kbar_bd|: checked against the exact scores.  Against the bf16-
    operand scores the rms difference must also be far below that (1e-4 of the rms).
  * selection: several block sets are correct when scores nearly tie.  Any selection that
    is a top-512 of scores within the bound above satisfies
    min_selected (I + delta) >= max_unselected (I - delta) for the EXACT scores I; beyond
    that, the kernel's set must agree with the top-512 of the bf16-operand scores on at least
    99% of its entries.  Counts, order, padding and the token sets are exact.
"""
import zlib

import numpy as np
import pytest

import gdn_inputs as gi
from gdn_testutil import to_dev
from oracle import qsa_indexer as qi

pytestmark = pytest.mark.gpu

EPS, THETA = 1e-6, 10000.0


def _mods():
    import torch
    import linear_attention_recurrence_05_b200 as gdn
    return torch, gdn


def _i32(torch, a):
    return torch.tensor(np.asarray(a, dtype=np.int32), device="cuda")


def _host(t):
    import torch
    return t.to(torch.float64).cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def _keys_f64(inp):
    return gi.bf16_bits_to_f32(inp.k).astype(np.float64)


def _q_f64(inp):
    return gi.bf16_bits_to_f32(inp.q).astype(np.float64)


def _build_cache(torch, gdn, inp, nb_max, kpos=None, fill=0.0):
    B, T = inp.k.shape[:2]
    kbar = torch.full((B, nb_max, 128), fill, dtype=torch.bfloat16, device="cuda")
    kp = _i32(torch, kpos if kpos is not None else [0] * B)
    k = to_dev(np.ascontiguousarray(inp.k[:, :T - T % 4]), "bf16")    # complete blocks only
    gdn.qsa_block_keys(k, to_dev(inp.w_k, "f32"), kp, kbar, eps=EPS, theta=THETA)
    return kbar


# ----------------------------------------------------------------------------- block keys
def test_block_keys():
    torch, gdn = _mods()
    B, T = 5, 96
    inp = gi.make_qsa_inputs(B, T, 1, seed=101)
    nb_max = 262160
    kpos = [0, 8, 4096, 4 * (nb_max - 2), (1 << 20) - 4 * 30]   # row 3: only 2 blocks fit
    kbar = _build_cache(torch, gdn, inp, nb_max, kpos, fill=7.0)
    k64 = _keys_f64(inp)
    diff_frac, written = [], 0
    for b in range(B):
        ref = qi.block_keys(k64[b], inp.w_k, EPS, THETA, pos0=kpos[b], operands="bf16")
        j0 = kpos[b] // 4
        n = min(T // 4, nb_max - j0)
        g = _host(kbar[b, j0:j0 + n])
        r = ref[:n]
        assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.maximum(np.abs(r), np.abs(g)) + 1e-30), b
        diff_frac.append(np.mean(g != r))
        written += n
    # nothing outside the written blocks changed
    assert int((kbar != 7.0).any(dim=-1).sum()) <= written
    for b in range(B):
        j0 = kpos[b] // 4
        n = min(T // 4, nb_max - j0)
        assert bool((kbar[b, :j0] == 7.0).all()) and bool((kbar[b, j0 + n:] == 7.0).all()), b
    assert max(diff_frac) < 0.02, diff_frac


def test_block_keys_rejects_misaligned_rows():
    torch, gdn = _mods()
    inp = gi.make_qsa_inputs(2, 16, 1, seed=102)
    kbar = _build_cache(torch, gdn, inp, 64, kpos=[6, -4], fill=3.0)
    assert torch.all(kbar == 3.0)          # positions not on a block boundary write nothing


# ----------------------------------------------------------------------------- scores
SCORE_CASES = {
    # name: (B, T, Qn, qpos per row, n_blocks per row or None = T // 4, nb_max)
    "tiny": (2, 300, 37, [263, 0], None, 75),
    "tiles": (1, 2000, 150, [1850], None, 500),              # 4 key tiles (last ragged), 3 query tiles
    "decode": (5, 1200, 1, [1199, 600, 3, 1000, 1199], [300, 150, 300, 10, 300], 300),
    "mtp4": (3, 1000, 4, [996, 500, 2], None, 250),
    "odd_q": (2, 777, 5, [700, 771], None, 194),
}


def _oracle_scores(inp, b, qpos_b, Qn, n_blocks_b, T, operands="exact"):
    k64, q64 = _keys_f64(inp), _q_f64(inp)
    kb = qi.block_keys(k64[b, :T], inp.w_k, EPS, THETA, operands=operands)
    pos = qpos_b + np.arange(Qn)
    qh = qi.query_heads(q64[b], inp.w_q, pos, EPS, THETA, operands=operands)
    s = qi.block_scores(qh, kb, pos, n_blocks_b)
    A = np.einsum("nhd,bd->nb", np.abs(qh), np.abs(kb))
    return s, A, pos


@pytest.mark.parametrize("name", list(SCORE_CASES))
def test_block_scores(name):
    torch, gdn = _mods()
    B, T, Qn, qpos, nblk, nb_max = SCORE_CASES[name]
    nblk = nblk or [T // 4] * B
    inp = gi.make_qsa_inputs(B, T, Qn, seed=zlib.crc32(name.encode()) % 10000)
    kbar = _build_cache(torch, gdn, inp, nb_max)
    sc = gdn.qsa_block_scores(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, qpos), kbar,
                              _i32(torch, nblk), eps=EPS, theta=THETA)
    got = _host(sc)
    checked = 0
    for b in range(B):
        ref, A, _ = _oracle_scores(inp, b, qpos[b], Qn, nblk[b], T)               # exact operands
        rbf, _, _ = _oracle_scores(inp, b, qpos[b], Qn, nblk[b], T, "bf16")     # the kernels' choice
        fin = np.isfinite(ref[:, :nb_max])
        g, r, a = got[b][fin], ref[:, :nb_max][fin], A[:, :nb_max][fin]
        assert np.all(np.abs(g - r) <= (2.0 ** -7 + 2.0 ** -16) * a), name
        rb = rbf[:, :nb_max][fin]
        if r.size:
            assert np.sqrt(np.mean((g - rb) ** 2)) <= 1e-4 * np.sqrt(np.mean(rb ** 2)) + 1e-12, name
        checked += r.size
    assert checked > 0


# ----------------------------------------------------------------------------- selection
def _check_row(blocks, tokens, s, A, i, nvis, s_bf16=None):
    """One query's block set (and token set) against the oracle's exact scores s [nb] and
    bound A; the overlap is taken with the top-512 of the bf16-operand scores s_bf16."""
    sel = blocks[blocks >= 0]
    m = min(nvis, qi.K_B)
    assert len(sel) == m and np.all(blocks[m:] == -1)
    assert np.all(np.diff(sel) > 0) and (m == 0 or (sel[0] >= 0 and sel[-1] < nvis))
    overlap = 1.0
    if nvis > qi.K_B:
        cand = s[:nvis]
        delta = (2.0 ** -7 + 2.0 ** -16) * A[:nvis]
        mask = np.zeros(nvis, dtype=bool)
        mask[sel] = True
        assert np.min(cand[mask] + delta[mask]) >= np.max(cand[~mask] - delta[~mask])
        ref = qi.top_blocks(cand if s_bf16 is None else s_bf16[:nvis], qi.K_B)
        overlap = len(np.intersect1d(ref, sel)) / qi.K_B
    if tokens is not None:
        want = np.full(qi.TOKEN_SLOTS, -1, dtype=np.int64)
        want[:4 * m] = (4 * sel[:, None] + np.arange(4)).reshape(-1)
        t0 = 4 * ((i + 1) // 4)
        tail = np.arange(t0, i + 1)
        want[4 * m:4 * m + len(tail)] = tail
        assert np.array_equal(tokens, want)
    return overlap


SELECT_CASES = {
    # name: (B, T, Qn, qpos, n_blocks or None, nb_max)
    "budget_edge": (2, 6000, 70, [5930, 2000], None, 1500),     # row 1 crosses 512 candidates
    "short": (2, 400, 33, [367, 0], None, 100),                 # fewer candidates than the budget
    "capped": (3, 5000, 6, [4994, 4994, 4994], [1250, 700, 300], 1250),
    "decode": (4, 9000, 1, [8999, 8000, 2500, 8999], None, 2250),
}


@pytest.mark.parametrize("name", list(SELECT_CASES))
def test_select(name):
    torch, gdn = _mods()
    B, T, Qn, qpos, nblk, nb_max = SELECT_CASES[name]
    nblk = nblk or [T // 4] * B
    inp = gi.make_qsa_inputs(B, T, Qn, seed=zlib.crc32(name.encode()) % 10000 + 7)
    kbar = _build_cache(torch, gdn, inp, nb_max)
    blocks, tokens = gdn.qsa_select(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, qpos), kbar,
                                    _i32(torch, nblk), eps=EPS, theta=THETA, with_tokens=True)
    bl, tk = _host(blocks), _host(tokens)
    overlaps = []
    for b in range(B):
        s, A, pos = _oracle_scores(inp, b, qpos[b], Qn, nblk[b], T)
        sb, _, _ = _oracle_scores(inp, b, qpos[b], Qn, nblk[b], T, "bf16")
        for j in range(Qn):
            nvis = qi.n_complete(pos[j], min(nblk[b], nb_max))
            overlaps.append(_check_row(bl[b, j], tk[b, j], s[j], A[j], int(pos[j]), nvis, sb[j]))
    assert np.mean(overlaps) >= 0.99 and min(overlaps) >= 0.97, (np.mean(overlaps), min(overlaps))


@pytest.mark.parametrize("T", [4096, 32768])
def test_select_ties_take_lower_blocks(T):
    """Identical block keys (same raw keys, rotated dims weighted 0) give identical scores:
    the first 512 candidates are selected (T = 32768: more equal scores than the candidate
    set holds, so the row takes the full-row path)."""
    torch, gdn = _mods()
    B, Qn = 1, 3
    inp = gi.make_qsa_inputs(B, T, Qn, seed=55)
    inp.k[:] = inp.k[:, :1, :]                 # every token the same key row
    inp.w_k[:64] = 0.0                          # nothing left for the rotation to move
    kbar = _build_cache(torch, gdn, inp, T // 4)
    qpos = [T - Qn]
    blocks, tokens = gdn.qsa_select(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, qpos), kbar,
                                    _i32(torch, [T // 4]), eps=EPS, theta=THETA, with_tokens=True)
    bl = _host(blocks)
    for j in range(Qn):
        assert np.array_equal(bl[0, j], np.arange(512)), j
    # and the oracle agrees (its tie rule is the same)
    s, A, pos = _oracle_scores(inp, 0, qpos[0], Qn, T // 4, T)
    assert np.array_equal(qi.top_blocks(s[0], 512), np.arange(512))


# ----------------------------------------------------------------------------- full size
@pytest.mark.parametrize("wl", ["prefill", "decode"])
def test_select_full_size_sampled(wl):
    """The benchmarked workloads, in the launch configuration bench.py times; every row's
    structure is checked on the device, sampled rows against the oracle."""
    torch, gdn = _mods()
    cfg = gi.QSA_PREFILL if wl == "prefill" else gi.QSA_DECODE
    B = cfg["B"] if wl == "prefill" else 4          # 4 of the 64 decode rows (same per-row shape)
    T, Qn = cfg["context"], cfg["queries"]
    nb = T // 4
    inp = gi.make_qsa_inputs(B, T, Qn, seed=2024 + len(wl))
    kbar = _build_cache(torch, gdn, inp, nb)
    qpos = [T - Qn] * B
    blocks, tokens = gdn.qsa_select(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, qpos), kbar,
                                    _i32(torch, [nb] * B), eps=cfg["eps"], theta=cfg["theta"], with_tokens=True)
    torch.cuda.synchronize()
    # every row: 512 distinct ascending candidates
    assert bool((blocks >= 0).all()) and bool((blocks[..., 1:] > blocks[..., :-1]).all())
    lim = torch.tensor([(T - Qn + j + 1) // 4 for j in range(Qn)], device="cuda", dtype=torch.int32)
    assert bool((blocks < lim[None, :, None]).all())
    rng = np.random.default_rng(3)
    rows = sorted(set([0, Qn - 1] + list(rng.integers(0, Qn, 10))))
    k64, q64 = _keys_f64(inp), _q_f64(inp)
    overlaps = []
    for b in range(B):
        kb = qi.block_keys(k64[b], inp.w_k, cfg["eps"], cfg["theta"], operands="exact")
        kbb = qi.block_keys(k64[b], inp.w_k, cfg["eps"], cfg["theta"], operands="bf16")
        for j in rows:
            i = T - Qn + j
            qh = qi.query_heads(q64[b, j:j + 1], inp.w_q, [i], cfg["eps"], cfg["theta"], operands="exact")
            qhb = qi.query_heads(q64[b, j:j + 1], inp.w_q, [i], cfg["eps"], cfg["theta"], operands="bf16")
            s = qi.block_scores(qh, kb, [i])[0]
            sb = qi.block_scores(qhb, kbb, [i])[0]
            A = np.einsum("hd,bd->b", np.abs(qh[0]), np.abs(kb))
            overlaps.append(_check_row(_host(blocks[b, j]), _host(tokens[b, j]), s, A, i,
                                       qi.n_complete(i, nb), sb))
    assert np.mean(overlaps) >= 0.99, overlaps


@pytest.mark.parametrize("ties", [False, True])
def test_select_long_rows(ties):
    """Rows of more than 32768 candidate blocks (the CTA-per-query selection): random scores
    take the sampled candidate path, identical scores the full-row path."""
    torch, gdn = _mods()
    B, T, Qn = 2, 160000, 3
    nb = T // 4
    inp = gi.make_qsa_inputs(B, T, Qn, seed=31 + int(ties))
    if ties:
        inp.k[:] = inp.k[:, :1, :]
        inp.w_k[:64] = 0.0
    kbar = _build_cache(torch, gdn, inp, nb)
    qpos = [T - Qn, T - 50000]
    blocks, tokens = gdn.qsa_select(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, qpos), kbar,
                                    _i32(torch, [nb] * B), eps=EPS, theta=THETA, with_tokens=True)
    bl, tk = _host(blocks), _host(tokens)
    overlaps = []
    for b in range(B):
        s, A, pos = _oracle_scores(inp, b, qpos[b], Qn, nb, T)
        sb, _, _ = _oracle_scores(inp, b, qpos[b], Qn, nb, T, "bf16")
        for j in range(Qn):
            nvis = qi.n_complete(pos[j], nb)
            overlaps.append(_check_row(bl[b, j], tk[b, j], s[j], A[j], int(pos[j]), nvis, sb[j]))
            if ties:
                assert np.array_equal(bl[b, j], np.arange(512))
    assert np.mean(overlaps) >= 0.99, overlaps


@pytest.mark.parametrize("ties", [False, True])
def test_select_many_queries(ties):
    """2048 queries (the warp-per-query selection).  Random scores: positions 1900..3947 cross
    the budget (<= 512 candidates, all candidates, then the sampled threshold) and every row is
    checked; identical scores take the full-row path and give blocks 0..511."""
    torch, gdn = _mods()
    B, Qn = 1, 2048
    T = 32768 if ties else 12000
    q0 = T - Qn if ties else 1900
    nb = T // 4
    inp = gi.make_qsa_inputs(B, T, Qn, seed=57 + int(ties))
    if ties:
        inp.k[:] = inp.k[:, :1, :]
        inp.w_k[:64] = 0.0
    kbar = _build_cache(torch, gdn, inp, nb)
    blocks, tokens = gdn.qsa_select(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, [q0]), kbar,
                                    _i32(torch, [nb]), eps=EPS, theta=THETA, with_tokens=True)
    bl, tk = _host(blocks), _host(tokens)
    if ties:
        assert np.array_equal(bl[0], np.broadcast_to(np.arange(512), (Qn, 512)))
        return
    s, A, pos = _oracle_scores(inp, 0, q0, Qn, nb, T)
    sb, _, _ = _oracle_scores(inp, 0, q0, Qn, nb, T, "bf16")
    overlaps = [_check_row(bl[0, j], tk[0, j], s[j], A[j], int(pos[j]), qi.n_complete(pos[j], nb), sb[j])
                for j in range(Qn)]
    assert np.mean(overlaps) >= 0.99 and min(overlaps) >= 0.97, (np.mean(overlaps), min(overlaps))


def test_select_degenerate_rows():
    """Clamped device-side values: a row of negative query positions (no candidates, no tail),
    a row whose cache holds no valid block (tail tokens only), and a normal row."""
    torch, gdn = _mods()
    B, T, Qn, nb_max = 3, 6400, 5, 1600
    inp = gi.make_qsa_inputs(B, T, Qn, seed=77)
    kbar = _build_cache(torch, gdn, inp, nb_max)
    qpos, nblk = [-10, 10, 6000], [100, 0, 1600]
    blocks, tokens = gdn.qsa_select(to_dev(inp.q, "bf16"), to_dev(inp.w_q, "f32"), _i32(torch, qpos), kbar,
                                    _i32(torch, nblk), eps=EPS, theta=THETA, with_tokens=True)
    bl, tk = _host(blocks), _host(tokens)
    assert np.all(bl[0] == -1) and np.all(tk[0] == -1)
    assert np.all(bl[1] == -1)
    for j in range(Qn):
        i = qpos[1] + j
        want = np.full(qi.TOKEN_SLOTS, -1)
        tail = np.arange(4 * ((i + 1) // 4), i + 1)
        want[:len(tail)] = tail
        assert np.array_equal(tk[1, j], want), j
    s, A, pos = _oracle_scores(inp, 2, qpos[2], Qn, nblk[2], T)
    sb, _, _ = _oracle_scores(inp, 2, qpos[2], Qn, nblk[2], T, "bf16")
    ov = [_check_row(bl[2, j], tk[2, j], s[j], A[j], int(pos[j]), qi.n_complete(pos[j], nblk[2]), sb[j])
          for j in range(Qn)]
    assert min(ov) >= 0.97
