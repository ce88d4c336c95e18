"""fp64 reference of the QSA indexer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU leg may use it; the
product never imports it and shares no code with it.

Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (the QSA indexer figure, its BLOCK
SCORE and CAUSAL SPARSE SET formulas and the five-step list under "QSA"), with the
config table of section 01 (indexer: 4 query heads sharing 1 key head, head dim 128,
budget 512 blocks = 2048 tokens):

  key side     the indexer keys of r = 4 consecutive tokens are averaged into one block key,
               RMS-normalised, and given a partial rotary encoding (64 of the 128 dims) at
               the block's position;
  query side   each of the 4 query heads of a token is RMS-normalised and given the same
               partial rotary encoding at the token's own position;
  block score  I[i, b] = sum over the 4 heads of ReLU(<q_i^h, kbar_b>) when block b is
               complete at token i (p_b + r - 1 <= i, p_b = r b its first token), else -inf;
  block set    B_i = the K_B = 512 highest-scoring blocks (all complete blocks when fewer);
  token set    S_i = the tokens of the blocks of B_i, plus the tokens of the current
               incomplete block: r floor((i + 1) / r), ..., i.

Readings where the page leaves a step open (each also listed in the design notes):
  * RMSNorm: x / sqrt(mean(x^2) + eps) * w, with one weight vector of 128 for the keys and
    one shared by the 4 query heads; eps a parameter (default 1e-6).
  * Rotary encoding: the first 64 dims rotate, dim d paired with dim d + 32 (d < 32) at
    angle pos * theta^(-d / 32), dims 64..127 pass unchanged; theta is not printed on the
    pages and is a parameter (default 10000).
  * A block's position is its first token's position p_b = r b, in the same units as the
    query position i.
  * Equal scores: the lower block index ranks first.  B_i is returned in ascending block
    order, padded with -1 to K_B entries; S_i ascending, padded with -1 to r K_B + r - 1.
  * Precision: the score's operands (the rotated query heads and block keys) are rounded
    to bf16 when ``operands="bf16"`` (the precision the selection is taken in on the GPU);
    ``operands="exact"`` keeps them in fp64.
"""
from __future__ import annotations

import numpy as np

R = 4            # tokens per block
D_I = 128        # indexer head dim
H_I = 4          # indexer query heads (one shared key head)
ROPE_DIMS = 64   # rotated dims of the 128
K_B = 512        # block budget
TOKEN_SLOTS = R * K_B + R - 1


def bf16_round(x):
    """Round fp64 values to the nearest bf16 (8 significant bits, ties to even), in fp64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def rms_norm(x, w, eps):
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def rope_partial(x, pos, theta):
    """Rotate dims (d, d + 32), d < 32, of x [..., 128] by pos * theta^(-d/32); pos
    broadcasts against x's leading axes."""
    x = np.array(x, dtype=np.float64)
    half = ROPE_DIMS // 2
    freq = theta ** (-np.arange(half, dtype=np.float64) / half)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half].copy(), x[..., half:ROPE_DIMS].copy()
    x[..., :half] = a * c - b * s
    x[..., half:ROPE_DIMS] = b * c + a * s
    return x


def block_keys(k, w_k, eps=1e-6, theta=10000.0, pos0=0, operands="exact"):
    """k [T, 128] indexer keys of tokens pos0 .. pos0 + T - 1 (pos0 % r == 0) ->
    kbar [T // r, 128]: block j covers tokens pos0 + r j .. pos0 + r j + r - 1."""
    k = np.asarray(k, dtype=np.float64)
    nb = k.shape[0] // R
    pooled = k[:nb * R].reshape(nb, R, D_I).mean(axis=1)
    p = pos0 + R * np.arange(nb)
    out = rope_partial(rms_norm(pooled, w_k, eps), p, theta)
    return bf16_round(out) if operands == "bf16" else out


def query_heads(q, w_q, pos, eps=1e-6, theta=10000.0, operands="exact"):
    """q [n, 4, 128] indexer query heads of tokens at positions pos [n] -> rotated heads."""
    q = np.asarray(q, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    out = rope_partial(rms_norm(q, w_q, eps), pos[:, None], theta)
    return bf16_round(out) if operands == "bf16" else out


def n_complete(i, n_blocks=None):
    """Blocks complete at token i (those with r b + r - 1 <= i), capped by the cache size."""
    n = max(0, (int(i) + 1) // R)
    return n if n_blocks is None else min(n, int(n_blocks))


def block_scores(qh, kbar, pos, n_blocks=None):
    """qh [n, 4, 128], kbar [nb, 128] -> I [n, nb]: sum_h ReLU(<q^h, kbar_b>), -inf where
    block b is not complete at the query's position (or lies beyond n_blocks)."""
    dots = np.einsum("nhd,bd->nhb", qh, kbar)
    score = np.maximum(dots, 0.0).sum(axis=1)
    nb = kbar.shape[0]
    for r, i in enumerate(np.asarray(pos)):
        score[r, n_complete(i, n_blocks):nb] = -np.inf
    return score


def top_blocks(score_row, k_b=K_B):
    """The k_b highest finite scores of one row (ties: lower index first), returned in
    ascending block order and padded with -1 to k_b entries."""
    s = np.asarray(score_row, dtype=np.float64)
    idx = np.flatnonzero(np.isfinite(s))
    order = idx[np.lexsort((idx, -s[idx]))][:k_b]
    out = np.full(k_b, -1, dtype=np.int64)
    out[:len(order)] = np.sort(order)
    return out


def token_set(blocks, i, k_b=K_B):
    """S_i: the r tokens of every selected block, then the current incomplete block's
    tokens r floor((i + 1) / r) .. i; padded with -1 to r k_b + r - 1 entries."""
    sel = [int(b) for b in blocks if b >= 0]
    toks = [R * b + t for b in sel for t in range(R)]
    toks += list(range(R * ((int(i) + 1) // R), int(i) + 1))
    out = np.full(R * k_b + R - 1, -1, dtype=np.int64)
    out[:len(toks)] = toks
    return out


def indexer(q, k, w_q, w_k, q_pos, eps=1e-6, theta=10000.0, operands="bf16", k_b=K_B,
            n_blocks=None):
    """End to end for one sequence: keys k [T, 128] of tokens 0 .. T - 1, queries
    q [n, 4, 128] at positions q_pos -> (kbar, scores [n, nb], blocks [n, k_b],
    tokens [n, r k_b + r - 1])."""
    kbar = block_keys(k, w_k, eps, theta, 0, operands)
    qh = query_heads(q, w_q, q_pos, eps, theta, operands)
    score = block_scores(qh, kbar, q_pos, n_blocks)
    blocks = np.full((len(score), k_b), -1, dtype=np.int64)
    tokens = np.full((len(score), R * k_b + R - 1), -1, dtype=np.int64)
    for r, i in enumerate(q_pos):
        blocks[r] = top_blocks(score[r], k_b)
        tokens[r] = token_set(blocks[r], i, k_b)
    return kbar, score, blocks, tokens
