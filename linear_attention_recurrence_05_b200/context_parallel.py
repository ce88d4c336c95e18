"""Context-parallel prefill of one long sequence, split into consecutive spans.

The gated delta rule (page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03) is affine in
the state entering a span: for fixed keys, gates and values of the span,

    S_out = M S_in + B,

with M (d_k x d_k) the product of the span's per-token maps alpha_t (I - beta_t k_t k_t^T)
and B the state the span leaves from a zero state.  So each span can be processed
independently: its B is the final state of a prefill from zero, and its M the final state of
a prefill of the same keys and gates with zero values from the identity state (then
S_out = M I + 0).  Combining the maps of the spans before it gives a span's true entering
state, and one more prefill from that state gives the span's outputs.

Two drivers share that plan: ``cp_prefill`` runs the spans of a process group's ranks
(one span each; one all-gather of 2 x Hv x 128 x 128 fp32 per rank is the only exchange),
``cp_prefill_spans`` runs a list of spans one after another in one process.  Both take the
prefill as a callable with the signature of :func:`gdn_prefill` (the default) and the
combination of the maps as a callable with the signature of :func:`affine_combine` (the
default; both run in libgdn), and return each span's outputs and final state.  This module
itself only moves data: the sequence's conv history is carried between spans as the 3 raw
rows before each span.
"""
from __future__ import annotations

import torch

__all__ = ["span_affine_map", "combine_prefix", "cp_prefill_spans", "cp_prefill"]


def _v_channel_slice(cfg):
    qkc = cfg.n_qk_heads * cfg.d_k
    return slice(2 * qkc, 2 * qkc + cfg.n_v_heads * cfg.d_v)


def _one(cu_device, T):
    return torch.tensor([0, T], dtype=torch.int32, device=cu_device)


def span_affine_map(prefill, q, k, v, w, alpha, beta, *, cfg, conv_rows=None):
    """(M, B) of one span: each [Hv, 128, 128] fp32, S_out = M @ S_in + B per V head.

    ``conv_rows``: [3, channels] raw rows before the span (None = zero history).
    """
    T, dev = q.shape[0], q.device
    cu = _one(dev, T)
    cs = None if conv_rows is None else conv_rows.unsqueeze(0)
    _, B, _ = prefill(q, k, v, *w, alpha, beta, cu, cfg=cfg, initial_state=None, conv_state_in=cs)
    # the linear part: zero values (and zero value history), identity state
    cs0 = None
    if cs is not None:
        cs0 = cs.clone()
        cs0[..., _v_channel_slice(cfg)] = 0
    eye = torch.eye(cfg.d_k, dtype=torch.float32, device=dev).expand(1, cfg.n_v_heads, cfg.d_k, cfg.d_v)
    _, M, _ = prefill(q, k, torch.zeros_like(v), *w, alpha, beta, cu, cfg=cfg,
                      initial_state=eye.contiguous(), conv_state_in=cs0)
    return M[0], B[0]


def combine_prefix(Ms, Bs, S0, combine=None):
    """Entering states of spans 0..P-1: S_0 = S0, S_{p+1} = M_p S_p + B_p (per V head), by
    ``combine`` (default: libgdn's gdn_affine_combine)."""
    if combine is None:
        from . import affine_combine as combine
    def stacked(xs):
        if len(xs) > 1:
            return torch.stack(xs[:-1]).contiguous()
        return torch.empty((0,) + tuple(S0.shape), dtype=S0.dtype, device=S0.device)
    S = combine(stacked(Ms), stacked(Bs), S0.contiguous())
    return list(S.unbind(0))


def _last_rows(x_q, x_k, x_v, prev_rows, n=3):
    """The last n raw rows (q | k | v channels) of the prefix ending with this span."""
    T = x_q.shape[0]
    cur = torch.cat([x_q.reshape(T, -1), x_k.reshape(T, -1), x_v.reshape(T, -1)], dim=1)
    if prev_rows is not None:
        cur = torch.cat([prev_rows.to(cur.dtype), cur], dim=0)
    elif T < n:
        cur = torch.cat([torch.zeros((n - T, cur.shape[1]), dtype=cur.dtype, device=cur.device), cur], dim=0)
    return cur[-n:]


def cp_prefill_spans(spans, w, *, cfg, initial_state=None, conv_state=None, prefill=None, combine=None):
    """Spans of one sequence in one process.  ``spans``: list of (q, k, v, alpha, beta) of
    consecutive pieces; ``initial_state`` [Hv, 128, 128] or None; ``conv_state`` [3, channels]
    raw rows before the sequence or None.  Returns (list of y per span, final state)."""
    if prefill is None:
        from . import gdn_prefill as prefill
    rows, r = [], conv_state
    for (q, k, v, _, _) in spans:   # conv history entering each span
        rows.append(r)
        r = _last_rows(q, k, v, r)
    maps = [span_affine_map(prefill, q, k, v, w, a, b, cfg=cfg, conv_rows=rw)
            for (q, k, v, a, b), rw in zip(spans, rows)]
    dev = spans[0][0].device
    S0 = initial_state if initial_state is not None else torch.zeros(
        (cfg.n_v_heads, cfg.d_k, cfg.d_v), dtype=torch.float32, device=dev)
    S_in = combine_prefix([m for m, _ in maps], [b for _, b in maps], S0, combine)
    ys, fin = [], None
    for (q, k, v, a, b), rw, S in zip(spans, rows, S_in):
        y, f, _ = prefill(q, k, v, *w, a, b, _one(dev, q.shape[0]), cfg=cfg,
                          initial_state=S.unsqueeze(0).contiguous(),
                          conv_state_in=None if rw is None else rw.unsqueeze(0))
        ys.append(y)
        fin = f[0]
    return ys, fin


def cp_prefill(q, k, v, w, alpha, beta, *, cfg, group=None, initial_state=None, conv_state=None,
               prefill=None, combine=None):
    """This rank's span of one sequence (rank order = sequence order).  ``initial_state`` and
    ``conv_state`` are the sequence's (only rank 0's are used).  One all-gather carries every
    span's (M, B) and last raw rows.  Returns (y of this span, final state of the sequence
    after this span)."""
    import torch.distributed as dist
    if prefill is None:
        from . import gdn_prefill as prefill
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    dev = q.device
    Hv, d = cfg.n_v_heads, cfg.d_k
    # every span's last 3 raw rows (its own prefix only: the rows before it come from the
    # previous ranks, so spans must hold at least 3 tokens; all ranks check all lengths)
    lens = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(world)]
    dist.all_gather(lens, torch.tensor([q.shape[0]], dtype=torch.int64, device=dev), group=group)
    if min(int(x.item()) for x in lens) < 3:
        raise ValueError("every span needs at least 3 tokens")
    mine = _last_rows(q, k, v, None).to(torch.float32).contiguous()
    rows = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(rows, mine, group=group)
    if rank == 0:
        conv_rows = conv_state
    else:
        conv_rows = rows[rank - 1].to(q.dtype)
    M, B = span_affine_map(prefill, q, k, v, w, alpha, beta, cfg=cfg, conv_rows=conv_rows)
    both = torch.stack([M, B]).contiguous()
    got = [torch.empty_like(both) for _ in range(world)]
    dist.all_gather(got, both, group=group)
    S0 = torch.zeros((Hv, d, d), dtype=torch.float32, device=dev)
    if initial_state is not None:
        S0 = initial_state.to(torch.float32)
    src = torch.stack([S0]) if rank == 0 else torch.empty((1, Hv, d, d), dtype=torch.float32, device=dev)
    dist.broadcast(src, 0, group=group)   # the sequence's initial state, from rank 0
    S = combine_prefix([g[0] for g in got[:rank + 1]], [g[1] for g in got[:rank + 1]], src[0], combine)[rank]
    y, fin, _ = prefill(q, k, v, *w, alpha, beta, _one(dev, q.shape[0]), cfg=cfg,
                        initial_state=S.unsqueeze(0).contiguous(),
                        conv_state_in=None if conv_rows is None else conv_rows.unsqueeze(0))
    return y, fin[0]
