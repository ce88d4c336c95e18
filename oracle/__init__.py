"""fp64 CPU oracle of the Gated DeltaNet token mixer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
Python binding) never imports, links or runs it, and it shares no code with it.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, OpenMP over
(sequence, V head) units).  This module only builds it with gcc and marshals
numpy arrays through ctypes: the stored inputs (bf16 bits or fp32) are widened to
fp64 exactly before the call.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LOCK = threading.Lock()
_LIBS: dict = {}


class OracleShape(ctypes.Structure):
    _fields_ = [("n_qk_heads", ctypes.c_int), ("n_v_heads", ctypes.c_int),
                ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("conv_width", ctypes.c_int),
                ("q_scale", ctypes.c_double), ("l2_eps", ctypes.c_double), ("conv_silu", ctypes.c_int)]


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mut{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile gdn_oracle.c (optionally with one planted mistake) into a shared library."""
    out = lib_path(mutant)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    os.makedirs(_BUILD, exist_ok=True)
    tmp = f"{out}.{os.getpid()}.tmp"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-Wall", "-Wextra",
           f"-DGDN_ORACLE_MUTANT={mutant}", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


def _lib(mutant: int = 0):
    with _LOCK:
        if mutant not in _LIBS:
            lib = ctypes.CDLL(build(mutant))
            P = ctypes.POINTER
            d = P(ctypes.c_double)
            i32 = P(ctypes.c_int32)
            lib.oracle_gdn_prefill.argtypes = [P(OracleShape), d, d, d, d, d, d, d, d, i32,
                                               ctypes.c_int, d, d, i32, ctypes.c_int, d, d, d,
                                               ctypes.c_int]
            lib.oracle_gdn_prefill.restype = ctypes.c_int
            lib.oracle_gdn_conv_l2.argtypes = [P(OracleShape), d, d, d, d, d, d, i32, ctypes.c_int,
                                               d, d, d, d, ctypes.c_int]
            lib.oracle_gdn_conv_l2.restype = ctypes.c_int
            lib.oracle_mutant_id.restype = ctypes.c_int
            _LIBS[mutant] = lib
        return _LIBS[mutant]


def _dp(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def gdn_prefill_f64(q, k, v, w_q, w_k, w_v, alpha, beta, cu_seqlens, *, n_qk_heads, n_v_heads,
                    initial_state=None, conv_state=None, heads=None, q_scale=1.0, l2_eps=1e-6,
                    n_threads=None, mutant=0, conv_silu=False):
    """Run the oracle on fp64 arrays.

    Shapes: q,k [T,Hqk,dk]; v [T,Hv,dv]; w_* [channels, W]; alpha,beta [T,Hv];
    cu_seqlens [N+1]; initial_state [N,Hv,dk,dv]; conv_state [N,W-1,channels].
    ``heads`` restricts the work to those V heads (other heads' outputs stay NaN and
    their final states NaN).  Returns (y [T,Hv,dv], final_state [N,Hv,dk,dv],
    conv_state_out [N,W-1,channels]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    w_q, w_k, w_v = _f64(w_q), _f64(w_k), _f64(w_v)
    alpha, beta = _f64(alpha), _f64(beta)
    initial_state, conv_state = _f64(initial_state), _f64(conv_state)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T = q.shape[0]
    dk = q.shape[2]
    dv = v.shape[2]
    W = w_q.shape[1]
    n = len(cu) - 1
    assert int(cu[-1]) == T and q.shape == (T, n_qk_heads, dk) and v.shape == (T, n_v_heads, dv)
    sh = OracleShape(n_qk_heads, n_v_heads, dk, dv, W, float(q_scale), float(l2_eps), int(bool(conv_silu)))
    chans = 2 * n_qk_heads * dk + n_v_heads * dv
    out = np.full((T, n_v_heads, dv), np.nan)
    fin = np.full((n, n_v_heads, dk, dv), np.nan)
    cso = np.zeros((n, max(W - 1, 0), chans))
    hsel = None if heads is None else np.ascontiguousarray(heads, dtype=np.int32)
    rc = _lib(mutant).oracle_gdn_prefill(
        ctypes.byref(sh), _dp(q), _dp(k), _dp(v), _dp(w_q), _dp(w_k), _dp(w_v), _dp(alpha),
        _dp(beta), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n, _dp(initial_state),
        _dp(conv_state),
        None if hsel is None else hsel.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        0 if hsel is None else len(hsel), _dp(out), _dp(fin), _dp(cso),
        int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_gdn_prefill rejected its arguments")
    return out, fin, cso


def gdn_conv_l2_f64(q, k, v, w_q, w_k, w_v, cu_seqlens, *, n_qk_heads, n_v_heads,
                    conv_state=None, q_scale=1.0, l2_eps=1e-6, n_threads=None, mutant=0,
                    conv_silu=False):
    """ShortConv + L2 alone: returns (q^, k^, v^) in fp64 with the input shapes."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    w_q, w_k, w_v = _f64(w_q), _f64(w_k), _f64(w_v)
    conv_state = _f64(conv_state)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    dk, dv, W = q.shape[2], v.shape[2], w_q.shape[1]
    sh = OracleShape(n_qk_heads, n_v_heads, dk, dv, W, float(q_scale), float(l2_eps), int(bool(conv_silu)))
    qh, kh, vh = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    rc = _lib(mutant).oracle_gdn_conv_l2(
        ctypes.byref(sh), _dp(q), _dp(k), _dp(v), _dp(w_q), _dp(w_k), _dp(w_v),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu) - 1, _dp(conv_state),
        _dp(qh), _dp(kh), _dp(vh), int(n_threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_gdn_conv_l2 rejected its arguments")
    return qh, kh, vh


# ------------------------------------------------------------------ stored-input helpers
def _group_slices(shape, heads):
    """QK groups needed by ``heads`` and the V heads of those groups (in order)."""
    G = shape.n_v_heads // shape.n_qk_heads
    groups = sorted({int(h) // G for h in heads})
    vheads = [g * G + j for g in groups for j in range(G)]
    remap = [groups.index(int(h) // G) * G + int(h) % G for h in heads]
    return groups, vheads, remap


def _conv_state_columns(shape, groups, vheads):
    """Columns of a raw conv-state row (q | k | v channels) that the QK heads ``groups``
    and the V heads ``vheads`` read, in the order of the sliced problem."""
    dk, dv = shape.d_k, shape.d_v
    qkc = shape.n_qk_heads * dk
    qch = [g * dk + i for g in groups for i in range(dk)]
    vch = [h * dv + i for h in vheads for i in range(dv)]
    return qch + [qkc + c for c in qch] + [2 * qkc + c for c in vch]


def prefill(inp, heads=None, n_threads=None, q_scale=1.0, l2_eps=1e-6, initial_state=None,
            conv_state=None, mutant=0, conv_silu=False):
    """Oracle on a ``gdn_inputs.PrefillInputs`` bundle (stored values widened to fp64).

    With ``heads`` only the QK groups those V heads read are widened and computed; the
    returned arrays keep the full head axes, NaN outside the selected heads (the conv
    state is returned for all channels).
    """
    from gdn_inputs import stored_to_f64
    dt = inp.dtype
    sh = inp.shape
    init = inp.initial_state if initial_state is None else initial_state
    cs = inp.conv_state if conv_state is None else conv_state
    T, n = inp.total_tokens, inp.n_seqs
    dk, dv = sh.d_k, sh.d_v

    def f64(a):
        return a if a.dtype == np.float64 else stored_to_f64(a, dt)
    if heads is None:
        groups, vheads, hsel = list(range(sh.n_qk_heads)), list(range(sh.n_v_heads)), None
    else:
        groups, vheads, hsel = _group_slices(sh, heads)
    cs_sub = None
    if cs is not None:
        cs_sub = f64(np.asarray(cs)[:, :, _conv_state_columns(sh, groups, vheads)])
    y, fin, _ = gdn_prefill_f64(
        f64(inp.q[:, groups]), f64(inp.k[:, groups]), f64(inp.v[:, vheads]),
        inp.w_q.reshape(sh.n_qk_heads, dk, -1)[groups].reshape(len(groups) * dk, -1),
        inp.w_k.reshape(sh.n_qk_heads, dk, -1)[groups].reshape(len(groups) * dk, -1),
        inp.w_v.reshape(sh.n_v_heads, dv, -1)[vheads].reshape(len(vheads) * dv, -1),
        f64(inp.alpha[:, vheads]), f64(inp.beta[:, vheads]), inp.cu_seqlens,
        n_qk_heads=len(groups), n_v_heads=len(vheads),
        initial_state=None if init is None else np.asarray(init, dtype=np.float64)[:, vheads],
        conv_state=cs_sub, heads=hsel, q_scale=q_scale, l2_eps=l2_eps, n_threads=n_threads,
        mutant=mutant, conv_silu=conv_silu)
    y_full = np.full((T, sh.n_v_heads, dv), np.nan)
    fin_full = np.full((n, sh.n_v_heads, dk, dv), np.nan)
    y_full[:, vheads] = y
    fin_full[:, vheads] = fin
    # conv state out: the last W-1 raw rows of every channel (pure data movement)
    return y_full, fin_full, _conv_state_rows(inp, cs)


def _conv_state_rows(inp, cs):
    from gdn_inputs import stored_to_f64
    W1 = inp.shape.conv_width - 1
    n = inp.n_seqs
    ch = inp.shape.channels
    out = np.zeros((n, W1, ch))
    for b in range(n):
        t0, t1 = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        lo = max(t0, t1 - W1)
        sh = inp.shape
        qk = sh.n_qk_heads * sh.d_k
        rows = np.concatenate([inp.q[lo:t1].reshape(t1 - lo, qk), inp.k[lo:t1].reshape(t1 - lo, qk),
                               inp.v[lo:t1].reshape(t1 - lo, sh.n_v_heads * sh.d_v)], axis=1)
        rows = rows.astype(np.float64) if rows.dtype != np.uint16 else stored_to_f64(rows, inp.dtype)
        hist = np.zeros((W1, ch))
        if cs is not None:
            c = np.asarray(cs)[b]
            hist = c.astype(np.float64) if c.dtype != np.uint16 else stored_to_f64(c, inp.dtype)
        out[b] = np.vstack([hist, rows])[-W1:]
    return out


def decode_steps(shape, dtype, dec, w, state, conv_state, rows=None, heads=None, steps=None,
                 q_scale=1.0, l2_eps=1e-6, n_threads=None, conv_silu=False):
    """Run ``steps`` single-token steps for decode rows ``rows`` (default all).

    ``dec`` is a ``gdn_inputs.DecodeInputs``; ``state`` [B,Hv,dk,dv] fp64 (or fp32)
    and ``conv_state`` [B,W-1,channels] (stored dtype or fp64) are the starting
    states of all rows.  Each step is one oracle call over the selected rows, each
    row a one-token sequence.  Returns (y [steps, nrows, Hv, dv], state, conv_state)
    for the selected rows, in fp64.
    """
    from gdn_inputs import stored_to_f64
    B = dec.q.shape[1]
    rows = np.arange(B) if rows is None else np.asarray(rows)
    steps = dec.q.shape[0] if steps is None else steps
    st = np.asarray(state, dtype=np.float64)[rows].copy()
    cs = conv_state[rows]
    cs = cs.astype(np.float64) if cs.dtype != np.uint16 else stored_to_f64(cs, dtype)
    n = len(rows)
    cu = np.arange(n + 1, dtype=np.int32)
    ys = np.zeros((steps, n, shape.n_v_heads, shape.d_v))
    for s in range(steps):
        y, st_new, cs_new = gdn_prefill_f64(
            stored_to_f64(dec.q[s, rows], dtype), stored_to_f64(dec.k[s, rows], dtype),
            stored_to_f64(dec.v[s, rows], dtype), w[0], w[1], w[2],
            stored_to_f64(dec.alpha[s, rows], dtype), stored_to_f64(dec.beta[s, rows], dtype),
            cu, n_qk_heads=shape.n_qk_heads, n_v_heads=shape.n_v_heads, initial_state=st,
            conv_state=cs, heads=heads, q_scale=q_scale, l2_eps=l2_eps, n_threads=n_threads,
            conv_silu=conv_silu)
        ys[s] = y
        if heads is None:
            st = st_new
        else:
            st[:, heads] = st_new[:, heads]
        cs = cs_new
    return ys, st, cs
