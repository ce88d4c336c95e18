"""libgdn: the Gated DeltaNet token mixer on B200 (sm_100a), Python binding.

Thin wrappers over the C ABI of ``include/libgdn.h``: they check tensor
placement and shapes, allocate outputs and workspace with PyTorch when the caller
does not pass them, and hand raw device pointers plus the current CUDA stream to
the library.  Every step of the computation runs in libgdn's CUDA kernels; there
is no CPU or PyTorch fallback.

    y, S, cs = gdn_prefill(q, k, v, w_q, w_k, w_v, alpha, beta, cu_seqlens, ...)
    y = gdn_decode_step(q, k, v, w_q, w_k, w_v, alpha, beta, state, conv_state, ...)
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _native
from ._native import GDN_BF16, GDN_F32, GdnError  # noqa: F401

__all__ = ["GdnConfig", "affine_combine", "gdn_prefill", "gdn_decode_step", "gdn_decode_multi",
           "gdn_output_gate", "prefill_workspace_size", "GdnError", "LaunchTrace", "library_path",
           "qsa_block_keys", "qsa_block_scores", "qsa_select", "qsa_select_workspace_size",
           "QSA_BUDGET", "QSA_TOKEN_SLOTS"]


@dataclass(frozen=True)
class GdnConfig:
    n_qk_heads: int = 16
    n_v_heads: int = 48
    d_k: int = 128
    d_v: int = 128
    conv_width: int = 4
    q_scale: float = 1.0
    l2_eps: float = 1e-6
    conv_activation: int = 0     # 0: none (the page names none), 1: SiLU on the conv outputs

    def c(self) -> _native.GdnConfigC:
        return _native.GdnConfigC(self.n_qk_heads, self.n_v_heads, self.d_k, self.d_v,
                                  self.conv_width, self.q_scale, self.l2_eps, self.conv_activation)

    @property
    def channels(self) -> int:
        return 2 * self.n_qk_heads * self.d_k + self.n_v_heads * self.d_v


def library_path() -> str:
    return _native.LIB_PATH


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bfloat16 or float32")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libgdn takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libgdn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def prefill_workspace_size(cfg: GdnConfig, dtype: torch.dtype, total_tokens: int, n_seqs: int,
                           max_seqlen: int | None = None) -> int:
    """Preferred workspace bytes of gdn_prefill (``max_seqlen``: bound of the longest sequence)."""
    n = ctypes.c_size_t(0)
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    c = cfg.c()
    _native.check("gdn_prefill_workspace_size", _native.lib().gdn_prefill_workspace_size(
        ctypes.byref(c), code, int(total_tokens), int(n_seqs), int(max_seqlen or 0), ctypes.byref(n)))
    return int(n.value)


def gdn_prefill(q, k, v, conv_w_q, conv_w_k, conv_w_v, alpha, beta, cu_seqlens, *,
                cfg: GdnConfig | None = None, initial_state=None, final_state=None,
                return_final_state: bool = True, conv_state_in=None, conv_state_out=None,
                return_conv_state: bool = False, out=None, out_dtype=torch.float32,
                workspace=None, max_seqlen: int | None = None, gate=None, stream=None):
    """Chunked prefill over packed sequences.  Returns (out, final_state, conv_state_out).

    ``max_seqlen`` is a host-side upper bound of the longest sequence (None: the total); with
    many sequences it lets the chunk ranges stay short, so the workspace stays small.
    ``gate`` = (z, norm_w, norm_eps) fuses the output tail into the store of y:
    out = y / sqrt(mean(y^2) + norm_eps) * norm_w * SiLU(z) per (token, V head).

    q, k [T, Hqk, 128], v [T, Hv, 128], alpha/beta [T, Hv] (bf16 or fp32, one dtype);
    conv_w_* fp32 [channels, 4]; cu_seqlens int32 [N+1] on the device;
    initial_state fp32 [N, Hv, 128, 128] or None; conv_state_in [N, 3, channels] or None.
    ``out`` (or ``out_dtype``, fp32 by default) fixes y's storage type.
    """
    T = q.shape[0]
    cfg = cfg or GdnConfig(n_qk_heads=q.shape[1], n_v_heads=v.shape[1])
    n = cu_seqlens.shape[0] - 1
    code = _dtype_code(q)
    for t in (k, v, alpha, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, alpha and beta must share one dtype")
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    dev = q.device
    if out is None:
        out = torch.empty((T, cfg.n_v_heads, cfg.d_v), dtype=out_dtype, device=dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((n, cfg.n_v_heads, cfg.d_k, cfg.d_v), dtype=torch.float32,
                                  device=dev)
    if conv_state_out is None and return_conv_state:
        conv_state_out = torch.empty((n, cfg.conv_width - 1, cfg.channels), dtype=q.dtype,
                                     device=dev)
    need = prefill_workspace_size(cfg, q.dtype, T, n, max_seqlen)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    c = cfg.c()
    common = (ctypes.byref(c), code, _dtype_code(out), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w_q), _ptr(conv_w_k),
              _ptr(conv_w_v), _ptr(alpha), _ptr(beta), _ptr(cu_seqlens), n, T, int(max_seqlen or 0),
              _ptr(initial_state), _ptr(final_state), _ptr(conv_state_in), _ptr(conv_state_out))
    tail = (_ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if gate is None:
        _native.check("gdn_prefill", _native.lib().gdn_prefill(*common, *tail))
    else:
        z, norm_w, norm_eps = gate
        if z.shape != out.shape:
            raise ValueError("z must have the shape of the output")
        _native.check("gdn_prefill_gated", _native.lib().gdn_prefill_gated(
            *common, _ptr(z), _dtype_code(z), _ptr(norm_w), float(norm_eps), *tail))
    return out, final_state, conv_state_out


def gdn_decode_step(q, k, v, conv_w_q, conv_w_k, conv_w_v, alpha, beta, state, conv_state=None,
                    *, state_slots=None, cfg: GdnConfig | None = None, out=None,
                    out_dtype=torch.float32, stream=None):
    """One token for each row of the batch; ``state`` (and ``conv_state``) update in place.

    q, k [B, Hqk, 128], v [B, Hv, 128], alpha/beta [B, Hv]; state fp32 [R, Hv, 128, 128];
    conv_state [R, 3, channels] or None; state_slots int32 [B] (row b uses state row
    state_slots[b]) or None (identity).  Returns out [B, Hv, 128] (``out_dtype``).
    """
    B = q.shape[0]
    cfg = cfg or GdnConfig(n_qk_heads=q.shape[1], n_v_heads=v.shape[1])
    code = _dtype_code(q)
    for t in (k, v, alpha, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, alpha and beta must share one dtype")
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    if state_slots is not None and state_slots.dtype != torch.int32:
        raise TypeError("state_slots must be int32")
    if out is None:
        out = torch.empty((B, cfg.n_v_heads, cfg.d_v), dtype=out_dtype, device=q.device)
    c = cfg.c()
    st = _native.lib().gdn_decode_step(
        ctypes.byref(c), code, _dtype_code(out), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w_q), _ptr(conv_w_k),
        _ptr(conv_w_v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(conv_state), _ptr(state_slots),
        state.shape[0], _ptr(out), B, _stream(stream))
    _native.check("gdn_decode_step", st)
    return out


def gdn_decode_multi(q, k, v, conv_w_q, conv_w_k, conv_w_v, alpha, beta, state, conv_state=None,
                     *, state_slots=None, state_ckpt=None, conv_ckpt=None, cfg: GdnConfig | None = None,
                     out=None, out_dtype=torch.float32, stream=None):
    """n consecutive tokens for each row of the batch; ``state`` (and ``conv_state``) advance by
    all of them in place.

    q, k [B, n, Hqk, 128], v [B, n, Hv, 128], alpha/beta [B, n, Hv]; state fp32 [R, Hv, 128, 128];
    conv_state [R, 3, channels] or None; state_slots int32 [B] or None.  ``state_ckpt``
    (fp32 [B, n, Hv, 128, 128]) and ``conv_ckpt`` ([B, n, 3, channels], q's dtype), when given,
    receive the state and the conv state after every token.  Returns out [B, n, Hv, 128].
    """
    B, n = q.shape[0], q.shape[1]
    cfg = cfg or GdnConfig(n_qk_heads=q.shape[2], n_v_heads=v.shape[2])
    code = _dtype_code(q)
    for t in (k, v, alpha, beta):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, alpha and beta must share one dtype")
    if state.dtype != torch.float32 or (state_ckpt is not None and state_ckpt.dtype != torch.float32):
        raise TypeError("state and state_ckpt must be float32")
    if conv_ckpt is not None and conv_ckpt.dtype != q.dtype:
        raise TypeError("conv_ckpt must have q's dtype")
    if state_slots is not None and state_slots.dtype != torch.int32:
        raise TypeError("state_slots must be int32")
    if out is None:
        out = torch.empty((B, n, cfg.n_v_heads, cfg.d_v), dtype=out_dtype, device=q.device)
    c = cfg.c()
    st = _native.lib().gdn_decode_multi(
        ctypes.byref(c), code, _dtype_code(out), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_w_q), _ptr(conv_w_k),
        _ptr(conv_w_v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(conv_state), _ptr(state_slots),
        state.shape[0], _ptr(state_ckpt), _ptr(conv_ckpt), _ptr(out), B, n, _stream(stream))
    _native.check("gdn_decode_multi", st)
    return out


def gdn_output_gate(y, z, norm_w, *, eps: float = 1e-6, cfg: GdnConfig | None = None, out=None,
                    out_dtype=None, stream=None):
    """Gated RMS normalisation of y per (token, V head): y / sqrt(mean(y^2) + eps) * norm_w * SiLU(z).

    y, z [..., Hv, 128] (bf16 or fp32, any mix); norm_w fp32 [128]; ``out`` may be ``y``.
    Returns out (``out_dtype``, default y's dtype).
    """
    if y.shape != z.shape:
        raise ValueError("y and z must have the same shape")
    if norm_w.dtype != torch.float32 or norm_w.numel() != y.shape[-1]:
        raise TypeError("norm_w must be float32 with one weight per channel")
    Hv = y.shape[-2]
    cfg = cfg or GdnConfig(n_qk_heads=1, n_v_heads=Hv)
    if out is None:
        out = torch.empty(y.shape, dtype=out_dtype or y.dtype, device=y.device)
    n_tokens = y.numel() // (Hv * y.shape[-1])
    c = cfg.c()
    st = _native.lib().gdn_output_gate(ctypes.byref(c), _dtype_code(y), _dtype_code(z), _dtype_code(out),
                                       _ptr(y), _ptr(z), _ptr(norm_w), float(eps), _ptr(out), n_tokens,
                                       _stream(stream))
    _native.check("gdn_output_gate", st)
    return out


def affine_combine(M, B, S0=None, *, cfg: GdnConfig | None = None, out=None, stream=None):
    """States entering consecutive spans of one sequence from the spans' affine maps
    (S_out = M S_in + B per V head): out[0] = S0 (zero if None), out[p+1] = M[p] out[p] + B[p].
    M, B fp32 [P, Hv, 128, 128]; returns fp32 [P + 1, Hv, 128, 128]."""
    if M.dtype != torch.float32 or B.dtype != torch.float32 or M.shape != B.shape or M.dim() != 4:
        raise ValueError("M and B must be fp32 [P, Hv, 128, 128] of one shape")
    P, Hv = M.shape[0], M.shape[1]
    cfg = cfg or GdnConfig(n_qk_heads=1, n_v_heads=Hv)
    if out is None:
        out = torch.empty((P + 1,) + tuple(M.shape[1:]), dtype=torch.float32, device=M.device)
    if S0 is not None and (S0.dtype != torch.float32 or tuple(S0.shape) != tuple(M.shape[1:])):
        raise ValueError("S0 must be fp32 [Hv, 128, 128]")
    c = cfg.c()
    _native.check("gdn_affine_combine", _native.lib().gdn_affine_combine(
        ctypes.byref(c), _ptr(M), _ptr(B), P, _ptr(S0), _ptr(out), _stream(stream)))
    return out


class LaunchTrace:
    """Context manager around gdn_trace_begin/gdn_trace_end (this host thread only).

    with LaunchTrace(capacity) as tr: ...libgdn calls...
    torch.cuda.synchronize(); tr.records() -> [(kernel_name, milliseconds), ...]
    """

    def __init__(self, capacity: int = 1024):
        self.capacity = int(capacity)
        self.events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(self.capacity)]
        s = torch.cuda.current_stream()
        for a, b in self.events:  # materialise the event handles
            a.record(s)
            b.record(s)
        self._arr = (_native.TraceEntryC * max(self.capacity, 1))()
        for i, (a, b) in enumerate(self.events):
            self._arr[i].start = a.cuda_event
            self._arr[i].stop = b.cuda_event
        self.count = 0

    def __enter__(self):
        _native.lib().gdn_trace_begin(self._arr, self.capacity)
        return self

    def __exit__(self, *exc):
        self.count = _native.lib().gdn_trace_end()
        return False

    def records(self):
        n = min(self.count, self.capacity)
        return [(self._arr[i].kernel.decode(), self.events[i][0].elapsed_time(self.events[i][1]))
                for i in range(n)]


# ----------------------------------------------------------------------------- QSA indexer
QSA_BUDGET = 512                  # blocks per query
QSA_TOKEN_SLOTS = 4 * 512 + 3     # token-set entries per query


def _qsa_check(name, t, dtype, shape_len):
    if t.dtype != dtype or t.dim() != shape_len or not t.is_contiguous() or not t.is_cuda:
        raise TypeError(f"{name}: expected a contiguous CUDA {dtype} tensor of rank {shape_len}")


def qsa_block_keys(k, w_k, kpos, kbar, *, eps: float = 1e-6, theta: float = 10000.0, stream=None):
    """Write the QSA block keys of k [B, Tn, 128] (bf16, tokens kpos[b] .. kpos[b]+Tn-1 of
    row b, Tn % 4 == 0) into the cache kbar [B, nb_max, 128] (bf16) at blocks kpos[b]/4 ...
    w_k fp32 [128]; kpos int32 [B] on the device.  Returns kbar."""
    _qsa_check("k", k, torch.bfloat16, 3)
    _qsa_check("kbar", kbar, torch.bfloat16, 3)
    _qsa_check("kpos", kpos, torch.int32, 1)
    _qsa_check("w_k", w_k, torch.float32, 1)
    B, Tn, _ = k.shape
    st = _native.lib().gdn_qsa_block_keys(_ptr(k), _ptr(w_k), _ptr(kpos), B, Tn, float(eps), float(theta),
                                          _ptr(kbar), kbar.shape[1], _stream(stream))
    _native.check("gdn_qsa_block_keys", st)
    return kbar


def _qsa_query_args(q, w_q, qpos, kbar, n_blocks):
    _qsa_check("q", q, torch.bfloat16, 4)
    _qsa_check("kbar", kbar, torch.bfloat16, 3)
    _qsa_check("qpos", qpos, torch.int32, 1)
    _qsa_check("n_blocks", n_blocks, torch.int32, 1)
    _qsa_check("w_q", w_q, torch.float32, 1)
    if q.shape[2] != 4 or q.shape[3] != 128 or kbar.shape[2] != 128 or kbar.shape[0] != q.shape[0]:
        raise ValueError("q must be [B, Qn, 4, 128] and kbar [B, nb_max, 128]")
    return q.shape[0], q.shape[1], kbar.shape[1]


def qsa_block_scores(q, w_q, qpos, kbar, n_blocks, *, eps: float = 1e-6, theta: float = 10000.0,
                     out=None, stream=None):
    """Block scores [B, Qn, nb_max] fp32 of the queries q [B, Qn, 4, 128] (bf16, tokens
    qpos[b] .. of row b) against the block-key cache; entries of blocks that are not
    candidates of a query are unspecified."""
    B, Qn, nb = _qsa_query_args(q, w_q, qpos, kbar, n_blocks)
    if out is None:
        out = torch.empty((B, Qn, nb), dtype=torch.float32, device=q.device)
    st = _native.lib().gdn_qsa_block_scores(_ptr(q), _ptr(w_q), _ptr(qpos), _ptr(kbar), _ptr(n_blocks), B, Qn, nb,
                                            float(eps), float(theta), _ptr(out), _stream(stream))
    _native.check("gdn_qsa_block_scores", st)
    return out


def qsa_select_workspace_size(B: int, Qn: int, nb_max: int) -> int:
    n = ctypes.c_size_t(0)
    st = _native.lib().gdn_qsa_select_workspace_size(B, Qn, nb_max, ctypes.byref(n))
    _native.check("gdn_qsa_select_workspace_size", st)
    return int(n.value)


def qsa_select(q, w_q, qpos, kbar, n_blocks, *, eps: float = 1e-6, theta: float = 10000.0,
               blocks=None, tokens=None, with_tokens: bool = False, workspace=None, stream=None):
    """Top-512 block set (and with ``with_tokens`` or a given ``tokens`` buffer, the token
    set) of every query.  Returns (blocks int32 [B, Qn, 512], tokens int32 [B, Qn, 2051]
    or None), ascending and padded with -1."""
    B, Qn, nb = _qsa_query_args(q, w_q, qpos, kbar, n_blocks)
    if blocks is None:
        blocks = torch.empty((B, Qn, QSA_BUDGET), dtype=torch.int32, device=q.device)
    if tokens is None and with_tokens:
        tokens = torch.empty((B, Qn, QSA_TOKEN_SLOTS), dtype=torch.int32, device=q.device)
    need = qsa_select_workspace_size(B, Qn, nb)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = _native.lib().gdn_qsa_select(_ptr(q), _ptr(w_q), _ptr(qpos), _ptr(kbar), _ptr(n_blocks), B, Qn, nb,
                                      float(eps), float(theta), _ptr(blocks),
                                      None if tokens is None else _ptr(tokens), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream))
    _native.check("gdn_qsa_select", st)
    return blocks, tokens
