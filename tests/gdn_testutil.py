"""Shared helpers of the parity tests: host<->device marshalling and error metrics."""
from __future__ import annotations

import numpy as np

import gdn_inputs as gi

BF16_TOL = 2e-2   # max|gpu - oracle| / rms(oracle), bf16 storage, fp32 state
F32_TOL = 1e-4    # same bound for the fp32-storage path


def tol(dtype: str) -> float:
    return BF16_TOL if dtype == gi.BF16 else F32_TOL


def to_dev(a: np.ndarray, dtype: str):
    """Stored numpy array (uint16 bf16 bits or fp32/int) -> CUDA tensor of the same bytes."""
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def rel_err(x: np.ndarray, ref: np.ndarray) -> float:
    """max |x - ref| / rms(ref) over finite reference entries."""
    m = np.isfinite(ref)
    if not m.any():
        return 0.0
    rms = float(np.sqrt(np.mean(ref[m] ** 2)))
    return float(np.max(np.abs(x[m] - ref[m])) / max(rms, 1e-30))


def prefill_dev(inp: gi.PrefillInputs, lib, *, with_conv_out=False, initial_state=None,
                conv_state=None, conv_activation=0):
    """Run the CUDA prefill on a stored-input bundle; returns (y, final_state, conv_out) tensors."""
    import torch
    d = inp.dtype
    cfg = lib.GdnConfig(inp.shape.n_qk_heads, inp.shape.n_v_heads, conv_activation=conv_activation)
    init = inp.initial_state if initial_state is None else initial_state
    cs = inp.conv_state if conv_state is None else conv_state
    return lib.gdn_prefill(
        to_dev(inp.q, d), to_dev(inp.k, d), to_dev(inp.v, d), to_dev(inp.w_q, d),
        to_dev(inp.w_k, d), to_dev(inp.w_v, d), to_dev(inp.alpha, d), to_dev(inp.beta, d),
        torch.from_numpy(inp.cu_seqlens).cuda(), cfg=cfg,
        initial_state=None if init is None else torch.from_numpy(np.asarray(init, np.float32)).cuda(),
        conv_state_in=None if cs is None else to_dev(cs, d), return_conv_state=with_conv_out)


def rel_err_bf16_out(x: np.ndarray, ref: np.ndarray) -> float:
    """Like rel_err for outputs stored as bf16: each entry may additionally carry the
    half-ulp of its own bf16 rounding (2^-9 of its magnitude)."""
    m = np.isfinite(ref)
    rms = float(np.sqrt(np.mean(ref[m] ** 2)))
    excess = np.abs(x[m] - ref[m]) - 2.0 ** -9 * np.abs(ref[m]) * 1.001
    return float(max(np.max(excess), 0.0) / max(rms, 1e-30))


def prefill_args(inp: gi.PrefillInputs, lib):
    """Device tensors of a stored-input bundle in gdn_prefill's positional order."""
    import torch
    d = inp.dtype
    return (to_dev(inp.q, d), to_dev(inp.k, d), to_dev(inp.v, d), to_dev(inp.w_q, d),
            to_dev(inp.w_k, d), to_dev(inp.w_v, d), to_dev(inp.alpha, d), to_dev(inp.beta, d),
            torch.from_numpy(inp.cu_seqlens).cuda())
