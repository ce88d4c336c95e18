"""ctypes view of libgdn.so (the C ABI declared in include/libgdn.h).

Loading fails loudly when the library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_BF16 = 0
GDN_F32 = 1

STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_WORKSPACE",
          4: "GDN_ERR_CUDA", 5: "GDN_ERR_TIMEOUT"}

# every entry point the header declares (checked by the CPU test suite)
EXPORTS = ("gdn_status_string", "gdn_last_cuda_error", "gdn_api_version",
           "gdn_prefill_workspace_size", "gdn_prefill", "gdn_prefill_gated", "gdn_decode_step", "gdn_decode_multi",
           "gdn_output_gate", "gdn_affine_combine", "gdn_trace_begin",
           "gdn_trace_end", "gdn_prefill_static_scratch", "gdn_qsa_block_keys",
           "gdn_qsa_block_scores", "gdn_qsa_select_workspace_size", "gdn_qsa_select")

STATIC_SCRATCH_BYTES = 64 << 20  # GDN_STATIC_SCRATCH_BYTES


class TraceEntryC(ctypes.Structure):
    _fields_ = [("start", ctypes.c_void_p), ("stop", ctypes.c_void_p), ("kernel", ctypes.c_char_p)]


class GdnConfigC(ctypes.Structure):
    _fields_ = [("n_qk_heads", ctypes.c_int), ("n_v_heads", ctypes.c_int), ("d_k", ctypes.c_int),
                ("d_v", ctypes.c_int), ("conv_width", ctypes.c_int), ("q_scale", ctypes.c_float),
                ("l2_eps", ctypes.c_float), ("conv_activation", ctypes.c_int)]


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        msg = f"{fn} failed: {STATUS.get(status, status)}"
        if status == 4:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)
        self.status = status
        self.cuda_error = cuda_error


_lock = threading.Lock()
_lib = None


def lib():
    """The loaded libgdn.so (raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m linear_attention_recurrence_05_b200.build` (there is no fallback)")
            L = ctypes.CDLL(LIB_PATH)
            vp, i32p, fp = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
            L.gdn_status_string.argtypes = [ctypes.c_int]
            L.gdn_status_string.restype = ctypes.c_char_p
            L.gdn_last_cuda_error.argtypes = []
            L.gdn_last_cuda_error.restype = ctypes.c_int
            L.gdn_api_version.argtypes = []
            L.gdn_api_version.restype = ctypes.c_int
            L.gdn_prefill_workspace_size.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int,
                                                     ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                                     ctypes.POINTER(ctypes.c_size_t)]
            L.gdn_prefill_workspace_size.restype = ctypes.c_int
            L.gdn_prefill.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int, ctypes.c_int, vp, vp,
                                      vp, fp, fp,
                                      fp, vp, vp, i32p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                      fp, fp, vp, vp, vp, vp, ctypes.c_size_t, vp]
            L.gdn_prefill.restype = ctypes.c_int
            L.gdn_prefill_gated.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                            fp, fp, fp, vp, vp, i32p, ctypes.c_int, ctypes.c_int64,
                                            ctypes.c_int64, fp, fp, vp, vp, vp, ctypes.c_int, fp,
                                            ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
            L.gdn_prefill_gated.restype = ctypes.c_int
            L.gdn_decode_step.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int, ctypes.c_int, vp,
                                          vp, vp, fp,
                                          fp, fp, vp, vp, fp, vp, i32p, ctypes.c_int, vp,
                                          ctypes.c_int, vp]
            L.gdn_decode_step.restype = ctypes.c_int
            L.gdn_decode_multi.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int, ctypes.c_int, vp,
                                           vp, vp, fp, fp, fp, vp, vp, fp, vp, i32p, ctypes.c_int,
                                           fp, vp, vp, ctypes.c_int, ctypes.c_int, vp]
            L.gdn_decode_multi.restype = ctypes.c_int
            L.gdn_output_gate.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          vp, vp, fp, ctypes.c_float, vp, ctypes.c_int64, vp]
            L.gdn_output_gate.restype = ctypes.c_int
            L.gdn_affine_combine.argtypes = [ctypes.POINTER(GdnConfigC), fp, fp, ctypes.c_int, fp, fp, vp]
            L.gdn_affine_combine.restype = ctypes.c_int
            L.gdn_trace_begin.argtypes = [ctypes.POINTER(TraceEntryC), ctypes.c_int]
            L.gdn_trace_begin.restype = None
            L.gdn_trace_end.argtypes = []
            L.gdn_trace_end.restype = ctypes.c_int
            L.gdn_prefill_static_scratch.argtypes = [ctypes.POINTER(GdnConfigC), ctypes.c_int,
                                                     ctypes.c_int, vp, vp, vp, fp, fp, fp, vp, vp,
                                                     i32p, ctypes.c_int, ctypes.c_int64, fp, fp,
                                                     vp, vp, vp, vp]
            L.gdn_prefill_static_scratch.restype = ctypes.c_int
            ci, cf = ctypes.c_int, ctypes.c_float
            L.gdn_qsa_block_keys.argtypes = [vp, fp, i32p, ci, ci, cf, cf, vp, ci, vp]
            L.gdn_qsa_block_keys.restype = ctypes.c_int
            L.gdn_qsa_block_scores.argtypes = [vp, fp, i32p, vp, i32p, ci, ci, ci, cf, cf, fp, vp]
            L.gdn_qsa_block_scores.restype = ctypes.c_int
            L.gdn_qsa_select_workspace_size.argtypes = [ci, ci, ci, ctypes.POINTER(ctypes.c_size_t)]
            L.gdn_qsa_select_workspace_size.restype = ctypes.c_int
            L.gdn_qsa_select.argtypes = [vp, fp, i32p, vp, i32p, ci, ci, ci, cf, cf, i32p, i32p, vp,
                                         ctypes.c_size_t, vp]
            L.gdn_qsa_select.restype = ctypes.c_int
            _lib = L
        return _lib


def check(fn: str, status: int) -> None:
    if status != 0:
        raise GdnError(fn, status, lib().gdn_last_cuda_error())
