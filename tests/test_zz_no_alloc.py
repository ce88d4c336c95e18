"""gdn_prefill_static_scratch: the prefill entry point for callers that cannot allocate.

Such callers (a plugin whose framework forbids device allocation while it executes,
a runtime that owns all device memory, C code without an allocator) get the same
results as gdn_prefill while the library keeps the scratch in its own fixed device
array.  This file is collected last so that a run stopping at the first failure has
run every other test already; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import gdn_inputs as gi
from gdn_testutil import to_dev, to_host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _case(shape, lengths, dtype, seed):
    inp = gi.make_prefill_inputs(shape, lengths, dtype, seed, with_initial_state=True,
                                 with_conv_state=True)
    d = {name: to_dev(getattr(inp, name), dtype)
         for name in ("q", "k", "v", "w_q", "w_k", "w_v", "alpha", "beta")}
    d["cu"] = torch.from_numpy(inp.cu_seqlens).cuda()
    d["init"] = torch.from_numpy(inp.initial_state).cuda()
    d["cs"] = to_dev(inp.conv_state, dtype)
    return inp, d


def _static_call(lib, native, inp, d):
    """The new entry point, called through the C ABI with caller-owned outputs only."""
    T, n = inp.total_tokens, inp.n_seqs
    sh = inp.shape
    out = torch.full((T, sh.n_v_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    fin = torch.full((n, sh.n_v_heads, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    cso = torch.empty_like(d["cs"])
    cfg = native.GdnConfigC(sh.n_qk_heads, sh.n_v_heads, 128, 128, 4, 1.0, 1e-6)
    code = native.GDN_BF16 if inp.dtype == gi.BF16 else native.GDN_F32
    st = native.lib().gdn_prefill_static_scratch(
        ctypes.byref(cfg), code, native.GDN_F32, _ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]),
        _ptr(d["w_q"]), _ptr(d["w_k"]), _ptr(d["w_v"]), _ptr(d["alpha"]), _ptr(d["beta"]),
        _ptr(d["cu"]), n, T, _ptr(d["init"]), _ptr(fin), _ptr(d["cs"]), _ptr(cso), _ptr(out),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, native.STATUS.get(st, st)
    return out, fin, cso


def _check_against_prefill(gdn, native, inp, d):
    cfg = gdn.GdnConfig(inp.shape.n_qk_heads, inp.shape.n_v_heads)
    y_ref, f_ref, c_ref = gdn.gdn_prefill(
        d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["w_v"], d["alpha"], d["beta"], d["cu"],
        cfg=cfg, initial_state=d["init"], conv_state_in=d["cs"], return_conv_state=True)
    y, f, c = _static_call(gdn, native, inp, d)
    torch.cuda.synchronize()
    # the same kernels on the same inputs: the chunk arithmetic is identical and the state
    # crosses chunk ranges exactly (fp32 in memory), so the results are bit for bit those of
    # gdn_prefill, whatever range length each call chose
    assert np.array_equal(to_host_f64(y), to_host_f64(y_ref))
    assert np.array_equal(to_host_f64(f), to_host_f64(f_ref))
    assert np.array_equal(to_host_f64(c), to_host_f64(c_ref))
    assert np.isfinite(to_host_f64(y)).all()


def test_static_scratch_matches_prefill_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_attention_recurrence_05_b200 as gdn
    from linear_attention_recurrence_05_b200 import _native as native

    # two different problems in a row: the second runs on the scratch the first left behind
    cases = [_case(gi.GdnShape(4, 12), [300, 0, 65, 200], gi.BF16, 501),
             _case(gi.GdnShape(2, 6), [129, 7], gi.F32, 502)]
    for inp, d in cases:
        _check_against_prefill(gdn, native, inp, d)


def test_static_scratch_several_chunk_ranges():
    """Problems that take more than one chunk range through this entry point: at 2 / 6 heads
    a 4,200-token sequence runs the same three ranges as gdn_prefill (tiles of range r+1
    made on the auxiliary stream while the chains run range r); at 16 / 48 heads a
    4,096-token sequence does not fit the scratch with gdn_prefill's ranges and runs in
    shorter ones."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_attention_recurrence_05_b200 as gdn
    from linear_attention_recurrence_05_b200 import _native as native
    for shape, lengths, seed in ((gi.GdnShape(2, 6), [4200], 503), (gi.GdnShape(16, 48), [4096], 504)):
        inp, d = _case(shape, lengths, gi.BF16, seed)
        _check_against_prefill(gdn, native, inp, d)


def test_static_scratch_rejects_oversized_problem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrence_05_b200 import _native as native
    cfg = native.GdnConfigC(16, 48, 128, 128, 4, 1.0, 1e-6)
    need = ctypes.c_size_t(0)
    T = 4096
    # 16 sequences: even one chunk slot per sequence exceeds the scratch
    n = 16
    assert native.lib().gdn_prefill_workspace_size(ctypes.byref(cfg), 0, T, n, 0,
                                                   ctypes.byref(need)) == 0
    assert need.value > native.STATIC_SCRATCH_BYTES
    # rejected on the host, before any pointer is looked at or anything is enqueued
    A = 1 << 20
    st = native.lib().gdn_prefill_static_scratch(
        ctypes.byref(cfg), 0, 1, A, A, A, A, A, A, A, A, A, n, T, None, None, None, None, A, None)
    assert st == 3  # GDN_ERR_WORKSPACE
