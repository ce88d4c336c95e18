"""The C-ABI library loads, exports every entry point the header declares, and rejects
bad arguments on the host before touching the device (CPU only: no compute call)."""
import ctypes
import os
import re

import pytest

import linear_attention_recurrence_05_b200 as gdn
from linear_attention_recurrence_05_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "libgdn.h")


def header_exports():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_EXPORT\s+[\w\s\*]*?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert header_exports() == sorted(_native.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = _native.lib()
    for name in header_exports():
        assert hasattr(lib, name), name
    assert lib.gdn_api_version() == 2


def test_binding_all_names_exist():
    missing = [n for n in gdn.__all__ if not hasattr(gdn, n)]
    assert not missing, missing


def test_status_strings():
    lib = _native.lib()
    for code, name in _native.STATUS.items():
        assert lib.gdn_status_string(code).decode() == name
    assert lib.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"


def _cfg(**kw):
    base = dict(n_qk_heads=16, n_v_heads=48, d_k=128, d_v=128, conv_width=4, q_scale=1.0,
                l2_eps=1e-6, conv_activation=0)
    base.update(kw)
    return _native.GdnConfigC(*base.values())


def _ws(cfg, dtype=0, T=8192, n=1, max_seqlen=0):
    out = ctypes.c_size_t(0)
    st = _native.lib().gdn_prefill_workspace_size(ctypes.byref(cfg), dtype, T, n, max_seqlen,
                                                  ctypes.byref(out))
    return st, out.value


# tiles of one (sequence, chunk) slot at 16 QK / 48 V heads: [K;Q] 64 KB and K (fp16) 16 KB per
# QK head; V (fp16) 16 KB, T_beta (fp16) 8 KB, T_beta_gamma 16 KB, P (fp16) 8 KB and a 640-byte
# gates record per V head
SLOT = 16 * (65536 + 16384) + 48 * (16384 + 8192 + 16384 + 8192 + 640)
STATE = 128 * 128 * 4


def test_workspace_size_bf16_is_two_chunk_ranges():
    # one 8192-token sequence: ranges of 32 chunks, two buffers, one carried state per head
    st, b = _ws(_cfg(), 0, 8192, 1)
    assert st == 0
    assert 2 * 32 * SLOT + 48 * STATE <= b < 2 * 32 * SLOT + 48 * STATE + 64 * 1024
    # the size depends on the range length, not on the number of tokens
    st2, b2 = _ws(_cfg(), 0, 262144, 1, 262144)
    st3, b3 = _ws(_cfg(), 0, 2 * 262144, 1, 2 * 262144)
    assert st2 == st3 == 0 and b2 == b3 < 2 * 128 * SLOT + 48 * STATE + 64 * 1024
    # 32 packed sequences up to 64K tokens: 16 chunks per sequence per range
    st4, b4 = _ws(_cfg(), 0, 602887, 32, 65536)
    assert st4 == 0 and b4 < 2 * 32 * 16 * SLOT + 32 * 48 * STATE + 64 * 1024
    assert _ws(_cfg(), 0, 0, 3)[0] == 0


def test_workspace_size_fp32_rows():
    # q^, k^ (2 x T x 16 x 128) + v^ (T x 48 x 128) in fp32, plus two small int tables
    rows = 8192 * (2 * 16 + 48) * 128 * 4
    st, b = _ws(_cfg(), 1, 8192, 1)
    assert st == 0 and rows <= b < rows + 4096


@pytest.mark.parametrize("kw,code", [
    (dict(d_k=64), 2), (dict(d_v=256), 2), (dict(conv_width=3), 2),
    (dict(n_v_heads=47), 1), (dict(n_qk_heads=0), 1), (dict(l2_eps=-1.0), 1),
    (dict(q_scale=float("nan")), 1), (dict(conv_activation=2), 1), (dict(conv_activation=-1), 1),
])
def test_config_rejected(kw, code):
    assert _ws(_cfg(**kw))[0] == code


def test_workspace_size_bad_args():
    lib = _native.lib()
    c = _cfg()
    assert lib.gdn_prefill_workspace_size(ctypes.byref(c), 0, 10, 1, 0, None) == 1
    assert _ws(c, 0, -1, 1)[0] == 1
    assert _ws(c, 0, 1 << 31, 1)[0] == 1
    assert _ws(c, 7, 10, 1)[0] == 1
    assert _ws(c, 0, 10, 1, -1)[0] == 1
    assert lib.gdn_prefill_workspace_size(None, 0, 10, 1, 0, ctypes.byref(ctypes.c_size_t())) == 1


def _prefill(**over):
    """gdn_prefill with fake (never dereferenced) aligned device addresses."""
    A = 1 << 20
    args = dict(cfg=_cfg(), dtype=0, odt=1, q=A, k=2 * A, v=3 * A, wq=4 * A, wk=5 * A, wv=6 * A,
                alpha=7 * A, beta=8 * A, cu=9 * A, n=1, T=100, ms=0, init=None, fin=None, csi=None,
                cso=None, out=10 * A, ws=11 * A, wsb=1 << 40, stream=None)
    args.update(over)
    c = args["cfg"]
    return _native.lib().gdn_prefill(
        ctypes.byref(c) if c is not None else None, args["dtype"], args["odt"], args["q"], args["k"], args["v"],
        args["wq"], args["wk"], args["wv"], args["alpha"], args["beta"], args["cu"], args["n"],
        args["T"], args["ms"], args["init"], args["fin"], args["csi"], args["cso"], args["out"], args["ws"],
        args["wsb"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(v=None), 1), (dict(out=None), 1), (dict(cu=None), 1),
    (dict(wq=None), 1), (dict(q=(1 << 20) + 8), 1), (dict(out=(1 << 20) + 4), 1),
    (dict(alpha=(1 << 20) + 1), 1), (dict(init=(1 << 20) + 8), 1), (dict(cso=(1 << 20) + 2), 1),
    (dict(T=-5), 1), (dict(n=-1), 1), (dict(T=1 << 31), 1), (dict(dtype=3), 1),
    (dict(ws=None), 3), (dict(wsb=16), 3), (dict(ws=(11 << 20) + 64), 3),
    (dict(cfg=None), 1), (dict(cfg=_cfg(d_k=96)), 2), (dict(odt=2), 1), (dict(ms=-1), 1),
])
def test_prefill_rejects_before_launch(over, code):
    assert _prefill(**over) == code


def test_prefill_zero_sequences_is_noop():
    assert _prefill(n=0, q=None, k=None, v=None, out=None, ws=None) == 0


def _decode(**over):
    A = 1 << 20
    args = dict(cfg=_cfg(), dtype=0, odt=1, q=A, k=2 * A, v=3 * A, wq=4 * A, wk=5 * A, wv=6 * A,
                alpha=7 * A, beta=8 * A, state=9 * A, conv=10 * A, slots=None, rows=4, out=11 * A,
                batch=4, stream=None)
    args.update(over)
    c = args["cfg"]
    return _native.lib().gdn_decode_step(
        ctypes.byref(c), args["dtype"], args["odt"], args["q"], args["k"], args["v"], args["wq"],
        args["wk"], args["wv"], args["alpha"], args["beta"], args["state"], args["conv"], args["slots"],
        args["rows"], args["out"], args["batch"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(state=None), 1), (dict(q=None), 1), (dict(out=None), 1), (dict(state=(9 << 20) + 4), 1),
    (dict(conv=(10 << 20) + 2), 1), (dict(rows=2), 1), (dict(batch=-1), 1),
    (dict(slots=(12 << 20) + 2), 1), (dict(cfg=_cfg(conv_width=2)), 2), (dict(odt=-1), 1),
])
def test_decode_rejects_before_launch(over, code):
    assert _decode(**over) == code


def test_decode_empty_batch_is_noop():
    assert _decode(batch=0, q=None) == 0


def _decode_multi(**over):
    A = 1 << 20
    args = dict(cfg=_cfg(), dtype=0, odt=1, q=A, k=2 * A, v=3 * A, wq=4 * A, wk=5 * A, wv=6 * A,
                alpha=7 * A, beta=8 * A, state=9 * A, conv=10 * A, slots=None, rows=4, ck=None, cck=None,
                out=11 * A, batch=4, n=4, stream=None)
    args.update(over)
    c = args["cfg"]
    return _native.lib().gdn_decode_multi(
        ctypes.byref(c), args["dtype"], args["odt"], args["q"], args["k"], args["v"], args["wq"],
        args["wk"], args["wv"], args["alpha"], args["beta"], args["state"], args["conv"], args["slots"],
        args["rows"], args["ck"], args["cck"], args["out"], args["batch"], args["n"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(n=0), 1), (dict(n=-3), 1), (dict(n=9), 2), (dict(state=None), 1), (dict(out=None), 1),
    (dict(ck=(12 << 20) + 8), 1), (dict(cck=(13 << 20) + 2), 1), (dict(rows=2), 1),
    (dict(cfg=_cfg(d_k=64)), 2),
])
def test_decode_multi_rejects_before_launch(over, code):
    assert _decode_multi(**over) == code


def test_decode_multi_empty_batch_is_noop():
    assert _decode_multi(batch=0, q=None) == 0


def _gate(**over):
    A = 1 << 20
    args = dict(cfg=_cfg(), ydt=1, zdt=0, odt=1, y=A, z=2 * A, w=3 * A, eps=1e-6, out=4 * A, n=10, stream=None)
    args.update(over)
    c = args["cfg"]
    return _native.lib().gdn_output_gate(ctypes.byref(c), args["ydt"], args["zdt"], args["odt"], args["y"],
                                         args["z"], args["w"], args["eps"], args["out"], args["n"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(y=None), 1), (dict(z=None), 1), (dict(w=None), 1), (dict(out=None), 1), (dict(n=-1), 1),
    (dict(eps=-1.0), 1), (dict(eps=float("inf")), 1), (dict(eps=float("nan")), 1), (dict(zdt=7), 1),
    (dict(z=(2 << 20) + 8), 1), (dict(cfg=_cfg(d_v=64)), 2),
])
def test_output_gate_rejects_before_launch(over, code):
    assert _gate(**over) == code


def test_output_gate_no_tokens_is_noop():
    assert _gate(n=0, y=None, out=None) == 0


def _qkeys(**over):
    A = 1 << 20
    a = dict(k=A, w=2 * A, kpos=3 * A, B=2, Tn=8, eps=1e-6, theta=1e4, kbar=4 * A, nb=16, stream=None)
    a.update(over)
    return _native.lib().gdn_qsa_block_keys(a["k"], a["w"], a["kpos"], a["B"], a["Tn"], a["eps"], a["theta"],
                                            a["kbar"], a["nb"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(k=None), 1), (dict(w=None), 1), (dict(kpos=None), 1), (dict(kbar=None), 1), (dict(Tn=6), 1),
    (dict(B=-1), 1), (dict(nb=0), 1), (dict(eps=-1.0), 1), (dict(theta=0.0), 1), (dict(theta=float("nan")), 1),
    (dict(k=(1 << 20) + 4), 1), (dict(B=70000), 1), (dict(B=4, nb=1 << 29), 1),
])
def test_qsa_block_keys_rejects_before_launch(over, code):
    assert _qkeys(**over) == code


def test_qsa_block_keys_empty_is_noop():
    assert _qkeys(B=0, k=None, kbar=None) == 0
    assert _qkeys(Tn=0, k=None, kbar=None) == 0


def _qsel(fn="gdn_qsa_select", **over):
    A = 1 << 20
    a = dict(q=A, w=2 * A, qpos=3 * A, kbar=4 * A, nblk=5 * A, B=2, Qn=3, nb=100, eps=1e-6, theta=1e4,
             blocks=6 * A, tokens=None, ws=8 * A, wsb=3072, stream=None)
    a.update(over)
    L = _native.lib()
    head = (a["q"], a["w"], a["qpos"], a["kbar"], a["nblk"], a["B"], a["Qn"], a["nb"], a["eps"], a["theta"])
    if fn == "gdn_qsa_block_scores":
        return L.gdn_qsa_block_scores(*head, a["blocks"], a["stream"])
    return L.gdn_qsa_select(*head, a["blocks"], a["tokens"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(w=None), 1), (dict(qpos=None), 1), (dict(kbar=None), 1), (dict(nblk=None), 1),
    (dict(blocks=None), 1), (dict(Qn=-1), 1), (dict(nb=0), 1), (dict(eps=float("inf")), 1),
    (dict(theta=-1.0), 1), (dict(tokens=(7 << 20) + 4), 1), (dict(ws=None), 3), (dict(wsb=3071), 3),
    (dict(ws=(8 << 20) + 16), 3),
])
def test_qsa_select_rejects_before_launch(over, code):
    assert _qsel(**over) == code


@pytest.mark.parametrize("over,code", [(dict(q=None), 1), (dict(blocks=None), 1), (dict(B=-2), 1),
                                       (dict(blocks=(6 << 20) + 4), 1)])
def test_qsa_block_scores_rejects_before_launch(over, code):
    assert _qsel("gdn_qsa_block_scores", **over) == code


def test_qsa_select_workspace_and_empty():
    n = ctypes.c_size_t(0)
    assert _native.lib().gdn_qsa_select_workspace_size(2, 3, 100, ctypes.byref(n)) == 0
    assert n.value == 3072                      # 2 x 3 rows of 100 fp32 scores, each padded to 128
    assert _native.lib().gdn_qsa_select_workspace_size(2, 3, 0, ctypes.byref(n)) == 1
    assert _qsel(Qn=0, q=None, blocks=None, ws=None) == 0
    assert _qsel("gdn_qsa_block_scores", B=0, q=None, blocks=None) == 0


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(_native, "LIB_PATH", os.path.join(ROOT, "tests", "no-such-dir", "missing.so"))
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        _native.lib()


def test_product_does_not_import_oracle():
    pkg = os.path.join(ROOT, "linear_attention_recurrence_05_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f


def test_qsa_binding_rejects_host_tensors_and_dtypes():
    import torch
    import linear_attention_recurrence_05_b200 as gdn
    k = torch.zeros((1, 8, 128), dtype=torch.bfloat16)
    kbar = torch.zeros((1, 4, 128), dtype=torch.bfloat16)
    w = torch.ones(128)
    pos = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(TypeError):
        gdn.qsa_block_keys(k, w, pos, kbar)                        # host tensors
    q = torch.zeros((1, 2, 4, 128), dtype=torch.float32)
    with pytest.raises(TypeError):
        gdn.qsa_select(q, w, pos, kbar, pos)                        # fp32 queries
    with pytest.raises(TypeError):
        gdn.qsa_block_scores(q.to(torch.bfloat16), w, pos.long(), kbar, pos)   # int64 positions
