"""Seeded synthetic inputs for the Gated DeltaNet token mixer.

This module is the one piece shared by the fp64 oracle (``oracle/``) and the CUDA
path (``linear_attention_recurrence_05_b200``): it draws the random tensors and
quantises them to the storage dtype ONCE, so both sides consume identical bytes.
It holds none of the method's arithmetic (no conv, no normalisation, no
recurrence): only random draws, the gate distributions and bf16 rounding.

Distributions (the workloads of the GDN layer with 48 value heads, 16 QK heads,
head dim 128 and a kernel-4 ShortConv):
  * raw q, k, v ~ N(0, 1)
  * ShortConv weights ~ N(0, 1/4) (standard deviation 0.5), fp32
  * alpha = exp(-c * softplus(x)), x ~ N(0, 1), one value per (token, V head)
    (c = 0.1 gives E[alpha] ~ 0.924; c = 0.025 gives E[alpha] ~ 0.980)
  * beta = sigmoid(N(0, 1)), one value per (token, V head)
Every tensor draws from its own spawned PCG64 stream of one seed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BF16 = "bf16"
F32 = "f32"

# sub-stream order of SeedSequence(seed).spawn(): fixed, one per tensor
_STREAMS = ("q", "k", "v", "w_q", "w_k", "w_v", "x_alpha", "x_beta", "lengths",
            "state", "conv_state")


# --------------------------------------------------------------------------- bf16
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    nan = np.isnan(x)
    out = r.astype(np.uint16)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def stored_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Widen stored values (bf16 bits or fp32) to fp64, exactly."""
    if dtype == BF16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def quantize(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage form of ``x`` in ``dtype``: uint16 bf16 bits or float32."""
    if dtype == BF16:
        return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))
    return np.ascontiguousarray(x, dtype=np.float32)


# --------------------------------------------------------------------------- draws
def _rngs(seed: int) -> dict:
    return _rngs_entropy(seed)


def _rngs_entropy(entropy) -> dict:
    kids = np.random.SeedSequence(entropy).spawn(len(_STREAMS))
    return {name: np.random.Generator(np.random.PCG64(s)) for name, s in zip(_STREAMS, kids)}


def _normal_f32(rng: np.random.Generator, shape, block: int = 1 << 24) -> np.ndarray:
    """N(0,1) in fp32, drawn in blocks so huge tensors need no fp64 temporary."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, block):
        e = min(n, s + block)
        rng.standard_normal(e - s, dtype=np.float32, out=out[s:e])
    return out.reshape(shape)


def _normal_stored(rng: np.random.Generator, shape, dtype: str, block: int = 1 << 24) -> np.ndarray:
    """N(0,1) drawn in fp32 blocks and quantised block by block into the storage dtype."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if dtype == BF16 else np.float32)
    tmp = np.empty(min(block, max(n, 1)), dtype=np.float32)
    for s in range(0, n, block):
        e = min(n, s + block)
        t = tmp[:e - s]
        rng.standard_normal(e - s, dtype=np.float32, out=t)
        out[s:e] = quantize(t, dtype)
    return out.reshape(shape)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def draw_alpha(rng, shape, c: float) -> np.ndarray:
    x = rng.standard_normal(shape)  # fp64
    return np.exp(-c * _softplus(x))


def draw_beta(rng, shape) -> np.ndarray:
    x = rng.standard_normal(shape)
    return 1.0 / (1.0 + np.exp(-x))


def loguniform_lengths(rng, n: int, lo: int, hi: int) -> np.ndarray:
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return np.rint(np.exp(u)).astype(np.int64)


# --------------------------------------------------------------------------- bundles
@dataclass
class GdnShape:
    n_qk_heads: int
    n_v_heads: int
    d_k: int = 128
    d_v: int = 128
    conv_width: int = 4

    @property
    def channels(self) -> int:
        """Width of one raw conv-state row: q | k | v channels."""
        return 2 * self.n_qk_heads * self.d_k + self.n_v_heads * self.d_v


@dataclass
class PrefillInputs:
    """Stored inputs of one prefill call (all host numpy, storage dtype)."""
    shape: GdnShape
    dtype: str
    q: np.ndarray            # [T, Hqk, dk]
    k: np.ndarray            # [T, Hqk, dk]
    v: np.ndarray            # [T, Hv, dv]
    w_q: np.ndarray          # [Hqk*dk, W] fp32
    w_k: np.ndarray          # [Hqk*dk, W] fp32
    w_v: np.ndarray          # [Hv*dv, W] fp32
    alpha: np.ndarray        # [T, Hv]
    beta: np.ndarray         # [T, Hv]
    cu_seqlens: np.ndarray   # [N+1] int32
    initial_state: np.ndarray | None = None   # [N, Hv, dk, dv] fp32
    conv_state: np.ndarray | None = None      # [N, W-1, channels] storage dtype
    meta: dict = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def n_seqs(self) -> int:
        return len(self.cu_seqlens) - 1


def make_conv_weights(shape: GdnShape, seed: int, weight_std: float = 0.5):
    """ShortConv weights of one layer: (w_q, w_k, w_v), fp32, [channels, W]."""
    r = _rngs(seed)
    H, Hv, dk, dv, W = shape.n_qk_heads, shape.n_v_heads, shape.d_k, shape.d_v, shape.conv_width
    w_q = (weight_std * r["w_q"].standard_normal((H * dk, W))).astype(np.float32)
    w_k = (weight_std * r["w_k"].standard_normal((H * dk, W))).astype(np.float32)
    w_v = (weight_std * r["w_v"].standard_normal((Hv * dv, W))).astype(np.float32)
    return w_q, w_k, w_v


def make_prefill_inputs(shape: GdnShape, lengths, dtype: str, seed: int, c: float = 0.1,
                        weight_std: float = 0.5, with_initial_state: bool = False,
                        state_std: float = 0.05, with_conv_state: bool = False,
                        weights=None) -> PrefillInputs:
    """Draw one packed variable-length prefill problem.

    ``lengths`` are the sequence lengths (zero allowed); they are packed back to
    back and described by ``cu_seqlens``.  Optional synthetic initial states are
    N(0, state_std^2) fp32 and optional conv states are N(0,1) raw rows.
    ``weights`` (w_q, w_k, w_v) overrides the conv weights drawn from ``seed``.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    T = int(lengths.sum())
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    r = _rngs(seed)
    H, Hv, dk, dv, W = shape.n_qk_heads, shape.n_v_heads, shape.d_k, shape.d_v, shape.conv_width
    q = _normal_stored(r["q"], (T, H, dk), dtype)
    k = _normal_stored(r["k"], (T, H, dk), dtype)
    v = _normal_stored(r["v"], (T, Hv, dv), dtype)
    w_q, w_k, w_v = weights if weights is not None else make_conv_weights(shape, seed, weight_std)
    alpha = quantize(draw_alpha(r["x_alpha"], (T, Hv), c), dtype)
    beta = quantize(draw_beta(r["x_beta"], (T, Hv)), dtype)
    init = None
    if with_initial_state:
        init = (state_std * _normal_f32(r["state"], (len(lengths), Hv, dk, dv))).astype(np.float32)
    cs = None
    if with_conv_state:
        cs = _normal_stored(r["conv_state"], (len(lengths), W - 1, shape.channels), dtype)
    return PrefillInputs(shape, dtype, q, k, v, w_q, w_k, w_v, alpha, beta, cu, init, cs,
                         meta={"seed": seed, "c": c, "lengths": lengths.tolist()})


@dataclass
class DecodeInputs:
    """Fresh per-step inputs of a decode batch (storage dtype).  Leading axis: steps."""
    q: np.ndarray       # [steps, B, Hqk, dk]
    k: np.ndarray       # [steps, B, Hqk, dk]
    v: np.ndarray       # [steps, B, Hv, dv]
    alpha: np.ndarray   # [steps, B, Hv]
    beta: np.ndarray    # [steps, B, Hv]


def make_decode_step(shape: GdnShape, batch: int, step: int, dtype: str, seed: int,
                     c: float = 0.1) -> DecodeInputs:
    """Inputs of decode step ``step`` alone (its own seed stream: SeedSequence([seed, step]))."""
    r = _rngs_entropy([seed, step])
    H, Hv, dk, dv = shape.n_qk_heads, shape.n_v_heads, shape.d_k, shape.d_v
    return DecodeInputs(
        q=_normal_stored(r["q"], (1, batch, H, dk), dtype),
        k=_normal_stored(r["k"], (1, batch, H, dk), dtype),
        v=_normal_stored(r["v"], (1, batch, Hv, dv), dtype),
        alpha=quantize(draw_alpha(r["x_alpha"], (1, batch, Hv), c), dtype),
        beta=quantize(draw_beta(r["x_beta"], (1, batch, Hv)), dtype),
    )


def make_decode_inputs(shape: GdnShape, batch: int, steps: int, dtype: str, seed: int,
                       c: float = 0.1, first_step: int = 0) -> DecodeInputs:
    """Steps first_step .. first_step+steps-1 stacked (each drawn by make_decode_step)."""
    parts = [make_decode_step(shape, batch, s, dtype, seed, c)
             for s in range(first_step, first_step + steps)]
    return DecodeInputs(*(np.concatenate([getattr(p, f) for p in parts])
                          for f in ("q", "k", "v", "alpha", "beta")))


# --------------------------------------------------------------------------- workloads
BASE_SEED = 20260000
PAGES_SHAPE = GdnShape(n_qk_heads=16, n_v_heads=48)
TINY_SHAPE = GdnShape(n_qk_heads=2, n_v_heads=6)

WORKLOADS = {
    0: dict(name="tiny-fp32-T512-h2x6", shape=TINY_SHAPE, dtype=F32, lengths=[512], c=0.1),
    1: dict(name="layer-bf16-T8192-h16x48", shape=PAGES_SHAPE, dtype=BF16, lengths=[8192], c=0.1),
    2: dict(name="longctx-bf16-T262144-h16x48", shape=PAGES_SHAPE, dtype=BF16, lengths=[262144], c=0.025),
    3: dict(name="decode-bf16-B256x1024steps-h16x48", shape=PAGES_SHAPE, dtype=BF16, batch=256,
            steps=1024, warm_tokens=4096, c=0.1),
    4: dict(name="varlen-bf16-32seqs-logU1k-64k-h16x48", shape=PAGES_SHAPE, dtype=BF16, n_seqs=32,
            len_lo=1024, len_hi=65536, warm_tokens=2048, c=0.1),
}


def workload_seed(index: int) -> int:
    return BASE_SEED + index


def varlen_lengths(index: int = 4) -> np.ndarray:
    w = WORKLOADS[index]
    r = _rngs(workload_seed(index))
    return loguniform_lengths(r["lengths"], w["n_seqs"], w["len_lo"], w["len_hi"])


def make_workload(index: int) -> PrefillInputs:
    """Stored inputs of prefill workloads 0, 1, 2 and 4 (without 4's warm-up states)."""
    w = WORKLOADS[index]
    if index == 3:
        raise ValueError("workload 3 is a decode workload: use make_decode_inputs")
    lengths = varlen_lengths(index) if index == 4 else w["lengths"]
    return make_prefill_inputs(w["shape"], lengths, w["dtype"], workload_seed(index), c=w["c"])


def workload_weights(index: int):
    return make_conv_weights(WORKLOADS[index]["shape"], workload_seed(index))


def warmup_prefill_inputs(index: int, rows) -> PrefillInputs:
    """The seeded prefills whose final states and last raw rows seed workloads 3 and 4.

    One ``warm_tokens``-token sequence per decode row / packed sequence in ``rows``
    (each row has its own seed stream, so any subset can be drawn alone), run
    through the same layer (the workload's conv weights); returned packed.
    """
    w = WORKLOADS[index]
    rows = [int(r) for r in rows]
    parts = [make_prefill_inputs(w["shape"], [w["warm_tokens"]], w["dtype"],
                                 [workload_seed(index), 1000, r], c=w["c"],
                                 weights=workload_weights(index)) for r in rows]
    first = parts[0]
    cat = {f: np.concatenate([getattr(p, f) for p in parts]) for f in ("q", "k", "v", "alpha", "beta")}
    cu = np.arange(len(rows) + 1, dtype=np.int32) * w["warm_tokens"]
    return PrefillInputs(w["shape"], w["dtype"], cat["q"], cat["k"], cat["v"], first.w_q, first.w_k,
                         first.w_v, cat["alpha"], cat["beta"], cu, meta={"rows": rows})


def decode_workload_step(step: int, index: int = 3) -> DecodeInputs:
    """Inputs of one step of the decode workload (all rows)."""
    w = WORKLOADS[index]
    return make_decode_step(w["shape"], w["batch"], step, w["dtype"], workload_seed(index) + 2000,
                            c=w["c"])


# --------------------------------------------------------------------------- QSA indexer
# The indexer's inputs are projections of the hidden state (outside the path): raw key
# rows [B, T, 128] and query heads [B, Qn, 4, 128], N(0, 1) stored as bf16, and the two
# RMSNorm weights ~ U(0.5, 1.5) in fp32.  The workloads are the pages' indexer setting
# (r = 4, 512-block budget) at long context: a chunk of queries at the end of a sequence
# whose block-key cache covers all earlier tokens.
_QSA_STREAMS = ("k", "q", "w_k", "w_q")


@dataclass
class QsaInputs:
    k: np.ndarray      # uint16 bf16 bits [B, T, 128]
    q: np.ndarray      # uint16 bf16 bits [B, Qn, 4, 128]
    w_k: np.ndarray    # float32 [128]
    w_q: np.ndarray    # float32 [128]


def make_qsa_inputs(B: int, T: int, Qn: int, seed: int) -> QsaInputs:
    kids = np.random.SeedSequence([seed, 0x05A]).spawn(len(_QSA_STREAMS))
    r = {n: np.random.Generator(np.random.PCG64(s)) for n, s in zip(_QSA_STREAMS, kids)}
    return QsaInputs(k=_normal_stored(r["k"], (B, T, 128), BF16),
                     q=_normal_stored(r["q"], (B, Qn, 4, 128), BF16),
                     w_k=r["w_k"].uniform(0.5, 1.5, 128).astype(np.float32),
                     w_q=r["w_q"].uniform(0.5, 1.5, 128).astype(np.float32))


# chunked prefill at 64K context: 8192 query tokens (positions 57344..65535) of one
# sequence over its 16384 block keys
QSA_PREFILL = {"B": 1, "context": 65536, "queries": 8192, "theta": 10000.0, "eps": 1e-6}
# decode with 3 speculative tokens: 64 rows x 4 query tokens at 128K context
QSA_DECODE = {"B": 64, "context": 131072, "queries": 4, "theta": 10000.0, "eps": 1e-6}
