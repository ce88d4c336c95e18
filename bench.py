#!/usr/bin/env python
"""Throughput of libgdn (the Gated DeltaNet token mixer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  `value` is prefill tokens/s of one GDN layer at the
pages' shape (T = 8192, 16 QK / 48 V heads, d = 128, bf16 inputs, fp32 state, fp32
output) with inputs resident in HBM and L2 flushed between steps; the `decode` object
is the batched decode workload (256 rows x 1024 consecutive steps on resident fp32
states).  `e2e` repeats the prefill measurement through the public API from pinned
host buffers, every step's copies included (uploads, kernels and downloads of
consecutive steps overlap on three streams).  `roofline` describes the dominant prefill kernel,
timed live with the library's launch trace; its `traffic` is the DRAM bytes of one launch from
an ncu capture recorded in the profile summaries together with the sha256 of the kernel
sources it was built from, and is null when the sources have changed since.  `step` gives the
whole prefill step against the TF32 and bf16 tensor peaks.  `prefill_longctx` (T = 262,144,
mean alpha 0.98) and `prefill_varlen` (32 packed sequences of log-uniform lengths with initial
states) are the two other prefill workloads, each with its roofline and oracle baseline.
`prefill_gated` is the headline prefill with the output tail (gated RMS norm) fused into the
store of y, beside the same two steps unfused.  `cpu_baseline` is the fp64 oracle on all host
cores and `cpu_baseline_1core` on one (rank 0, N = 1 only).  `qsa` holds the QSA indexer's two workloads (chunked
prefill: 8192 queries at 64K context; decode: 64 rows x 4 tokens at 128K) in query tokens/s
with the rooflines of its scores and top-512 kernels; `--qsa-only` runs just those.

With N > 1 (torchrun), every rank runs its own independent problem of the same size
(the path shards by sequence with no exchange): weak scaling, no data-path collective;
the time is the max over ranks.  `--impl reference` times the oracle instead (the
only reference this path has), rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gdn_inputs as gi  # noqa: E402

METRIC = "GDN prefill tokens/s and decode tokens/s on 1 B200; % of tensor/HBM roofline"
UNIT = "tokens/s"
D = 128
CHUNK = 64
# algorithmic work of the chunked prefill per (token, V head), full 64-row tiles:
# W.S, K~^T.u, Q.S (2 d^2 each) + T.(beta gamma K), T.(beta V), P.u (2 C d each)
# + K.K^T and Q.K^T (2 C d each, shared by the 3 V heads of a QK head)
PREFILL_FLOP_TV = 6 * D * D + 2 * CHUNK * D * (3 + 2 / 3)
# the same counting only the triangles the chunked form needs: K.K^T and Q.K^T half each
# (shared by 3 V heads: 1/3 together), T.(beta gamma K), T.(beta V) and P.u half each
PREFILL_FLOP_TV_TRI = 6 * D * D + 2 * CHUNK * D * 11 / 6
# tensor-core work of the chunk-chain kernel per (token, V head): S^T[K;Q]^T (4 d^2) and
# X T_beta_gamma^T (2 C d) on TF32 operands (5/9 of it); V^T T_beta^T (2 C d), u~^T K (2 d^2)
# and u^T P^T (2 C d) on fp16 operands (4/9)
CHAIN_FLOP_TV_TF32 = 4 * D * D + 2 * CHUNK * D
CHAIN_FLOP_TV_F16 = 2 * D * D + 2 * 2 * CHUNK * D
CHAIN_FLOP_TV = CHAIN_FLOP_TV_TF32 + CHAIN_FLOP_TV_F16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
TF32_PER_BF16 = 1.1 / 2.25   # nominal dense tf32 : bf16 tensor throughput on B200
FP32_LANES_PER_SM = 128
N_SM = 148


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples (200 ms) while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.device_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(",") for r in self.tmp.read().strip().splitlines() if r.count(",") >= 7]
        self.tmp.close()
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx.append(float(r[1]))
            except ValueError:
                continue
            for name, val in zip(names, r[4:8]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def device_id_for_smi() -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")
        return vis[torch.cuda.current_device()] if vis and vis[0] else "0"


# ----------------------------------------------------------------------------- helpers
def to_dev(a, torch):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


class Dist:
    """Ranks of a torchrun launch (RANK / LOCAL_RANK / WORLD_SIZE from the environment): NCCL
    on the local GPU for the timed runs; the same logic over gloo on the CPU in the tests."""

    def __init__(self, torch, backend: str = "nccl", device: str = "cuda"):
        self.torch = torch
        self.backend, self.device = backend, device
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self):
        import datetime
        torch = self.torch
        if self.device == "cuda":
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import torch.distributed as dist
            kw = {"device_id": torch.device("cuda", self.local)} if self.device == "cuda" else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist
        return self

    def barrier(self):
        if self.pg:
            self.pg.barrier()
        if self.device == "cuda":
            self.torch.cuda.synchronize()

    def max(self, x: float) -> float:
        """The largest x over the ranks (a step's time is the slowest rank's)."""
        if not self.pg:
            return x
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def gpu_gate_inputs(torch, gen, shape, c, dtype):
    x = torch.randn(shape, generator=gen, device="cuda")
    alpha = torch.exp(-c * torch.nn.functional.softplus(x)).to(dtype)
    beta = torch.sigmoid(torch.randn(shape, generator=gen, device="cuda")).to(dtype)
    return alpha, beta


# ----------------------------------------------------------------------------- prefill
def device_prefill_problem(torch, gdn, idx, rank):
    """Device-resident inputs of prefill workload ``idx`` (1, 2 or 4), each rank its own draw.

    Workload 1 is drawn on the host by the seeded input module (the same bytes the parity
    tests give the oracle); workloads 2 and 4 are drawn on the device with a seeded torch
    generator from the same distributions (their size makes host draws slow).  Workload 4's
    initial states and conv states are the final states of a seeded 2048-token prefill per
    sequence, made by libgdn itself (timing inputs only, never compared with anything)."""
    w = gi.WORKLOADS[idx]
    shape = w["shape"]
    H, Hv = shape.n_qk_heads, shape.n_v_heads
    bf = torch.bfloat16
    cfg = gdn.GdnConfig(H, Hv)
    wq, wk, wv = (to_dev(x, torch) for x in gi.workload_weights(idx))
    p = {"cfg": cfg, "wq": wq, "wk": wk, "wv": wv, "init": None, "conv_in": None, "name": w["name"]}
    if idx == 1:
        T = w["lengths"][0]
        inp = gi.make_prefill_inputs(shape, [T], w["dtype"], gi.workload_seed(1) + 7919 * rank, c=w["c"],
                                     weights=gi.workload_weights(1))
        p.update(q=to_dev(inp.q, torch), k=to_dev(inp.k, torch), v=to_dev(inp.v, torch),
                 al=to_dev(inp.alpha, torch), be=to_dev(inp.beta, torch),
                 cu=torch.from_numpy(inp.cu_seqlens).cuda(), lengths=[T])
        return p
    gen = torch.Generator(device="cuda")
    gen.manual_seed(gi.workload_seed(idx) + 7919 * rank)
    lengths = list(w["lengths"]) if idx == 2 else [int(x) for x in gi.varlen_lengths(idx)]
    T, n = sum(lengths), len(lengths)
    cu = torch.zeros(n + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    p.update(q=torch.randn((T, H, D), generator=gen, device="cuda").to(bf),
             k=torch.randn((T, H, D), generator=gen, device="cuda").to(bf),
             v=torch.randn((T, Hv, D), generator=gen, device="cuda").to(bf),
             cu=cu.cuda(), lengths=lengths)
    p["al"], p["be"] = gpu_gate_inputs(torch, gen, (T, Hv), w["c"], bf)
    if idx == 4:
        Tw = w["warm_tokens"]
        init = torch.empty((n, Hv, D, D), dtype=torch.float32, device="cuda")
        conv = torch.empty((n, 3, cfg.channels), dtype=bf, device="cuda")
        for r0 in range(0, n, 8):
            m = min(8, n - r0)
            q = torch.randn((m * Tw, H, D), generator=gen, device="cuda").to(bf)
            k = torch.randn((m * Tw, H, D), generator=gen, device="cuda").to(bf)
            v = torch.randn((m * Tw, Hv, D), generator=gen, device="cuda").to(bf)
            al, be = gpu_gate_inputs(torch, gen, (m * Tw, Hv), w["c"], bf)
            wcu = torch.arange(m + 1, dtype=torch.int32, device="cuda") * Tw
            gdn.gdn_prefill(q, k, v, wq, wk, wv, al, be, wcu, cfg=cfg, final_state=init[r0:r0 + m],
                            conv_state_out=conv[r0:r0 + m], out=torch.empty((m * Tw, Hv, D), device="cuda"),
                            max_seqlen=Tw)
            del q, k, v, al, be
        torch.cuda.synchronize()
        p["init"], p["conv_in"] = init, conv
    return p


def time_prefill(args, dist, torch, gdn, call, flush, steps):
    """`steps` timed calls (L2 flushed before each, CUDA events around each), after warm-up;
    then the same number under the launch trace for per-kernel durations."""
    for _ in range(args.warmup):
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clocks = ClockSampler(device_id_for_smi())
    dist.barrier()
    clocks.start()
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        call()
        ev[i][1].record()
    dist.barrier()
    clk = clocks.stop()
    ms_max = dist.max(sum(a.elapsed_time(b) for a, b in ev))
    # per-kernel durations: the same steps again under the launch trace (its events add a
    # little time of their own, so the steps above run without it)
    trace = gdn.LaunchTrace(capacity=1024 * steps)
    with trace:
        for _ in range(steps):
            flush.zero_()
            call()
    dist.barrier()
    per_kernel = {}
    for name, t in trace.records():
        per_kernel.setdefault(name, []).append(t)
    return ms_max, clk, {n: {"launches": len(v), "avg_ms": sum(v) / len(v), "total_ms": sum(v)}
                         for n, v in per_kernel.items()}, trace.count


def bench_prefill(args, dist, torch, gdn, peaks, idx=1, e2e=True):
    """Prefill of workload ``idx`` on resident inputs; for the headline workload also the same
    through the public API from pinned host buffers (``e2e``)."""
    p = device_prefill_problem(torch, gdn, idx, dist.rank)
    q, k, v, al, be, cu, cfg = p["q"], p["k"], p["v"], p["al"], p["be"], p["cu"], p["cfg"]
    wq, wk, wv = p["wq"], p["wk"], p["wv"]
    T, n, Hv = q.shape[0], len(p["lengths"]), cfg.n_v_heads
    out = torch.empty((T, Hv, D), dtype=torch.float32, device="cuda")
    fin = torch.empty((n, Hv, D, D), dtype=torch.float32, device="cuda")
    ms = max(p["lengths"])   # the longest sequence, known on the host
    ws = torch.empty(gdn.prefill_workspace_size(cfg, torch.bfloat16, T, n, ms), dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # > 126 MB L2

    def call():
        gdn.gdn_prefill(q, k, v, wq, wk, wv, al, be, cu, cfg=cfg, initial_state=p["init"],
                        conv_state_in=p["conv_in"], out=out, final_state=fin, workspace=ws, max_seqlen=ms)

    K = args.steps if idx == 1 else max(1, min(args.steps, args.long_steps))
    ms_max, clk, per_kernel, launches = time_prefill(args, dist, torch, gdn, call, flush, K)
    tokens_all = T * dist.world * K
    res = {"value": tokens_all / (ms_max / 1e3), "ms_per_step": ms_max / K, "clocks": clk,
           "per_kernel": per_kernel, "launches": launches / K, "tokens_per_step": T, "steps": K,
           "n_v_heads": Hv, "n_qk_heads": cfg.n_qk_heads, "n_seqs": n, "workload": p["name"],
           "workspace_bytes": ws.numel()}
    if not e2e:
        return res

    # e2e: public API from pinned host buffers, every step's copies inside the timed region.
    # Steps run as a pipeline on three streams (upload, compute, download) over two sets of
    # device buffers: step i+1's inputs go up and step i-1's y comes down while step i
    # computes, so the copies of both directions share the bus with the kernels.
    hq, hk, hv = (torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (q, k, v))
    ha, hb = (torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (al, be))
    for h, d in ((hq, q), (hk, k), (hv, v), (ha, al), (hb, be)):
        h.copy_(d)
    host_in = (hq, hk, hv, ha, hb)
    dev_in = [(q, k, v, al, be)] + [tuple(torch.empty_like(x) for x in (q, k, v, al, be))]
    dev_out = [out, torch.empty_like(out)]
    hy = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = hy[0].numel() * hy[0].element_size()
    s_up, s_dn = torch.cuda.Stream(), torch.cuda.Stream()
    comp = torch.cuda.current_stream()

    def ev():
        return torch.cuda.Event()

    def e2e_steps(n_steps):
        up_done, comp_done, dn_done = [], [], []
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(comp)
        s_up.wait_stream(comp)
        s_dn.wait_stream(comp)
        for i in range(n_steps):
            b = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(comp_done[i - 2])      # set b no longer read
                for h, d in zip(host_in, dev_in[b]):
                    d.copy_(h, non_blocking=True)
                up_done.append(ev())
                up_done[i].record(s_up)
            comp.wait_event(up_done[i])
            if i >= 2:
                comp.wait_event(dn_done[i - 2])            # y of set b already read back
            flush.zero_()
            xq, xk, xv, xa, xb = dev_in[b]
            gdn.gdn_prefill(xq, xk, xv, wq, wk, wv, xa, xb, cu, cfg=cfg, out=dev_out[b],
                            final_state=fin, workspace=ws, max_seqlen=ms)
            comp_done.append(ev())
            comp_done[i].record(comp)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(comp_done[i])
                hy[b].copy_(dev_out[b], non_blocking=True)
                dn_done.append(ev())
                dn_done[i].record(s_dn)
        comp.wait_stream(s_up)
        comp.wait_stream(s_dn)
        end.record(comp)
        return start, end

    e2e_steps(max(args.warmup, 3))
    dist.barrier()
    e0, e1 = e2e_steps(K)
    dist.barrier()
    e2e_ms = dist.max(e0.elapsed_time(e1))
    res["e2e"] = {"value": tokens_all / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K}
    return res


# ----------------------------------------------------------------------------- traffic records
_COMMENT_OR_LITERAL = re.compile(r'//[^\n]*|/\*.*?\*/|("(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\')', re.S)


def code_only(text):
    """C/C++/CUDA source with its comments removed (string and character literals kept as
    written) and its blank lines and trailing blanks dropped: the code the compiler turns
    into kernels, less comments and layout."""
    text = _COMMENT_OR_LITERAL.sub(lambda m: m.group(1) or " ", text)
    return "\n".join(ln for ln in (ln.rstrip() for ln in text.split("\n")) if ln)


def kernel_sources_sha256():
    """sha256 over the library's kernel and ABI sources (file names and code with comments
    and blank lines removed, files sorted): the identity of the kernels whose DRAM traffic a
    record describes.  An edit to a comment leaves it unchanged; any change to the code
    changes it."""
    import hashlib
    h = hashlib.sha256()
    roots = [os.path.join(ROOT, "linear_attention_recurrence_05_b200", "csrc"), os.path.join(ROOT, "include")]
    for r in roots:
        for name in sorted(os.listdir(r)):
            if name.endswith((".cu", ".cuh", ".h")):
                h.update(name.encode())
                with open(os.path.join(r, name), encoding="utf-8") as f:
                    h.update(code_only(f.read()).encode())
    return h.hexdigest()


def traffic_records():
    """`traffic-record:` lines of the ncu summaries: DRAM read + write bytes of one launch of a
    kernel, the sources it was built from and the work of that launch.  A record may also name
    larger workloads of the same kernel (`applies_to`) whose launches move the same bytes per
    unit of work, so that their figure scales from the captured one."""
    recs = {}
    pdir = os.path.join(ROOT, "profiles")
    for name in sorted(os.listdir(pdir)) if os.path.isdir(pdir) else []:
        if not name.endswith(".md"):
            continue
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                if line.startswith("traffic-record:"):
                    try:
                        r = json.loads(line.split(":", 1)[1])
                    except ValueError:
                        continue
                    for wl in [r["workload"]] + list(r.get("applies_to", [])):
                        recs[(r["kernel"], wl)] = dict(r, file=name)
    return recs


def traffic_for(kernel, workload, units_per_launch, sha):
    """The recorded per-launch DRAM bytes of `kernel` scaled to `units_per_launch` (tokens or
    rows; the kernels' traffic grows in proportion to them), or None with the reason when no
    record matches the sources that were built."""
    r = traffic_records().get((kernel, workload))
    if r is None:
        return None, "no ncu record"
    if r.get("sources_sha256") != sha:
        return None, f"stale: {r['file']} was captured on other sources"
    return r["bytes_per_launch"] * units_per_launch / r["units_per_launch"], r["file"]


def prefill_roofline(res, peaks, peak_src, sha):
    pk = res["per_kernel"]
    dom = max(pk, key=lambda n: pk[n]["total_ms"])
    avg_s = pk[dom]["avg_ms"] / 1e3
    # a step may run a kernel several times over consecutive chunk ranges (pipelined path):
    # the work of one launch is the step's tokens over its launches per step
    T = res["tokens_per_step"] * res["steps"] / pk[dom]["launches"]
    Hv = res["n_v_heads"]
    step_ms = sum(v["total_ms"] for v in pk.values())
    share = {n: round(v["total_ms"] / step_ms, 4) for n, v in pk.items()}
    bf16 = peaks["bf16_tflops"]
    if dom == "scan_simt":
        flops = PREFILL_FLOP_TV * T * Hv
        peak = N_SM * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        return {"kernel": dom, "bound": "alu", "achieved": flops / avg_s / 1e12, "peak": peak,
                "unit": "TFLOP/s", "frac": flops / avg_s / 1e12 / peak, "traffic": None,
                "peak_source": f"148 SMs x 128 fp32 FMA lanes x 2 x {peaks.get('sm_max_mhz')} MHz",
                "algorithmic_per_launch": flops, "tokens_per_launch": T, "kernel_share": share}
    if dom.startswith("prefill_tc"):
        flops = CHAIN_FLOP_TV * T * Hv
        # the time the chain's MMAs take at peak: the TF32 part at the TF32 rate, the fp16
        # part at the fp16 (= bf16) rate
        tf32 = bf16 * TF32_PER_BF16
        peak = CHAIN_FLOP_TV / (CHAIN_FLOP_TV_TF32 / tf32 + CHAIN_FLOP_TV_F16 / bf16)
        traffic, tsrc = traffic_for(dom, res["workload"], T, sha)
        ach = flops / avg_s / 1e12
        return {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peak,
                "unit": "TFLOP/s", "frac": ach / peak, "frac_of_bf16_peak": ach / bf16,
                "traffic": traffic, "traffic_source": tsrc,
                "peak_source": (f"{peak_src} bf16 {bf16} for the fp16 4/9 of the MMA flops, "
                                f"x 1.1/2.25 nominal (tf32) for the other 5/9"),
                "algorithmic_per_launch": flops, "tokens_per_launch": T, "kernel_share": share}
    # a tile-making pass dominates (chunk prep or the conv pass): its algorithmic bytes per
    # token at the run's head counts, the tiles being what the chain needs and nothing more
    Hq = res["n_qk_heads"]
    if dom == "chunk_prep":
        # reads the [K;Q] tile of every (chunk, QK head); writes T_beta (fp16), T_beta_gamma
        # (fp32), P (fp16) and the gates record of every (chunk, V head)
        per_tok = (Hq * 65536 + Hv * (8192 + 16384 + 8192 + 640)) / CHUNK
    elif dom == "conv_l2":
        # reads q, k, v (bf16); writes the [K;Q] tile (fp32), the K tile and the V tile (fp16)
        per_tok = (2 * Hq * D * 2 + Hv * D * 2) + (2 * Hq * D * 4 + Hq * D * 2 + Hv * D * 2)
    else:
        per_tok = 2 * Hq * D * 2 + Hv * D * 2 + Hv * D * 4
    byts = per_tok * T
    traffic, tsrc = traffic_for(dom, res["workload"], T, sha)
    return {"kernel": dom, "bound": "hbm", "achieved": byts / avg_s / 1e9, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": byts / avg_s / 1e9 / peaks["hbm_gbs"], "traffic": traffic,
            "traffic_source": tsrc, "peak_source": peak_src, "algorithmic_per_launch": byts,
            "tokens_per_launch": T, "kernel_share": share}


def prefill_step_summary(res, peaks):
    """Whole-step rates of a prefill leg against both tensor peaks and the copy bandwidth.
    The step's minimum bytes per token are the method's own inputs and output: raw q, k, v and
    alpha, beta in bf16 and y in bf16 (32,960 B at 16/48 heads; this path writes y in fp32)."""
    s = res["ms_per_step"] / 1e3
    T = res["tokens_per_step"]
    Hq, Hv = res["n_qk_heads"], res["n_v_heads"]
    flops = PREFILL_FLOP_TV * T * Hv
    tri = PREFILL_FLOP_TV_TRI * T * Hv
    byts = (2 * Hq * D * 2 + Hv * D * 2 + Hv * D * 2 + 2 * Hv * 2) * T
    tf32 = peaks["bf16_tflops"] * TF32_PER_BF16
    return {"tflops": flops / s / 1e12, "frac_of_tf32_peak": flops / s / 1e12 / tf32,
            "frac_of_bf16_peak": flops / s / 1e12 / peaks["bf16_tflops"],
            "algorithmic_flops_per_step": flops,
            "tflops_triangles_only": tri / s / 1e12, "algorithmic_flops_per_step_triangles_only": tri,
            "gbs": byts / s / 1e9, "frac_of_hbm": byts / s / 1e9 / peaks["hbm_gbs"],
            "algorithmic_bytes_per_step": byts}


def bench_prefill_gated(args, dist, torch, gdn, peaks):
    """The headline prefill with the output tail fused into the store of y (gdn_prefill_gated:
    gate input z bf16, gated output bf16), against the same two steps unfused (gdn_prefill with
    fp32 y, then gdn_output_gate); L2 flushed between steps."""
    p = device_prefill_problem(torch, gdn, 1, dist.rank)
    q, k, v, al, be, cu, cfg = p["q"], p["k"], p["v"], p["al"], p["be"], p["cu"], p["cfg"]
    w3 = (p["wq"], p["wk"], p["wv"])
    T, Hv = q.shape[0], cfg.n_v_heads
    gen = torch.Generator(device="cuda")
    gen.manual_seed(gi.workload_seed(1) + 53 + 7919 * dist.rank)
    z = torch.randn((T, Hv, D), generator=gen, device="cuda").to(torch.bfloat16)
    nw = torch.ones(D, device="cuda")
    o = torch.empty((T, Hv, D), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, Hv, D), dtype=torch.float32, device="cuda")
    fin = torch.empty((1, Hv, D, D), dtype=torch.float32, device="cuda")
    ws = torch.empty(gdn.prefill_workspace_size(cfg, torch.bfloat16, T, 1, T), dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def fused():
        gdn.gdn_prefill(q, k, v, *w3, al, be, cu, cfg=cfg, out=o, final_state=fin, workspace=ws, max_seqlen=T,
                        gate=(z, nw, 1e-6))

    def unfused():
        gdn.gdn_prefill(q, k, v, *w3, al, be, cu, cfg=cfg, out=y, final_state=fin, workspace=ws, max_seqlen=T)
        gdn.gdn_output_gate(y, z, nw, cfg=cfg, out=o)

    res = {}
    for name, fn in (("fused", fused), ("unfused", unfused)):
        ms, _, per_kernel, _ = time_prefill(args, dist, torch, gdn, fn, flush, args.steps)
        res[name] = {"value": T * dist.world * args.steps / (ms / 1e3), "ms_per_step": ms / args.steps,
                     "kernels": {n: round(v["avg_ms"], 4) for n, v in per_kernel.items()}}
    return {"value": res["fused"]["value"], "unit": UNIT, "workload": f"{p['name']}+gated-rmsnorm-out-bf16",
            "ms_per_step": res["fused"]["ms_per_step"], "unfused": res["unfused"]}


def bench_output_gate(args, dist, torch, gdn, peaks, peak_src):
    """The output tail on a prefill output of the workload's shape: y fp32 [T, Hv, 128] (as
    gdn_prefill returns it), gate z bf16, out bf16; L2 flushed between steps."""
    w = gi.WORKLOADS[1]
    T, Hv = w["lengths"][0], w["shape"].n_v_heads
    gen = torch.Generator(device="cuda")
    gen.manual_seed(gi.workload_seed(1) + 31 + 7919 * dist.rank)
    y = torch.randn((T, Hv, D), generator=gen, device="cuda")
    z = torch.randn((T, Hv, D), generator=gen, device="cuda").to(torch.bfloat16)
    nw = torch.ones(D, device="cuda")
    out = torch.empty((T, Hv, D), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    cfg = gdn.GdnConfig(w["shape"].n_qk_heads, Hv)
    for _ in range(args.warmup):
        gdn.gdn_output_gate(y, z, nw, cfg=cfg, out=out)
    K = args.steps
    trace = gdn.LaunchTrace(capacity=K + 4)
    dist.barrier()
    with trace:
        for _ in range(K):
            flush.zero_()
            gdn.gdn_output_gate(y, z, nw, cfg=cfg, out=out)
    dist.barrier()
    recs = [t for n, t in trace.records() if n == "output_gate"]
    avg_ms = dist.max(sum(recs) / len(recs))
    byts = T * Hv * D * (4 + 2 + 2)
    achieved = byts / (avg_ms / 1e3) / 1e9
    return {"value": T * dist.world / (avg_ms / 1e3), "unit": UNIT, "workload": f"output-gate-T{T}-h{Hv}",
            "ms_per_step": avg_ms,
            "roofline": {"kernel": "output_gate", "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "peak_source": peak_src, "algorithmic_bytes_per_launch": byts}}


# ----------------------------------------------------------------------------- QSA indexer
QSA_FLOP_PER_CAND = 4 * D * 2       # per (query, candidate block): 4 head dot products of 128
QSA_UNIT = "query tokens/s"


def qsa_candidates(B, T, Qn):
    """Candidate blocks summed over the queries (positions T-Qn .. T-1 of each row)."""
    i = np.arange(T - Qn, T, dtype=np.int64)
    return int(B * np.sum((i + 1) // 4))


def bench_qsa(args, dist, torch, gdn, peaks, peak_src, wl):
    """QSA indexer step on resident inputs: the step's new block keys into the cache, then the
    block scores and top-512 selection of its queries (token sets included); L2 flushed
    between steps.  prefill: 8192 queries at the end of a 64K-token sequence; decode: 64 rows
    x 4 query tokens at 128K (the newest block completes within the step)."""
    cfg = gi.QSA_PREFILL if wl == "prefill" else gi.QSA_DECODE
    B, T, Qn, eps, theta = cfg["B"], cfg["context"], cfg["queries"], cfg["eps"], cfg["theta"]
    nb = T // 4
    gen = torch.Generator(device="cuda")
    gen.manual_seed(gi.BASE_SEED + 4242 + (0 if wl == "prefill" else 1) + 7919 * dist.rank)
    k = torch.randn((B, T, D), generator=gen, device="cuda").to(torch.bfloat16)
    q = torch.randn((B, Qn, 4, D), generator=gen, device="cuda").to(torch.bfloat16)
    w_k = torch.rand(D, generator=gen, device="cuda") + 0.5
    w_q = torch.rand(D, generator=gen, device="cuda") + 0.5
    new0 = T - Qn if wl == "prefill" else T - 4        # first token whose key the step adds
    kbar = torch.zeros((B, nb, D), dtype=torch.bfloat16, device="cuda")
    i32 = torch.int32
    gdn.qsa_block_keys(k[:, :new0].contiguous(), w_k, torch.zeros(B, dtype=i32, device="cuda"), kbar,
                       eps=eps, theta=theta)
    k_new = k[:, new0:].contiguous()
    kpos = torch.full((B,), new0, dtype=i32, device="cuda")
    qpos = torch.full((B,), T - Qn, dtype=i32, device="cuda")
    nblk = torch.full((B,), nb, dtype=i32, device="cuda")
    blocks = torch.empty((B, Qn, gdn.QSA_BUDGET), dtype=i32, device="cuda")
    tokens = torch.empty((B, Qn, gdn.QSA_TOKEN_SLOTS), dtype=i32, device="cuda")
    ws = torch.empty(gdn.qsa_select_workspace_size(B, Qn, nb), dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def step():
        gdn.qsa_block_keys(k_new, w_k, kpos, kbar, eps=eps, theta=theta)
        gdn.qsa_select(q, w_q, qpos, kbar, nblk, eps=eps, theta=theta, blocks=blocks, tokens=tokens,
                       workspace=ws)

    for _ in range(args.warmup):
        step()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    dist.barrier()
    for i in range(K):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    dist.barrier()
    ms = dist.max(sum(a.elapsed_time(b) for a, b in ev)) / K
    trace = gdn.LaunchTrace(capacity=4 * K + 8)
    with trace:
        for _ in range(K):
            flush.zero_()
            step()
    dist.barrier()
    per = {}
    for n, t in trace.records():
        per.setdefault(n, []).append(t)
    per_kernel = {n: {"launches": len(v), "avg_ms": sum(v) / len(v), "total_ms": sum(v)} for n, v in per.items()}
    cand = qsa_candidates(B, T, Qn)
    sc_s = per_kernel["qsa_scores"]["avg_ms"] / 1e3
    flops = cand * QSA_FLOP_PER_CAND
    byts = cand * 4 + B * nb * D * 2 + B * Qn * 4 * D * 2       # scores out, keys and queries in
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        roof = {"kernel": "qsa_scores", "bound": "tensor", "achieved": flops / sc_s / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": flops / sc_s / 1e12 / peaks["bf16_tflops"]}
    else:
        roof = {"kernel": "qsa_scores", "bound": "hbm", "achieved": byts / sc_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": byts / sc_s / 1e9 / peaks["hbm_gbs"]}
    roof.update({"traffic": None, "peak_source": peak_src, "algorithmic_flops_per_launch": flops,
                 "algorithmic_bytes_per_launch": byts, "candidates_per_launch": cand})
    tk_s = per_kernel["qsa_topk"]["avg_ms"] / 1e3
    tk_bytes = cand * 4 + B * Qn * (gdn.QSA_BUDGET + gdn.QSA_TOKEN_SLOTS) * 4
    topk = {"kernel": "qsa_topk", "bound": "hbm", "achieved": tk_bytes / tk_s / 1e9, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": tk_bytes / tk_s / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": tk_bytes}
    return {"value": B * Qn * dist.world / (ms / 1e3), "unit": QSA_UNIT, "ms_per_step": ms,
            "workload": f"qsa-{wl}-B{B}-ctx{T}-q{Qn}", "kernels": per_kernel, "roofline": roof, "topk": topk,
            "l2": "flushed: 256 MiB write between steps"}


def qsa_oracle_rows_per_s(target_s: float):
    """The oracle on sampled query rows of the prefill workload (one row = its 4 heads
    against every candidate block, then the top-512 and token set)."""
    from oracle import qsa_indexer as qi
    cfg = gi.QSA_PREFILL
    T, Qn = cfg["context"], cfg["queries"]
    inp = gi.make_qsa_inputs(1, T, 8, seed=77)
    k64 = gi.bf16_bits_to_f32(inp.k[0]).astype(np.float64)
    q64 = gi.bf16_bits_to_f32(inp.q[0]).astype(np.float64)
    t0 = time.perf_counter()
    kb = qi.block_keys(k64, inp.w_k, cfg["eps"], cfg["theta"], operands="bf16")
    rows = 0
    while True:
        j = rows % 8
        i = T - Qn + j * (Qn // 8)
        qh = qi.query_heads(q64[j:j + 1], inp.w_q, [i], cfg["eps"], cfg["theta"], operands="bf16")
        s = qi.block_scores(qh, kb, [i])[0]
        qi.token_set(qi.top_blocks(s), i)
        rows += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            return rows / dt, rows, dt


# ----------------------------------------------------------------------------- decode
def decode_bytes_per_row(shape, in_bytes=2, out_bytes=4):
    Hqk, Hv = shape.n_qk_heads, shape.n_v_heads
    ch = shape.channels
    return (2 * Hv * D * D * 4            # state read + write
            + 6 * ch * in_bytes           # conv state: 3 rows read, 3 rows written
            + ch * in_bytes               # this step's raw q, k, v
            + Hv * D * out_bytes          # y
            + 2 * Hv * in_bytes)          # alpha, beta


def bench_decode(args, dist, torch, gdn, peaks, peak_src):
    w = gi.WORKLOADS[3]
    shape = w["shape"]
    B, steps, warm_T = w["batch"], args.decode_steps, w["warm_tokens"]
    H, Hv, ch = shape.n_qk_heads, shape.n_v_heads, shape.channels
    bf = torch.bfloat16
    gen = torch.Generator(device="cuda")
    gen.manual_seed(gi.workload_seed(3) + 7919 * dist.rank)
    wq, wk, wv = (to_dev(x, torch) for x in gi.workload_weights(3))
    cfg = gdn.GdnConfig(H, Hv)
    # resident states: final states of a seeded warm_T-token prefill per row (libgdn prefill)
    state = torch.empty((B, Hv, D, D), dtype=torch.float32, device="cuda")
    conv = torch.empty((B, 3, ch), dtype=bf, device="cuda")
    per = 32
    for r0 in range(0, B, per):
        n = min(per, B - r0)
        Tw = n * warm_T
        q = torch.randn((Tw, H, D), generator=gen, device="cuda").to(bf)
        k = torch.randn((Tw, H, D), generator=gen, device="cuda").to(bf)
        v = torch.randn((Tw, Hv, D), generator=gen, device="cuda").to(bf)
        al, be = gpu_gate_inputs(torch, gen, (Tw, Hv), w["c"], bf)
        cu = torch.arange(n + 1, dtype=torch.int32, device="cuda") * warm_T
        gdn.gdn_prefill(q, k, v, wq, wk, wv, al, be, cu, cfg=cfg, final_state=state[r0:r0 + n],
                        conv_state_out=conv[r0:r0 + n], out=torch.empty((Tw, Hv, D), device="cuda"),
                        max_seqlen=warm_T)
        del q, k, v, al, be
    torch.cuda.synchronize()
    # fresh inputs for every step
    dq = torch.randn((steps, B, H, D), generator=gen, device="cuda").to(bf)
    dk = torch.randn((steps, B, H, D), generator=gen, device="cuda").to(bf)
    dv = torch.randn((steps, B, Hv, D), generator=gen, device="cuda").to(bf)
    da, db = gpu_gate_inputs(torch, gen, (steps, B, Hv), w["c"], bf)
    out = torch.empty((B, Hv, D), dtype=torch.float32, device="cuda")
    state0, conv0 = state.clone(), conv.clone()

    def step(i):
        gdn.gdn_decode_step(dq[i], dk[i], dv[i], wq, wk, wv, da[i], db[i], state, conv, cfg=cfg,
                            out=out)

    for i in range(args.warmup):
        step(i % steps)
    state.copy_(state0)
    conv.copy_(conv0)
    trace = gdn.LaunchTrace(capacity=steps + 8)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device_id_for_smi())
    dist.barrier()
    clocks.start()
    with trace:
        e0.record()
        for i in range(steps):
            step(i)
        e1.record()
    dist.barrier()
    clk = clocks.stop()
    ms = dist.max(e0.elapsed_time(e1))
    recs = [t for n, t in trace.records() if n == "decode"]
    avg_s = sum(recs) / len(recs) / 1e3
    bpr = decode_bytes_per_row(shape)
    achieved = bpr * B / avg_s / 1e9
    bpr_min = decode_bytes_per_row(shape, out_bytes=2)   # the minimum: y in bf16

    # e2e: pinned host inputs (a ring of 32 distinct steps), y read back every step
    ring = 32
    hq, hk, hv, ha, hb = (torch.empty((ring,) + tuple(x.shape[1:]), dtype=x.dtype, pin_memory=True)
                          for x in (dq, dk, dv, da, db))
    for h, d in ((hq, dq), (hk, dk), (hv, dv), (ha, da), (hb, db)):
        h.copy_(d[:ring])
    hy = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(x[0].numel() * x.element_size() for x in (hq, hk, hv, ha, hb))
    d2h = hy.numel() * hy.element_size()
    bq, bk, bv, ba, bb = (torch.empty_like(x[0]) for x in (dq, dk, dv, da, db))
    state.copy_(state0)
    conv.copy_(conv0)
    dist.barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record()
    for i in range(steps):
        j = i % ring
        for d, h in ((bq, hq), (bk, hk), (bv, hv), (ba, ha), (bb, hb)):
            d.copy_(h[j], non_blocking=True)
        gdn.gdn_decode_step(bq, bk, bv, wq, wk, wv, ba, bb, state, conv, cfg=cfg, out=out)
        hy.copy_(out, non_blocking=True)
    e3.record()
    dist.barrier()
    e2e_ms = dist.max(e2.elapsed_time(e3))
    toks = B * steps * dist.world
    dec_traffic, dec_tsrc = traffic_for("decode", w["name"], B, kernel_sources_sha256())
    multi = bench_decode_multi(args, dist, torch, gdn, peaks, peak_src, shape, cfg, (wq, wk, wv),
                               (dq, dk, dv, da, db), state, conv, state0, conv0)
    return {
        "multi": multi,
        "value": toks / (ms / 1e3), "unit": UNIT, "workload": w["name"], "batch": B,
        "steps": steps, "ms_per_step": ms / steps, "launches": trace.count, "clocks": clk,
        "roofline": {"kernel": "decode", "bound": "hbm", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": dec_traffic, "traffic_source": dec_tsrc, "peak_source": peak_src,
                     "algorithmic_bytes_per_row": bpr, "rows_per_launch": B,
                     "frac_of_min_bytes": bpr_min * B / avg_s / 1e9 / peaks["hbm_gbs"],
                     "min_bytes_per_row": bpr_min},
        "e2e": {"value": toks / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "note": "host inputs cycle through 32 pinned step sets"},
    }


def bench_decode_multi(args, dist, torch, gdn, peaks, peak_src, shape, cfg, wts, inputs, state, conv,
                       state0, conv0, n_tok=4):
    """The same token stream as the single-token run, n_tok tokens per call per row
    (multi-token verification step): tokens/s, and the HBM roofline of the call."""
    dq, dk, dv, da, db = inputs
    steps, B = dq.shape[0], dq.shape[1]
    calls = steps // n_tok
    if calls == 0:
        return None
    # [steps, B, ...] -> [calls, B, n_tok, ...]
    mq, mk, mv, ma, mb = (x[:calls * n_tok].view((calls, n_tok) + tuple(x.shape[1:])).transpose(1, 2).contiguous()
                          for x in (dq, dk, dv, da, db))
    out = torch.empty((B, n_tok, shape.n_v_heads, D), dtype=torch.float32, device="cuda")

    def call(i, **kw):
        gdn.gdn_decode_multi(mq[i], mk[i], mv[i], *wts, ma[i], mb[i], state, conv, cfg=cfg, out=out, **kw)

    def timed(**kw):
        state.copy_(state0)
        conv.copy_(conv0)
        for i in range(min(args.warmup, calls)):
            call(i, **kw)
        state.copy_(state0)
        conv.copy_(conv0)
        trace = gdn.LaunchTrace(capacity=calls + 8)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        with trace:
            e0.record()
            for i in range(calls):
                call(i, **kw)
            e1.record()
        dist.barrier()
        recs = [t for n, t in trace.records() if n == "decode_multi"]
        return dist.max(e0.elapsed_time(e1)), sum(recs) / len(recs) / 1e3

    ms, avg_s = timed()
    ch, Hv = shape.channels, shape.n_v_heads
    bpr = (2 * Hv * D * D * 4 + 6 * ch * 2 + n_tok * (ch * 2 + Hv * D * 4 + 2 * Hv * 2))
    achieved = bpr * B / avg_s / 1e9
    # with the state and conv state after every token written out (rollback checkpoints)
    ck = torch.empty((B, n_tok, Hv, D, D), dtype=torch.float32, device="cuda")
    cck = torch.empty((B, n_tok, 3, ch), dtype=conv.dtype, device="cuda")
    ms_ck, _ = timed(state_ckpt=ck, conv_ckpt=cck)
    del ck, cck
    toks = B * calls * n_tok * dist.world
    return {"value": toks / (ms / 1e3), "unit": UNIT, "n_tok": n_tok, "calls": calls, "batch": B,
            "ms_per_call": ms / calls, "value_with_checkpoints": toks / (ms_ck / 1e3),
            "roofline": {"kernel": "decode_multi", "bound": "hbm", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": None, "peak_source": peak_src, "algorithmic_bytes_per_row": bpr,
                         "rows_per_launch": B}}


# ----------------------------------------------------------------------------- oracle
def oracle_tokens_per_s(target_s: float, idx: int = 1, n_threads=None, seed_offset: int = 0):
    """Time the fp64 oracle on a bounded sample of prefill workload ``idx`` (all 48 V heads),
    sized to take about target_s seconds: the first T tokens of a seeded draw of the workload's
    distributions (workload 4: one sequence of the set's first length, with an initial state and
    a conv state).  The oracle's cost per token does not depend on the values, so tokens/s of
    the sample is the rate of the whole workload.  Returns (tokens/s, threads, sample, secs)."""
    import oracle
    w = gi.WORKLOADS[idx]
    threads = n_threads or oracle.default_threads()
    cap = w["lengths"][0] if idx != 4 else int(gi.varlen_lengths(idx)[0])

    def run(T):
        inp = gi.make_prefill_inputs(w["shape"], [T], w["dtype"], gi.workload_seed(idx) + seed_offset,
                                     c=w["c"], weights=gi.workload_weights(idx),
                                     with_initial_state=idx == 4, with_conv_state=idx == 4)
        t0 = time.perf_counter()
        oracle.prefill(inp, n_threads=threads)
        return time.perf_counter() - t0
    probe_T = 64 if threads == 1 else 128
    dt = run(probe_T)
    T = int(min(cap, 8192, max(probe_T, probe_T * target_s / max(dt, 1e-6))))
    dt = run(T)
    what = {1: "the T=8192 layer", 2: "the T=262,144 sequence (mean alpha 0.98)",
            4: "the first packed sequence, with initial and conv state"}[idx]
    return T / dt, threads, f"first {T} tokens of {what}, all 48 V heads, {threads} thread(s)", dt


def cpu_baseline(idx, target_s, n_threads=None):
    v, threads, sample, dt = oracle_tokens_per_s(target_s, idx, n_threads)
    return {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample, "seconds": dt}


def headline_config(world):
    """`config` of the JSON line: the headline prefill workload (both arms print the same)."""
    return {"workload": gi.WORKLOADS[1]["name"], "T": 8192, "n_qk_heads": 16, "n_v_heads": 48, "d": D,
            "chunk": CHUNK, "inputs": "bf16", "out": "f32", "state": "f32",
            "l2": "flushed: 256 MiB write between steps",
            "parallelism": f"dp{world} (independent sequences per GPU)"}


def run_reference(args):
    """--impl reference: the fp64 oracle timed on the host cores (rank 0 only)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    oracle.build()
    for _ in range(args.warmup):
        oracle_tokens_per_s(0.2)
    vals, secs, sample, threads = [], [], "", 1
    for _ in range(args.steps):
        v, threads, sample, dt = oracle_tokens_per_s(args.ref_step_s)
        vals.append(v)
        secs.append(dt)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": headline_config(world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-long", action="store_true", help="skip the long-context and varlen prefill legs")
    ap.add_argument("--long-steps", type=int, default=5, help="timed steps of those legs (at most --steps)")
    ap.add_argument("--no-qsa", action="store_true")
    ap.add_argument("--qsa-only", action="store_true", help="only the QSA indexer legs (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-baseline-s", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=5.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import linear_attention_recurrence_05_b200 as gdn
    dist = Dist(torch).init()
    peaks, peak_src = load_peaks()
    if args.qsa_only:
        qsa = {wl: bench_qsa(args, dist, torch, gdn, peaks, peak_src, wl) for wl in ("prefill", "decode")}
        if dist.rank == 0:
            print(json.dumps({"metric": "QSA indexer query tokens/s", "qsa": qsa, "peaks": peak_src}), flush=True)
        dist.close()
        return
    sha = kernel_sources_sha256()
    pre = bench_prefill(args, dist, torch, gdn, peaks)
    roof = prefill_roofline(pre, peaks, peak_src, sha)
    more = {}
    if not args.no_long:
        for idx, key in ((2, "prefill_longctx"), (4, "prefill_varlen")):
            r = bench_prefill(args, dist, torch, gdn, peaks, idx=idx, e2e=False)
            more[key] = {"value": r["value"], "unit": UNIT, "workload": r["workload"],
                         "ms_per_step": r["ms_per_step"], "steps": r["steps"], "n_seqs": r["n_seqs"],
                         "tokens_per_step": r["tokens_per_step"], "workspace_bytes": r["workspace_bytes"],
                         "gpu_launches_per_step": r["launches"], "clocks": r["clocks"],
                         "roofline": prefill_roofline(r, peaks, peak_src, sha),
                         "step": prefill_step_summary(r, peaks), "kernels": r["per_kernel"]}
            torch.cuda.empty_cache()
    dec = None if args.no_decode else bench_decode(args, dist, torch, gdn, peaks, peak_src)
    tail = bench_output_gate(args, dist, torch, gdn, peaks, peak_src)
    gated = bench_prefill_gated(args, dist, torch, gdn, peaks)
    qsa = None
    if not args.no_qsa:
        qsa = {wl: bench_qsa(args, dist, torch, gdn, peaks, peak_src, wl) for wl in ("prefill", "decode")}
        if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
            v, n, dt = qsa_oracle_rows_per_s(min(5.0, args.cpu_baseline_s))
            qsa["cpu_baseline"] = {"value": v, "unit": QSA_UNIT, "cores": 1, "kind": "oracle",
                                   "sample": f"{n} query rows of qsa-prefill (block keys of the full context once)",
                                   "seconds": dt}
    cpu = cpu1 = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(1, args.cpu_baseline_s)
        cpu1 = cpu_baseline(1, args.cpu_baseline_s / 2, n_threads=1)
        for idx, key in ((2, "prefill_longctx"), (4, "prefill_varlen")):
            if key in more:
                more[key]["cpu_baseline"] = cpu_baseline(idx, args.cpu_baseline_s / 3)
    if dist.rank == 0:
        line = {
            "metric": METRIC, "value": pre["value"], "unit": UNIT, "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "tf32",
            "data": "synthetic",
            "config": headline_config(dist.world),
            "clocks": pre["clocks"], "e2e": pre["e2e"], "gpu_launches": pre["launches"] * args.steps,
            "roofline": roof, "step": prefill_step_summary(pre, peaks), "kernels": pre["per_kernel"],
            "cpu_baseline": cpu, "cpu_baseline_1core": cpu1, **more,
            "decode": dec, "output_gate": tail, "prefill_gated": gated, "qsa": qsa, "peaks": peak_src, "sources_sha256": sha,
        }
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
