"""Host logic of bench.py that decides whether an ncu traffic record still describes the
kernels being timed: the comment-insensitive source hash and the record lookup."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_only_drops_comments_and_layout(bench):
    src = ("// file header\n"
           "#include \"a.h\"   \n"
           "\n"
           "/* block\n   comment */ int x = 1; // trailing\n"
           "int y = x /* inline */ + 2;\n"
           "\n\n")
    assert bench.code_only(src) == '#include "a.h"\n  int x = 1;\nint y = x   + 2;'


def test_code_only_keeps_literals(bench):
    src = ('asm("tanh.approx.f32 %0, %1; // not a comment /* nor this */" : "=f"(t));\n'
           "char c = '/'; char d = '\\''; const char *s = \"say \\\"//\\\"\"; // gone\n")
    out = bench.code_only(src)
    assert '"tanh.approx.f32 %0, %1; // not a comment /* nor this */"' in out
    assert "'/'" in out and "'\\''" in out and '"say \\"//\\""' in out
    assert "gone" not in out


def _tree(base, files):
    for rel, text in files.items():
        p = os.path.join(base, rel)
        os.makedirs(os.path.dirname(p), exist_ok=True)
        with open(p, "w") as f:
            f.write(text)


def test_hash_follows_code_not_comments(bench, repo_tmp, monkeypatch):
    csrc = os.path.join("linear_attention_recurrence_05_b200", "csrc")
    files = {os.path.join(csrc, "k.cu"): "// kernel\n__global__ void k(float *p) { p[0] = 1.f; }\n",
             os.path.join(csrc, "k.h"): "#pragma once\nconstexpr int kN = 64;  // tile\n",
             os.path.join(csrc, "notes.txt"): "not a source\n",
             os.path.join("include", "api.h"): "int api(void);\n"}
    _tree(repo_tmp, files)
    monkeypatch.setattr(bench, "ROOT", repo_tmp)
    h0 = bench.kernel_sources_sha256()

    _tree(repo_tmp, {os.path.join(csrc, "k.h"): "#pragma once\n\n/* tile rows */\nconstexpr int kN = 64;  // rows\n",
                     os.path.join(csrc, "notes.txt"): "edited\n"})
    assert bench.kernel_sources_sha256() == h0

    _tree(repo_tmp, {os.path.join(csrc, "k.h"): "#pragma once\nconstexpr int kN = 128;  // tile\n"})
    assert bench.kernel_sources_sha256() != h0

    _tree(repo_tmp, {os.path.join(csrc, "k.h"): "#pragma once\nconstexpr int kN = 64;  // tile\n",
                     os.path.join("include", "api.h"): "int api(int);\n"})
    assert bench.kernel_sources_sha256() != h0


def test_traffic_lookup_scales_and_refuses_stale(bench, repo_tmp, monkeypatch):
    rec = {"kernel": "prefill_tc", "workload": "small", "applies_to": ["large"],
           "bytes_per_launch": 1000, "units_per_launch": 10, "unit": "tokens", "sources_sha256": "ab" * 32}
    _tree(repo_tmp, {os.path.join("profiles", "k.md"): "# k\n\ntraffic-record: " + json.dumps(rec) + "\n",
                     os.path.join("profiles", "raw.txt"): "traffic-record: {\"kernel\": \"x\"}\n"})
    monkeypatch.setattr(bench, "ROOT", repo_tmp)
    assert bench.traffic_for("prefill_tc", "small", 30, "ab" * 32) == (3000, "k.md")
    assert bench.traffic_for("prefill_tc", "large", 5, "ab" * 32) == (500, "k.md")
    val, why = bench.traffic_for("prefill_tc", "small", 30, "cd" * 32)
    assert val is None and why.startswith("stale")
    val, why = bench.traffic_for("chunk_prep", "small", 30, "ab" * 32)
    assert val is None and why == "no ncu record"


def test_committed_records_are_well_formed(bench):
    recs = bench.traffic_records()
    kernels = {k for k, _ in recs}
    assert {"prefill_tc", "chunk_prep", "conv_l2", "decode"} <= kernels
    for r in recs.values():
        assert r["bytes_per_launch"] > 0 and r["units_per_launch"] > 0
        assert len(r["sources_sha256"]) == 64 and int(r["sources_sha256"], 16) >= 0


# The chain kernel's MMAs per chunk of 64 tokens and V head (M = d_v = 128 on the tensor-memory
# lanes): shape (M, N, K) and operand kind, as the kernel issues them.
CHAIN_MMAS = {"MMA_1 S^T [K;Q]^T": (128, 128, 128, "tf32"), "MMA_2a V^T T_beta^T": (128, 64, 64, "f16"),
              "MMA_2b X T_beta_gamma^T": (128, 64, 64, "tf32"), "MMA_3 u~^T K": (128, 128, 64, "f16"),
              "MMA_4 u^T P^T": (128, 64, 64, "f16")}


def test_chain_flops_follow_the_mma_shapes(bench):
    per_tok = {kind: sum(2 * m * n * k for m, n, k, t in CHAIN_MMAS.values() if t == kind) / 64
               for kind in ("tf32", "f16")}
    assert bench.CHAIN_FLOP_TV_TF32 == per_tok["tf32"] == 81920
    assert bench.CHAIN_FLOP_TV_F16 == per_tok["f16"] == 65536
    assert bench.CHAIN_FLOP_TV == 147456


def test_chain_roofline_blends_the_peaks_by_time(bench):
    """A launch that ran every MMA at its own peak reports frac = 1."""
    peaks = {"bf16_tflops": 1654.0, "hbm_gbs": 6553.0}
    tf32 = 1654.0 * 1.1 / 2.25
    T, Hv, launches, steps = 2048, 48, 4, 10
    t_ideal = (bench.CHAIN_FLOP_TV_TF32 / (tf32 * 1e12) + bench.CHAIN_FLOP_TV_F16 / (1654.0 * 1e12)) * T * Hv
    res = {"per_kernel": {"prefill_tc": {"total_ms": t_ideal * 1e3 * launches * steps, "avg_ms": t_ideal * 1e3,
                                         "launches": launches * steps},
                          "chunk_prep": {"total_ms": 1e-3, "avg_ms": 1e-4, "launches": launches * steps}},
           "tokens_per_step": T * launches, "steps": steps, "n_v_heads": Hv, "n_qk_heads": 16,
           "workload": "none"}
    r = bench.prefill_roofline(res, peaks, "measured", "0" * 64)
    assert r["kernel"] == "prefill_tc" and r["tokens_per_launch"] == T
    assert abs(r["frac"] - 1.0) < 1e-12
    assert abs(r["peak"] - 1046.30) < 0.01
    assert abs(r["frac_of_bf16_peak"] - r["achieved"] / 1654.0) < 1e-12
    assert r["traffic"] is None


def test_step_work_per_token_matches_the_stated_counts(bench):
    """Per token at 16 QK / 48 V heads: 7.60 MFLOP with full 64-row tiles, 6.16 MFLOP counting
    only the needed triangles, and a minimum of 32,960 bytes (raw q, k, v, gates, bf16 y)."""
    T = 8192
    res = {"ms_per_step": 1.0, "tokens_per_step": T, "n_qk_heads": 16, "n_v_heads": 48}
    r = bench.prefill_step_summary(res, {"bf16_tflops": 1654.0, "hbm_gbs": 6553.0})
    assert round(r["algorithmic_flops_per_step"] / T) == 7602176
    assert round(r["algorithmic_flops_per_step_triangles_only"] / T) == 6160384
    assert r["algorithmic_bytes_per_step"] == 32960 * T
    assert abs(r["gbs"] - 32960 * T / 1e-3 / 1e9) < 1e-6
    assert abs(r["frac_of_bf16_peak"] - r["tflops"] / 1654.0) < 1e-12


def test_decode_bytes_per_row(bench):
    """State read and written once (6,291,456 B), conv state read and written, this step's raw
    q, k, v, the gates and y: 6,447,296 B with bf16 y (the minimum), 6,459,584 with fp32 y."""
    import gdn_inputs as gi
    assert bench.decode_bytes_per_row(gi.PAGES_SHAPE, out_bytes=2) == 6447296
    assert bench.decode_bytes_per_row(gi.PAGES_SHAPE) == 6459584


def test_reference_arm_line(repo_tmp):
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one JSON line with
    the headline config, and ranks other than 0 print nothing."""
    import subprocess
    import sys
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
           "--warmup", "3", "--ref-step-s", "0.5"]
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=repo_tmp, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    ln = lines[0]
    assert ln["impl"] == "reference" and ln["unit"] == "tokens/s" and ln["value"] > 0
    assert ln["higher_is_better"] is True and ln["n_gpus"] == 1 and ln["steps"] == 1
    assert ln["config"]["workload"] == "layer-bf16-T8192-h16x48" and ln["config"]["T"] == 8192
    assert ln["cpu_baseline"]["kind"] == "oracle" and ln["cpu_baseline"]["cores"] >= 1
    assert ln["e2e"] == {"value": ln["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    r1 = subprocess.run(cmd, capture_output=True, text=True, cwd=repo_tmp,
                        env=dict(os.environ, RANK="1", WORLD_SIZE="2"), timeout=600)
    assert r1.returncode == 0 and not r1.stdout.strip()
