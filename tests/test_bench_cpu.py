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
