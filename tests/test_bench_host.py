"""Host-side pieces of bench.py that need no GPU: the attachment of committed ncu traffic
figures to the kernel code they were taken on."""
from __future__ import annotations

import os
import re

import pytest

import bench

PROFILES = [f for f in sorted(os.listdir(os.path.join(bench.ROOT, "profiles"))) if f.endswith(".md")]


def test_comment_stripping_keeps_code_and_string_literals():
    src = 'int a = 1; // note\n/* block\n comment */ asm("x // not a comment");\n  int   b;'
    assert bench._strip_c_comments(src) == 'int a = 1; asm("x // not a comment"); int b;'


def test_code_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "linear_recurrent_lm_b200" / "csrc"
    csrc.mkdir(parents=True)
    for h in bench._KERNEL_HEADERS:
        (csrc / h).write_text("// header\nconstexpr int kN = 64;\n")
    k = csrc / "k.cu"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    k.write_text("// v1\n__global__ void f() { int x = 1; }\n")
    h1 = bench.kernel_code_sha256("linear_recurrent_lm_b200/csrc/k.cu")
    k.write_text("/* reworded comment */\n__global__ void f() {\n  int x = 1;\n}\n")
    assert bench.kernel_code_sha256("linear_recurrent_lm_b200/csrc/k.cu") == h1
    k.write_text("__global__ void f() { int x = 2; }\n")
    assert bench.kernel_code_sha256("linear_recurrent_lm_b200/csrc/k.cu") != h1
    (csrc / "tc05.cuh").write_text("constexpr int kN = 32;\n")   # a shared header counts too
    k.write_text("// v1\n__global__ void f() { int x = 1; }\n")
    assert bench.kernel_code_sha256("linear_recurrent_lm_b200/csrc/k.cu") != h1


@pytest.mark.parametrize("name", PROFILES)
def test_profile_headers_are_well_formed(name):
    text = open(os.path.join(bench.ROOT, "profiles", name)).read()
    if "source_file:" not in text:
        pytest.skip("launch list, not a single-kernel capture")
    assert re.search(r"code_sha256:\s*[0-9a-f]{64}", text)
    assert re.search(r"traffic_bytes_per_launch:\s*[0-9]+", text)
    assert "--clock-control none" in text            # every ncu command leaves the clocks alone


def test_dominant_kernel_profile_matches_current_code():
    """The roofline line's traffic comes from the committed capture of the backward kernel: that
    capture must have been taken on the kernel's current code (else bench.py reports null)."""
    t = bench.kernel_traffic("chunk_bwd", "packed_train_B8_T4096_H32")
    assert t is not None and 2.0e9 < t < 3.0e9
