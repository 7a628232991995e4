"""The decode work split and the merge's view of it, checked on the host: the split helpers of
kvk_internal.cuh are compiled into a small host program (tests/split_check.cpp) that compares
them with brute-force ownership on random batches (every token owned once, contiguous CTA
ranges, merge pieces = the CTAs that own a sequence's tokens, empty CTAs skipped)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include():
    for base in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if base and os.path.isdir(os.path.join(base, "include")):
            return os.path.join(base, "include")
    return None


def test_work_split_matches_brute_force(tmp_path):
    cxx = shutil.which("g++")
    inc = _cuda_include()
    if not cxx or not inc:
        pytest.skip("needs g++ and the CUDA headers")
    exe = tmp_path / "split_check"
    subprocess.run([cxx, "-std=c++17", "-O2", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "compressed_decode_attention_kvk_b200", "csrc"),
                    "-I", inc, os.path.join(ROOT, "tests", "split_check.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
    assert int(r.stdout.split()[1]) > 100000
