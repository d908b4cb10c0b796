"""Host check of the decode's share split (csrc/pa_split.cuh): compiled with
the host C++ compiler and brute-forced over random lines, grids, early-CTA
counts and extras (tests/split_check.cpp states the invariants)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "paged_kv_attention_36_b200", "csrc")


def test_share_split_tiles_the_line_and_owner_inverts_start(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path / "split_check")
    subprocess.run([cxx, "-std=c++17", "-O2", "-Wall", "-I", CSRC, os.path.join(HERE, "split_check.cpp"), "-o", exe],
                   check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
