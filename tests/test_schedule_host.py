"""The device work split (paged_kv_cache_367_b200/csrc/schedule.cuh), compiled
for the host: every token of every unit is covered exactly once."""
import os
import shutil
import subprocess

import pytest

from conftest import ROOT

NVCC = "/usr/local/cuda/bin/nvcc"


@pytest.mark.skipif(not os.path.exists(NVCC) and not shutil.which("nvcc"), reason="needs nvcc")
def test_work_split_covers_every_token_once(tmp_path):
    exe = tmp_path / "schedule_check"
    subprocess.check_call([NVCC if os.path.exists(NVCC) else "nvcc", "-std=c++17", "-O1",
                           "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(ROOT, "paged_kv_cache_367_b200", "csrc"),
                           os.path.join(ROOT, "tests", "schedule_check.cu"), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("OK")
