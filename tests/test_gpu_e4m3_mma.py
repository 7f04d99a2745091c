"""The tcgen05 e4m3 MMA properties the e4m3 decode kernel relies on (B200):
its operand layouts give the right products and e4m3 products accumulate to
fp32 precision.  The probe program (tests/probes/e4m3_mma_probe.cu) is
compiled here and prints, per input set, the largest error against the exact
sum in fp32 ulps of sum |a b|."""
import json
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_e4m3_mma_layouts_and_fp32_accumulation(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "e4m3_mma_probe")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                    os.path.join(HERE, "probes", "e4m3_mma_probe.cu"), "-o", exe], check=True, timeout=300)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    sets = [json.loads(line) for line in r.stdout.splitlines() if line.startswith("{")]
    assert len(sets) == 3
    for s in sets:
        # a wrong layout gives errors of the order of the sums themselves (2^23 ulps)
        assert s["kmajor_ulps"] < 4 and s["mnmajor_ulps"] < 4, s
    assert sets[1]["kmajor_exact"] == 2048 and sets[1]["mnmajor_exact"] == 2048  # codes in [0.5, 4): exact sums
