"""Host-only checks of the tensor-core launch plans (tests/plan_check.cu): compiled with
nvcc and run on the CPU, no GPU needed."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_launch_plans_cover_k_fit_budgets_and_scratch():
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "plan_check")
        cmd = [nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
               "-I", os.path.join(ROOT, "transformer_decoder_kv_b200", "csrc"), "-I", os.path.join(ROOT, "include"),
               os.path.join(HERE, "plan_check.cu"), "-o", exe]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr[-3000:]
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-3000:]
    # the benchmark times the attention in the first chain's launch shape: its copy of the
    # chain rule must agree with the library's
    import bench
    chains = [tuple(int(v) for v in ln.split()[1:]) for ln in r.stdout.splitlines() if ln.startswith("chain ")]
    assert len(chains) > 100
    for B, n, first in chains:
        if B >= bench.SPLIT_MIN_BATCH:
            assert bench.chain_rows(B) == (n, first), (B, n, first, bench.chain_rows(B))
