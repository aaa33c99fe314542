"""CPU check of the backward's work items and dQ ordering.

Compiles tests/native/bwd_schedule_check.cu, which includes the kernel header
and calls its own decode_item / BwdItem on the host (nothing is launched), and
runs it over a range of tile counts, head counts and both masks. It checks that
every (key tile, query tile) pair is visited once, that each dQ sum's
contributors form one fixed order starting at position 0, and that each
contributor's predecessor is fetched earlier and visits the tile one step
(non-causal) or two steps (causal) earlier (no deadlock; no waiting between
items that start together).
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "native", "bwd_schedule_check.cu")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("sched") / "bwd_schedule_check")
    cmd = [nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "--expt-relaxed-constexpr",
           "-o", exe, SRC]
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=os.path.dirname(SRC))
    assert r.returncode == 0, r.stderr[-2000:]
    return exe


@pytest.mark.parametrize("causal", [0, 1])
def test_items_cover_pairs_once_and_dq_order_is_acyclic(checker, causal):
    args = []
    for ntiles in list(range(1, 41)) + [64, 128, 256]:
        for heads in (1, 3, 8, 13, 20):
            for group in ((1, 2, 8, 16) if causal else (1,)):
                args += [str(ntiles), str(heads), str(causal), str(group)]
    r = subprocess.run([checker] + args, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:]
    assert r.stdout.strip().startswith("OK")
