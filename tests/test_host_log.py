"""The library's stderr log (PA_LOG) and its optional NVTX ranges.

PA_LOG is read once per process, so each case runs a short host-only script
(block-manager calls only, no GPU) in a child process and reads its stderr.
The NVTX build is checked by compiling every source with PA_NVTX defined.
"""
import os
import shutil
import subprocess
import sys

import pytest

from pagedattention_decode_03_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import pagedattention_decode_03_b200 as pa
p = pa.pa_pool_create(num_layers=1, num_kv_heads=1, block_size=16, num_blocks=4,
                      max_seqs=4, max_blocks_per_seq=8, host_only=True)
pa.pa_alloc_blocks(p, 0, 20)
pa.pa_fork_cow(p, 0, 1)
try:
    pa.pa_alloc_blocks(p, 2, 100)     # 7 blocks from a pool of 4: refused
except pa.PAError:
    pass
pa.pa_free(p, 1)
print("done")
"""


@pytest.fixture(scope="module", autouse=True)
def built():
    pa_build.build()


def run_with(level):
    env = dict(os.environ)
    env.pop("PA_LOG", None)
    if level is not None:
        env["PA_LOG"] = level
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", SCRIPT], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().endswith("done")
    return [ln for ln in r.stderr.splitlines() if ln.startswith("[pa] ")]


@pytest.mark.parametrize("level", [None, "0", "abc"])
def test_log_off_by_default(level):
    assert run_with(level) == []


def test_log_level_1_reports_errors_only():
    lines = run_with("1")
    assert len(lines) == 1
    assert lines[0].startswith("[pa] PA_ERR_NO_BLOCKS: pa_alloc_blocks: free list too short")


def test_log_level_2_reports_calls():
    lines = run_with("2")
    text = "\n".join(lines)
    assert lines[0].startswith("[pa] pool_create: host only, 1 layers, 4 blocks of 16 tokens")
    assert "[pa] alloc_blocks: 1 of 1 sequences reserved, 0 block copies" in text
    assert "[pa] fork_cow: sequence 0 -> 1" in text
    assert "[pa] PA_ERR_NO_BLOCKS: pa_alloc_blocks: free list too short" in text
    assert "[pa] alloc_blocks: 0 of 1 sequences reserved" in text
    assert "[pa] free: sequence 1" in text
    # levels above 2 read as 2
    assert run_with("7") == lines


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
@pytest.mark.parametrize("src", ["api.cpp", "noalloc.cu"])
def test_nvtx_build_compiles(src, tmp_path):
    """Every C-ABI entry point opens a range when built with PA_NVTX; the
    sources that hold entry points compile that way."""
    cmd = [pa_build._nvcc(), *pa_build.ARCH, *pa_build.COMMON, *pa_build._defines(True),
           "-c", os.path.join(pa_build.CSRC, src), "-o", str(tmp_path / (src + ".o"))]
    if src.endswith(".cpp"):
        cmd[1:1] = ["-x", "cu"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    with open(os.path.join(pa_build.CSRC, src)) as f:
        text = f.read()
    assert text.count("PA_RANGE();") >= (20 if src == "api.cpp" else 2)
