"""PA_LOG=2 on a device pool: one stderr line per decode call naming the
kernel, the split mode and whether the plan was reused.  The child process
runs a tiny pool (prefill, one step, decodes in three split modes, the same
call twice) and its stderr is read here."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
sys.path.insert(0, "tests")
from paged_harness import Pair
from workloads import workload
w = workload("tiny")
p = Pair(w, oracle_seqs=[])
p.prefill()
seqs, pos = p.reserve_step(0)
p.append_step(0, 0, seqs, pos)
for part in (0, 0, -1, 512):
    p.decode(0, 0, seqs, part)
print("done")
"""


def test_decode_calls_are_logged():
    env = dict(os.environ, PA_LOG="2")
    r = subprocess.run([sys.executable, "-c", SCRIPT], capture_output=True, text=True, env=env,
                       cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    dec = [ln for ln in r.stderr.splitlines() if ln.startswith("[pa] decode: layer 0, 4 sequences, G=4")]
    assert len(dec) == 4, r.stderr[-3000:]
    assert "warp-level kernel, stream-K split" in dec[0] and "plan built" in dec[0]
    assert "plan reused" in dec[1]                       # same call, same tables
    assert "no split" in dec[2] and "fixed split" in dec[3]
    assert any(ln.startswith("[pa] pool_create: device buffers") for ln in r.stderr.splitlines())
    assert any(ln.startswith("[pa] append_kv: layer 0, 4 rows") for ln in r.stderr.splitlines())
