"""The host block manager (free list, reference counts, copy-on-write,
prefix trie with its open-addressing index, cached list) under
AddressSanitizer and UBSan: a random-operation driver (tests/native/bm_fuzz.cpp)
built with g++ against the library's own block_manager.cpp checks the index
against std::multimap under crowded keys, then the pool invariants after every
operation, and every 250 operations the state image: restored into a fresh
manager it gives the same state; corrupted (random words, truncations) it
loads into a consistent state or changes nothing.  No GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "pagedattention_decode_03_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_block_manager_fuzz_under_sanitizers():
    out = os.path.join(ROOT, "_build")
    os.makedirs(out, exist_ok=True)
    exe = os.path.join(out, "bm_fuzz")
    subprocess.run(["g++", "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined",
                    "-fno-sanitize-recover=undefined", "-I", CSRC,
                    os.path.join(ROOT, "tests", "native", "bm_fuzz.cpp"),
                    os.path.join(CSRC, "block_manager.cpp"), "-o", exe],
                   check=True, capture_output=True, timeout=300)
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0")
    r = subprocess.run([exe, "24"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    assert r.stdout.strip() == "ok"
