"""Beam-search bookkeeping on the block manager, bit-exact against the oracle
(no GPU).  Each step keeps k beams: beams that no new beam descends from are
released, a beam with c children keeps its id for the first and is forked for
the others, then every beam grows by one token.  Forked beams share every
block by reference count and a fresh block is taken only when a beam writes
into a tail block it still shares ("Managing the KV Cache", Block Tables and
Sharing; kv-cache-pagedattention-serving, The bonus: sharing via
copy-on-write): with all beams of one length, a step with a partly filled tail
makes exactly k - (number of distinct parents) copies, a step whose tail is
full makes none.
"""
import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa
from oracle import Status

from test_host_prefix import Both


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


@pytest.mark.parametrize("width,B,prompt,seed", [(4, 16, 100, 0), (8, 16, 37, 1), (8, 32, 64, 2),
                                                  (3, 16, 16, 3)])
def test_beam_steps_match_oracle_and_copy_only_on_divergence(width, B, prompt, seed):
    g = np.random.default_rng([seed, 41])
    x = Both(nb=width * 40 + 64, B=B, max_seqs=2 * width + 1, mbps=64)
    assert x.reserve(0, prompt) == Status.OK
    beams = [0]
    for c in range(1, width):                                 # the first step: width samples
        assert x.fork(0, c) == Status.OK
        beams.append(c)
    length = prompt
    for step in range(60):
        cows_before = len(pa.pa_get_cow_log(x.p))
        parents = len({x.o.table(s)[-1] for s in beams})        # distinct tail blocks
        # grow every beam by one token, in id order
        for s in sorted(beams):
            assert x.reserve(s, length + 1) == Status.OK
        cows = len(pa.pa_get_cow_log(x.p)) - cows_before
        if length % B:
            assert cows == width - parents
        else:
            assert cows == 0
        assert pa.pa_get_cow_log(x.p) == x.o.cow_log
        length += 1
        x.same()
        # choose the next beams' parents; drop the rest, fork for extra children
        pick = sorted(int(i) for i in g.integers(0, width, width))
        kids = {b: pick.count(i) for i, b in enumerate(beams)}
        for b in beams:
            if kids[b] == 0:
                assert x.release(b) == Status.OK
        new = []
        spare = [s for s in range(2 * width + 1) if s not in beams]
        for b in beams:
            for c in range(kids[b]):
                if c == 0:
                    new.append(b)
                else:
                    child = spare.pop(0)
                    assert x.fork(b, child) == Status.OK
                    new.append(child)
        beams = new
        x.same()
    # every beam shares the prompt's full blocks
    full = prompt // B
    first = x.o.table(beams[0])[:full]
    assert all(x.o.table(s)[:full] == first for s in beams)
