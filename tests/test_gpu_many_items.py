"""A decode call over more sequences than one launch takes (1,100 > 512): the
library cuts it into launches of at most 512 items, each with its own slice of
q / out / new rows.  Parity against the oracle in every split mode, with and
without the fused append, and with forked pairs that form sibling sets in the
first launch ("kv-cache-pagedattention-serving", PagedAttention: virtual
memory for GPUs; The bonus: sharing via copy-on-write)."""
import dataclasses

import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa
from paged_harness import Pair
from workloads import Purpose, rng, workload

pytestmark = pytest.mark.gpu

N = 1100


def many():
    g = rng(0, 9, Purpose.LENS)
    lens = {}
    for s in range(N):
        if s < 200 and s % 2 == 1:
            continue                                   # forked from s - 1 below
        lens[s] = int(g.integers(40, 81)) if s < 200 else int(g.integers(1, 41))
    forks = tuple((s, s + 1) for s in range(0, 200, 2))
    w = workload("tiny")
    return dataclasses.replace(w, name="many_items", cfg=9, num_blocks=4 * N + 64, max_seqs=N,
                               max_blocks_per_seq=8, seq_ids=tuple(range(N)),
                               prefill_lens=lens, forks=forks, steps=2)


@pytest.mark.parametrize("partition", [0, -1, 32])
def test_more_items_than_one_launch(partition):
    w = many()
    p = Pair(w, min_partition=16)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    p.check_metadata()
    p.check_cache(0)
    before = pa.pa_launch_count(p.pool)
    q, out = p.decode(0, 0, seqs, partition)
    assert pa.pa_launch_count(p.pool) - before >= 3
    p.check_attention(0, seqs, q, out)
    if partition == 0:
        sets, _ = pa.pa_last_decode_plan(p.pool)
        assert sets >= 1
    # the next step's append fused into the same multi-launch call
    seqs, pos = p.reserve_step(1)
    q, out = p.append_decode(1, 0, seqs, pos, partition)
    p.check_cache(0)
    p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0
