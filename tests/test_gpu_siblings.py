"""GPU parity of decode over forked sequences, where the library reads a
shared prompt prefix once for a whole sibling set (partition_tokens = 0).

Sequences forked from one prompt hold the prompt's physical blocks by
reference count ("Managing the KV Cache", Block Tables and Sharing;
"kv-cache-pagedattention-serving", The bonus: sharing via copy-on-write).
The attention each sequence sees is still plain softmax attention over its
own tokens, so every output is checked against the oracle, in all three
partition modes, with the same tolerances as every other decode test.
"""
import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle import Status
from paged_harness import Pair
from workloads import Workload, normal_bits, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()
    assert torch.cuda.is_available()


def family_workload(G, kv, families, extra_lens, steps, H=2, seed=5):
    """`families` = [(prompt tokens, members)]: member 0 is prefilled, the
    others are forked from it; `extra_lens` are unrelated sequences."""
    act = "fp16" if kv == "fp16" else "bf16"
    prefill, forks, sid = {}, [], 0
    for plen, members in families:
        prefill[sid] = plen
        forks += [(sid, sid + c) for c in range(1, members)]
        sid += members
    for n in extra_lens:
        prefill[sid] = n
        sid += 1
    lens = {s: prefill[s] for s in prefill}
    for parent, child in forks:
        lens[child] = lens[parent]
    need = sum(-(-(n + steps) // 16) for n in lens.values())
    mbps = max(-(-(n + steps) // 16) for n in lens.values()) + 1
    return Workload(
        name="siblings", cfg=6, num_layers=1, num_q_heads=H * G, num_kv_heads=H, head_dim=128,
        block_size=16, act_dtype=act, kv_dtype=kv, num_blocks=need + 32, max_seqs=sid,
        max_blocks_per_seq=mbps, seq_ids=tuple(range(sid)), prefill_lens=prefill,
        forks=tuple(forks), steps=steps, seed=seed)


def distinct_tiles(p, seqs):
    """(block, KV head) tiles a call over `seqs` must read at least once."""
    blocks = set()
    for s in seqs:
        n = p.oracle.lens[s]
        blocks.update(p.oracle.table(s)[: -(-n // 16)])
    return len(blocks) * p.w.num_kv_heads


def run_steps(p, w, check_sets):
    seqs = list(w.seq_ids)
    # right after the forks: members share every block, the partial tail too
    q, out = p.decode(0, 0, seqs, 0)
    p.check_attention(0, seqs, q, out)
    if check_sets:
        assert pa.pa_last_decode_plan(p.pool)[0] > 0
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        p.append_step(step, 0, seqs, pos)
        for part in (0, -1, 16):
            q, out = p.decode(step, 0, seqs, part)
            p.check_attention(0, seqs, q, out)
            sets, tiles = pa.pa_last_decode_plan(p.pool)
            if part == 0 and check_sets:
                assert sets > 0
                assert tiles < sum(-(-p.oracle.lens[s] // 16) for s in seqs) * w.num_kv_heads
                assert tiles >= distinct_tiles(p, seqs)
            if part != 0:
                assert sets == 0
    p.check_metadata()
    assert p.device_errors() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp16", "fp8_e4m3"])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_sibling_sets_match_oracle(G, kv):
    """Families larger than one set (8 / G members) split into several sets;
    prompt lengths put the shared run at 3 .. 40 blocks with ragged tails."""
    members = 8 // G + 3
    w = family_workload(G, kv, [(643, members), (50, 3), (200, 2)], [333, 50], steps=3)
    p = Pair(w, min_partition=16)
    p.prefill()
    run_steps(p, w, check_sets=True)


def test_sibling_tree_forks_at_different_depths():
    """Beam-search-like tree: forks of forks after private growth, so sets
    share prefixes of different lengths and some members only a short run."""
    w = family_workload(1, "bf16", [(420, 4)], [], steps=1, H=4, seed=9)
    w = Workload(**{**w.__dict__, "max_seqs": 10, "seq_ids": tuple(range(10)),
                    "num_blocks": w.num_blocks + 200, "max_blocks_per_seq": 64})
    p = Pair(w, min_partition=16)
    p.prefill()
    g = rng(w.seed, w.cfg, 7)

    def grow(active, steps):
        for _ in range(steps):
            lens = {s: p.oracle.lens[s] for s in active}
            pa.pa_alloc_blocks_n(p.pool, active, [lens[s] + 1 for s in active])
            for s in active:
                assert p.oracle.reserve(s, lens[s] + 1) is Status.OK
            k = normal_bits(g, (len(active), w.num_kv_heads, w.head_dim), w.act_dtype)
            v = normal_bits(g, (len(active), w.num_kv_heads, w.head_dim), w.act_dtype)
            p.append(0, active, [lens[s] for s in active], k, v)

    def check(active):
        """Sibling sets of the partition_tokens = 0 call."""
        q_bits = normal_bits(g, (len(active), w.num_q_heads, w.head_dim), w.act_dtype)
        sets = None
        for part in (0, -1):
            _, out = p.decode(0, 0, active, part, q_bits=q_bits)
            p.check_attention(0, active, q_bits, out)
            if part == 0:
                sets = pa.pa_last_decode_plan(p.pool)[0]
        return sets

    grow([0, 1, 2, 3], 37)            # private runs of 37 tokens after the prompt
    for parent, child in [(0, 4), (0, 5), (1, 6), (2, 7), (2, 8), (2, 9)]:
        pa.pa_fork_cow(p.pool, parent, child)
        assert p.oracle.fork(parent, child) is Status.OK
    active = list(range(10))
    assert check(active) > 0
    grow(active, 21)
    assert check(active) > 0
    check([9, 3, 6, 0])               # a subset, in another order
    p.check_metadata()
    assert p.device_errors() == 0


def test_short_common_prefix_is_not_grouped():
    """Two sequences that share only their first block (a one-block prompt)
    are decoded per sequence; results still match."""
    w = family_workload(1, "bf16", [(20, 2)], [300], steps=20)
    p = Pair(w, min_partition=16)
    p.prefill()
    seqs = list(w.seq_ids)
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        p.append_step(step, 0, seqs, pos)
    q, out = p.decode(w.steps, 0, seqs, 0)
    p.check_attention(0, seqs, q, out)
    assert pa.pa_last_decode_plan(p.pool)[0] == 0
    assert p.device_errors() == 0


def test_many_sets_and_wide_heads():
    """96 two-member families with G = 4 over 16 KV heads (64 query heads): many
    shared entries in one launch, each cut across workers."""
    w = family_workload(4, "bf16", [(16 * (3 + i % 29) + i % 16, 2) for i in range(96)], [],
                        steps=1, H=16, seed=11)
    p = Pair(w, min_partition=16)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    q, out = p.decode(0, 0, seqs, 0)
    p.check_attention(0, seqs, q, out)
    sets, tiles = pa.pa_last_decode_plan(p.pool)
    assert sets == 96
    assert tiles == distinct_tiles(p, seqs)  # every shared full block read once
    assert p.device_errors() == 0
