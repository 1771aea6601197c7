"""Randomised GPU parity sweep: shapes, query groups, KV dtypes, lengths, forks
and split modes drawn from a seeded generator, every decode output compared
with the oracle (same tolerances as the other decode tests).

The fixed tests pin the workloads of the pages; this sweep covers the cases in
between: odd head counts, one-token and block-aligned lengths, sibling sets of
every size, sequences named twice in one call, and split shares that begin or
end anywhere inside a sequence.
"""
import numpy as np
import pytest
import torch

from paged_harness import Pair
from workloads import Workload, normal_bits, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()
    assert torch.cuda.is_available()


def random_workload(seed):
    g = np.random.default_rng([seed, 41])
    G = int(g.choice([1, 2, 4, 8]))
    H = int(g.choice([1, 2, 3, 4, 8]))
    kv = str(g.choice(["bf16", "fp16", "fp8_e4m3"]))
    act = "fp16" if kv == "fp16" else "bf16"
    prefill, forks, sid = {}, [], 0
    for _ in range(int(g.integers(1, 5))):            # prompt families
        members = int(g.integers(1, 10))
        prefill[sid] = int(g.choice([int(g.integers(1, 40)), int(g.integers(16, 700)),
                                     16 * int(g.integers(1, 30))]))
        forks += [(sid, sid + c) for c in range(1, members)]
        sid += members
    for _ in range(int(g.integers(0, 6))):            # unrelated sequences
        prefill[sid] = int(g.integers(1, 900))
        sid += 1
    steps = int(g.integers(1, 4))
    lens = dict(prefill)
    for parent, child in forks:
        lens[child] = lens[parent]
    need = sum(-(-(n + steps) // 16) for n in lens.values())
    mbps = max(-(-(n + steps) // 16) for n in lens.values()) + 1
    w = Workload(
        name="random", cfg=7, num_layers=1, num_q_heads=H * G, num_kv_heads=H, head_dim=128,
        block_size=16, act_dtype=act, kv_dtype=kv, num_blocks=need + int(g.integers(0, 40)),
        max_seqs=sid, max_blocks_per_seq=mbps, seq_ids=tuple(range(sid)), prefill_lens=prefill,
        forks=tuple(forks), steps=steps, seed=seed)
    return w, g


@pytest.mark.parametrize("seed", range(24))
def test_random_workload_matches_oracle(seed):
    w, g = random_workload(seed)
    p = Pair(w, min_partition=16)
    p.prefill()
    parts = [0, -1, 16 * int(g.integers(1, 6))]
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        p.append_step(step, 0, seqs, pos)
        for part in parts:
            q, out = p.decode(step, 0, seqs, part)
            p.check_attention(0, seqs, q, out)
    # one more call over a shuffled subset that names a sequence twice
    ids = list(w.seq_ids)
    sub = [int(x) for x in g.permutation(ids)[: max(1, len(ids) // 2)]] + [ids[0]]
    q_bits = normal_bits(rng(w.seed, w.cfg, 7, 1), (len(sub), w.num_q_heads, w.head_dim), w.act_dtype)
    for part in parts:
        _, out = p.decode(0, 0, sub, part, q_bits=q_bits)
        p.check_attention(0, sub, q_bits, out)
    p.check_metadata()
    p.check_cache(0)
    assert p.device_errors() == 0
