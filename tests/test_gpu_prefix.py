"""GPU parity of decode over prefix-cached blocks.

Requests that start with a shared system prompt, multi-turn continuations of
finished conversations, decode steps (separate and fused append) and pool
pressure that evicts cached blocks, driven through the C ABI and the oracle
side by side.  Each position's K/V row is drawn from a generator seeded by the
whole token prefix ending there, so a reused block holds exactly the rows the
new request would have written ("kv-cache-pagedattention-serving", Beyond
paging: radix trees and continuous batching).  Compared after every call:
tables, reference counts, free and cached lists bit-exact, every valid cache
slot bit-exact, attention within 1e-2.
"""
import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle import Status
from paged_harness import Pair, to_dev
from workloads import Purpose, normal_bits, prefix_kv_bits, rng, workload

pytestmark = pytest.mark.gpu


class Run:
    def __init__(self, nb, seed=0, max_seqs=16, mbps=64):
        w = workload("tiny", seed=seed)
        self.w = dataclasses.replace(w, name="prefix", num_blocks=nb, max_seqs=max_seqs,
                                     max_blocks_per_seq=mbps)
        self.P = Pair(self.w, min_partition=16)
        self.hist = {}
        self.done = []
        self.calls = 0

    def check(self):
        P = self.P
        P.check_metadata()
        assert pa.pa_get_cached_blocks(P.pool) == P.oracle.cached_list()
        P.oracle.check_invariants()
        P.check_cache(0)

    def request(self, s, toks):
        """Reserve, write the uncached rows, register; None if the pool is full
        (the library and the oracle must agree on that)."""
        P, n = self.P, len(toks)
        want = P.oracle.reserve_prefix(s, toks)
        try:
            c = pa.pa_alloc_blocks_prefix(P.pool, s, toks)
        except pa.PAError as e:
            assert e.status == pa.PA_ERR_NO_BLOCKS and want == (Status.NO_BLOCKS, 0)
            return None
        assert want == (Status.OK, c)
        if n > c:
            k, v = prefix_kv_bits(self.w, 0, toks, c, n)
            P.append(0, [s] * (n - c), list(range(c, n)), k, v)
        pa.pa_prefix_register(P.pool, s, toks)
        assert P.oracle.register(s, toks) == Status.OK
        self.hist[s] = list(toks)
        return c

    def step(self, seqs, fused, partition_tokens=0, vocab=50000):
        P, w = self.P, self.w
        g = rng(w.seed, 77, Purpose.MISC, self.calls)
        self.calls += 1
        new = [len(self.hist[s]) + 1 for s in seqs]
        pa.pa_alloc_blocks_n(P.pool, seqs, new)
        for s, n in zip(seqs, new):
            assert P.oracle.reserve(s, n) == Status.OK
            self.hist[s].append(int(g.integers(0, vocab)))
        rows = [prefix_kv_bits(w, 0, self.hist[s], len(self.hist[s]) - 1, len(self.hist[s]))
                for s in seqs]
        k = np.concatenate([r[0] for r in rows])
        v = np.concatenate([r[1] for r in rows])
        pos = [len(self.hist[s]) - 1 for s in seqs]
        q_bits = normal_bits(g, (len(seqs), w.num_q_heads, w.head_dim), w.act_dtype)
        q = to_dev(q_bits, w.act_dtype)
        out = torch.empty_like(q)
        if fused:
            pa.pa_decode_attention_append(P.pool, 0, seqs, to_dev(k, w.act_dtype),
                                          to_dev(v, w.act_dtype), q, out, w.scale, partition_tokens)
            P.append(0, seqs, pos, k, v, gpu=False)
        else:
            P.append(0, seqs, pos, k, v)
            pa.pa_decode_attention(P.pool, 0, seqs, q, out, w.scale, partition_tokens)
        torch.cuda.synchronize()
        P.check_attention(0, seqs, q_bits, out)
        assert P.device_errors() == 0

    def finish(self, s):
        pa.pa_free(self.P.pool, s)
        assert self.P.oracle.release(s) == Status.OK
        self.done.append(self.hist.pop(s))


def test_shared_system_prompt_is_read_from_one_copy():
    r = Run(nb=200)
    g = np.random.default_rng(4)
    system = list(g.integers(0, 50000, 300))                        # 18 full blocks + 12
    cached = [r.request(s, system + list(g.integers(0, 50000, int(g.integers(10, 80)))))
              for s in range(6)]
    assert cached == [0] + [288] * 5
    r.check()
    seqs = list(range(6))
    r.step(seqs, fused=False)
    sets, _ = pa.pa_last_decode_plan(r.P.pool)
    assert sets >= 1                     # forks of the cached prompt form sibling sets
    r.step(seqs, fused=True)
    r.step(seqs, fused=False, partition_tokens=-1)
    r.step(seqs, fused=False, partition_tokens=64)
    r.check()


@pytest.mark.parametrize("seed", range(3))
def test_conversations_with_eviction(seed):
    """A 48-block pool (768 slots) under requests, continuations, decode steps
    and releases; cached blocks are evicted and rewritten along the way."""
    r = Run(nb=48, seed=seed)
    g = np.random.default_rng([seed, 5])
    systems = [list(g.integers(0, 50000, int(g.integers(40, 200)))) for _ in range(3)]
    free_ids = list(range(16))
    evicted = hits = 0
    for it in range(40):
        op = g.random()
        if op < 0.35 and free_ids:
            base = (r.done[int(g.integers(len(r.done)))] if r.done and g.random() < 0.5
                    else systems[int(g.integers(len(systems)))])
            toks = base + list(g.integers(0, 50000, int(g.integers(1, 60))))
            if len(toks) > 64 * 16 - 40:
                continue
            free_before = len(pa.pa_get_free_list(r.P.pool))
            c = r.request(free_ids[0], toks)
            if c is None:
                continue
            free_ids.pop(0)
            hits += c > 0
            evicted += max(0, -(-len(toks) // 16) - c // 16 - free_before)
        elif op < 0.8 and r.hist:
            seqs = sorted(r.hist)
            room = len(pa.pa_get_free_list(r.P.pool)) + len(pa.pa_get_cached_blocks(r.P.pool))
            if room < len(seqs):
                s = seqs[int(g.integers(len(seqs)))]
                r.finish(s)
                free_ids.append(s)
                continue
            r.step(seqs, fused=bool(it % 2))
        elif r.hist:
            s = sorted(r.hist)[int(g.integers(len(r.hist)))]
            r.finish(s)
            free_ids.append(s)
        r.check()
    assert evicted > 0 and hits > 0


def test_registered_blocks_refuse_writes():
    r = Run(nb=40)
    toks = list(range(1000, 1032))                                   # exactly two blocks
    r.request(0, toks)
    P, w = r.P, r.w
    before = pa.pa_launch_count(P.pool)
    k, v = prefix_kv_bits(w, 0, toks, 5, 6)
    with pytest.raises(pa.PAError) as e:
        pa.pa_append_kv(P.pool, 0, [0], [5], to_dev(k, w.act_dtype), to_dev(v, w.act_dtype))
    assert e.value.status == pa.PA_ERR_SHARED_BLOCK
    # the fused call writes slot len - 1, which is in the registered block 1
    q = to_dev(normal_bits(np.random.default_rng(0), (1, 8, 128), "bf16"), "bf16")
    out = torch.empty_like(q)
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_attention_append(P.pool, 0, [0], to_dev(k, w.act_dtype),
                                      to_dev(v, w.act_dtype), q, out, w.scale, 0)
    assert e.value.status == pa.PA_ERR_SHARED_BLOCK
    assert pa.pa_launch_count(P.pool) == before
    r.step([0], fused=True)                                          # the next token: a new block
    r.check()
