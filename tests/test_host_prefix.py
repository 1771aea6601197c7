"""The library's block-granular prefix cache against the oracle, bit-exact:
tables, reference counts, free list, cached (least-recently-used) list,
statuses and reused-token counts after every operation.  Host-only pools; no
GPU ("kv-cache-pagedattention-serving", Beyond paging: radix trees and
continuous batching; "Managing the KV Cache", Block Tables and Sharing).
"""
import json
import os

import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa
from oracle import PagedKVOracle, Status

from test_host_library import STATUS, status_of

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "prefix_granularity.json")


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


class Both:
    """One host-only library pool and one oracle pool, driven in lockstep."""

    def __init__(self, nb, B, max_seqs=24, mbps=64, order=None):
        self.p = pa.pa_pool_create(num_layers=1, num_kv_heads=1, block_size=B, num_blocks=nb,
                                   max_seqs=max_seqs, max_blocks_per_seq=mbps, host_only=True,
                                   free_order=order)
        self.o = PagedKVOracle(num_layers=1, num_kv_heads=1, head_dim=1, block_size=B,
                               num_blocks=nb, max_seqs=max_seqs, max_blocks_per_seq=mbps,
                               kv_dtype="bf16", free_order=order, stored_layers=[])

    def same(self):
        p, o = self.p, self.o
        assert pa.pa_get_free_list(p) == o.free_list()
        assert pa.pa_get_cached_blocks(p) == o.cached_list()
        assert pa.pa_get_refcounts(p) == o.refcounts()
        for s in range(p.max_seqs):
            if s in o.tables:
                n, tab = pa.pa_get_seq(p, s)
                assert n == o.lens[s] and tab == o.table(s), s
            else:
                assert status_of(pa.pa_get_seq, p, s) == Status.NO_SEQ
        o.check_invariants()

    def reserve_prefix(self, s, toks):
        want = self.o.reserve_prefix(s, toks)
        try:
            got = (Status.OK, pa.pa_alloc_blocks_prefix(self.p, s, toks))
        except pa.PAError as e:
            got = (STATUS[e.status], 0)
        assert got == want
        return want

    def register(self, s, toks):
        want = self.o.register(s, toks)
        assert status_of(pa.pa_prefix_register, self.p, s, toks) == want
        return want

    def reserve(self, s, n):
        want = self.o.reserve(s, n)
        assert status_of(pa.pa_alloc_blocks, self.p, s, n) == want
        return want

    def fork(self, a, b):
        want = self.o.fork(a, b)
        assert status_of(pa.pa_fork_cow, self.p, a, b) == want
        return want

    def release(self, s):
        want = self.o.release(s)
        assert status_of(pa.pa_free, self.p, s) == want
        return want

    def match(self, toks):
        m = self.o.match(toks) * self.o.B
        assert pa.pa_prefix_match(self.p, toks) == m
        return m


def test_worked_103_token_prompt_reuses_96():
    g = json.load(open(GOLDEN))["worked_103"]
    x = Both(64, g["block_size"])
    toks = list(np.random.default_rng(1).integers(0, 50000, g["prompt_tokens"]))
    assert x.reserve_prefix(0, toks) == (Status.OK, 0)
    assert x.register(0, toks) == Status.OK
    assert x.match(toks) == g["reused_tokens"]
    assert x.reserve_prefix(1, toks) == (Status.OK, g["reused_tokens"])
    assert g["prompt_tokens"] - g["reused_tokens"] == g["recomputed_tokens"]
    x.same()


def test_lru_trace_by_hand():
    """The oracle's hand trace at B = 16: six blocks, free list 0..5."""
    x = Both(6, 16)
    a = list(range(1, 49))                                           # 3 blocks
    x.reserve_prefix(0, a)
    x.register(0, a)
    x.release(0)
    assert pa.pa_get_cached_blocks(x.p) == [2, 1, 0]
    x.reserve(1, 32)
    assert x.reserve_prefix(2, a[:32] + [99, 98]) == (Status.OK, 32)
    x.reserve(3, 16)                                                 # evicts block 2
    assert pa.pa_get_seq(x.p, 3)[1] == [2] and x.match(a) == 32
    x.release(2)
    x.reserve(4, 32)                                                 # free 5, then evicts 1
    assert pa.pa_get_seq(x.p, 4)[1] == [5, 1] and x.match(a) == 16
    x.same()


def test_failures_change_nothing():
    x = Both(3, 16)
    a = list(range(48))
    x.reserve_prefix(0, a)
    x.register(0, a)
    x.release(0)
    assert x.reserve_prefix(1, a + [7]) == (Status.NO_BLOCKS, 0)     # every idle block reused, +1
    x.same()
    assert x.reserve_prefix(1, a) == (Status.OK, 48)
    assert x.reserve_prefix(1, a) == (Status.SEQ_EXISTS, 0)
    assert x.register(1, a + [3]) == Status.INVALID_ARG              # longer than the sequence
    x.same()
    # a block registered under one prefix cannot be registered under another
    y = Both(16, 16)
    b = list(range(100, 132))
    y.reserve_prefix(0, b)
    y.register(0, b[:16])
    assert y.register(0, list(range(16)) + b[16:]) == Status.INVALID_ARG
    assert y.match(b) == 16                                          # nothing more was registered
    y.same()
    with pytest.raises(pa.PAError) as e:
        pa.pa_alloc_blocks_prefix(y.p, 99, b)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PAError) as e:
        pa.pa_prefix_register(y.p, 5, b)
    assert e.value.status == pa.PA_ERR_NO_SEQ


def test_injected_failure_applies_to_prefix_reservations():
    x = Both(32, 16)
    a = list(range(80))
    x.reserve_prefix(0, a)
    x.register(0, a)
    pa.pa_debug_fail_after(x.p, 1)
    with pytest.raises(pa.PAError) as e:
        pa.pa_alloc_blocks_prefix(x.p, 1, list(range(120)))         # 5 cached blocks + 3 new
    assert e.value.status == pa.PA_ERR_NO_BLOCKS
    assert pa.pa_alloc_blocks_prefix(x.p, 1, a + [1, 2]) == 80       # one new block: allowed
    x.o.reserve_prefix(1, a + [1, 2])
    x.same()


def drive(seed, nb, B, vocab, steps, order=None):
    rng = np.random.default_rng([seed, 29])
    x = Both(nb, B, order=order)
    systems = [list(rng.integers(0, vocab, int(rng.integers(B, 6 * B)))) for _ in range(4)]
    hist, done, free_ids = {}, [], list(range(24))
    for _ in range(steps):
        op = rng.random()
        if op < 0.3 and free_ids:
            base = (done[int(rng.integers(len(done)))] if done and rng.random() < 0.5
                    else systems[int(rng.integers(len(systems)))])
            toks = base + list(rng.integers(0, vocab, int(rng.integers(0, 3 * B))))
            s = free_ids.pop(0)
            x.match(toks)
            st, _ = x.reserve_prefix(s, toks)
            if st != Status.OK:
                free_ids.insert(0, s)
                continue
            hist[s] = toks
            x.register(s, toks[: int(rng.integers(0, len(toks) + 1))])
        elif op < 0.4 and hist and free_ids:
            parent = list(hist)[int(rng.integers(len(hist)))]
            s = free_ids.pop(0)
            x.fork(parent, s)
            hist[s] = list(hist[parent])
        elif op < 0.8 and hist:
            s = list(hist)[int(rng.integers(len(hist)))]
            grow = int(rng.integers(1, 2 * B))
            if x.reserve(s, len(hist[s]) + grow) != Status.OK:
                continue
            hist[s] += list(rng.integers(0, vocab, grow))
            if rng.random() < 0.4:
                x.register(s, hist[s])
        elif hist:
            s = list(hist)[int(rng.integers(len(hist)))]
            x.release(s)
            done.append(hist.pop(s))
            free_ids.append(s)
        x.same()
    return x


@pytest.mark.parametrize("seed", range(8))
def test_random_conversations_match_oracle(seed):
    nb = [30, 60, 400][seed % 3]
    order = np.random.default_rng(seed).permutation(nb).tolist()
    x = drive(seed, nb, B=[16, 32][seed % 2], vocab=[2, 3, 50000][seed % 3], steps=250, order=order)
    assert x.o.registry or seed % 3 == 2


def test_long_prompts_many_sequences():
    """A 2,048-token system prompt shared by many requests, at B = 16."""
    rng = np.random.default_rng(5)
    x = Both(4000, 16, max_seqs=64, mbps=256)
    system = list(rng.integers(0, 50000, 2048))
    for s in range(48):
        toks = system + list(rng.integers(0, 50000, int(rng.integers(1, 300))))
        want = 0 if s == 0 else 2048
        assert x.reserve_prefix(s, toks) == (Status.OK, want)
        x.register(s, toks)
        if s % 5 == 4:
            x.release(s - 2)
    x.same()
