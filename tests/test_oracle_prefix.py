"""Pins of the oracle's block-granular prefix cache.

What the pages fix (kv-cache-pagedattention-serving, Beyond paging: radix
trees and continuous batching; "Managing the KV Cache", Block Tables and
Sharing and Answer Key item 4): prefixes are matched a whole block at a time
(a 103-token prompt reuses 96 tokens with 16-token blocks), cached blocks
stay reference counted and are evicted least recently used when the pool is
full.  The mathematics fixes the rest: the KV of token t is a function of
tokens 0..t, so a correct cache hands a new prompt exactly the KV it would
have computed itself.  The content test below writes, for every position, a
row that is a hash of the whole token prefix ending there; any wrong match,
stale registration after eviction, or block keyed by its own tokens only
shows up as a wrong row.
"""
import hashlib
import json
import os

import numpy as np
import pytest

from oracle import PagedKVOracle, Status

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "prefix_granularity.json")
D = 8


def pool(nb, B, max_seqs=16, mbps=64):
    return PagedKVOracle(num_layers=1, num_kv_heads=1, head_dim=D, block_size=B, num_blocks=nb,
                         max_seqs=max_seqs, max_blocks_per_seq=mbps, kv_dtype="bf16")


def row(prefix):
    """KV row of the last token of `prefix`: a hash of the whole prefix."""
    h = hashlib.blake2b(np.asarray(prefix, np.int64).tobytes(), digest_size=2 * D).digest()
    return np.frombuffer(h, np.uint16).copy()


def write(o, seq, tokens, lo, hi):
    """Append the rows of positions lo..hi-1 of `seq` (token history `tokens`)."""
    if hi <= lo:
        return
    k = np.stack([row(tokens[: t + 1]) for t in range(lo, hi)])[:, None, :]
    v = k ^ np.uint16(0x5A5A)
    st = o.append(0, [seq] * (hi - lo), list(range(lo, hi)), k, v, "bf16")
    assert st == Status.OK, st


def check_contents(o, hist):
    for s, toks in hist.items():
        assert o.lens[s] == len(toks)
        for t in range(len(toks)):
            b = o.tables[s][t // o.B]
            want = row(toks[: t + 1])
            assert np.array_equal(o.k[0][b, 0, t % o.B], want), (s, t)
            assert np.array_equal(o.v[0][b, 0, t % o.B], want ^ np.uint16(0x5A5A)), (s, t)


def prefill(o, seq, tokens):
    st, cached = o.reserve_prefix(seq, tokens)
    assert st == Status.OK
    write(o, seq, tokens, cached, len(tokens))
    assert o.register(seq, tokens) == Status.OK
    return cached


def test_worked_103_token_prompt_reuses_96():
    g = json.load(open(GOLDEN))["worked_103"]
    B, n = g["block_size"], g["prompt_tokens"]
    o = pool(64, B)
    toks = list(np.random.default_rng(1).integers(0, 1000, n))
    assert prefill(o, 0, toks) == 0
    st, cached = o.reserve_prefix(1, toks)
    assert st == Status.OK
    assert cached == g["reused_tokens"] and n - cached == g["recomputed_tokens"]
    # the same prefix inside a longer cached conversation: still whole blocks only
    o2 = pool(64, B)
    longer = toks + list(np.random.default_rng(2).integers(0, 1000, 97))
    prefill(o2, 0, longer)
    assert o2.reserve_prefix(1, toks) == (Status.OK, g["reused_tokens"])


def test_lru_trace_by_hand():
    """B = 4, six blocks, free list 0..5; every value below worked by hand."""
    o = pool(6, 4)
    a = list(range(1, 13))                                  # 12 tokens = 3 blocks
    assert prefill(o, 0, a) == 0 and o.table(0) == [0, 1, 2]
    assert o.release(0) == Status.OK
    assert o.free_list() == [3, 4, 5] and o.cached_list() == [2, 1, 0]
    assert o.reserve(1, 8) == Status.OK and o.table(1) == [3, 4]
    assert o.reserve_prefix(2, a[:8] + [99, 98]) == (Status.OK, 8)
    assert o.table(2) == [0, 1, 5] and o.free_list() == [] and o.cached_list() == [2]
    assert o.reserve(3, 4) == Status.OK and o.table(3) == [2]      # evicts block 2
    assert o.cached_list() == [] and o.match(a) == 2
    assert o.release(2) == Status.OK
    assert o.free_list() == [5] and o.cached_list() == [1, 0]
    assert o.reserve(4, 8) == Status.OK and o.table(4) == [5, 1]    # free first, then LRU
    assert o.cached_list() == [0] and o.match(a) == 1
    o.check_invariants()


def test_reusing_every_idle_block_and_needing_one_more_fails_cleanly():
    o = pool(3, 4)
    a = list(range(12))
    prefill(o, 0, a)
    o.release(0)
    assert o.free_list() == [] and o.cached_list() == [2, 1, 0]
    before = (o.free_list(), o.cached_list(), o.refcounts(), dict(o.registry))
    assert o.reserve_prefix(1, a + [7]) == (Status.NO_BLOCKS, 0)
    assert (o.free_list(), o.cached_list(), o.refcounts(), dict(o.registry)) == before
    assert 1 not in o.tables
    assert o.reserve_prefix(1, a) == (Status.OK, 12)               # fits without a new block
    o.check_invariants()


def test_registered_blocks_are_immutable_and_first_registration_wins():
    o = pool(16, 4)
    a = [5, 6, 7, 8, 9, 10]
    prefill(o, 0, a)
    assert o.slot(0, 2) == Status.SHARED_BLOCK                      # in the registered block 0
    assert o.slot(0, 5) == (o.table(0)[1], 1)                        # the partial tail is writable
    # an independent copy of the same prompt, written by hand, then registered
    assert o.reserve(1, 6) == Status.OK
    write(o, 1, a, 0, 6)
    assert o.register(1, a) == Status.OK
    assert o.registry[tuple(a[:4])] == o.table(0)[0]
    assert o.table(1)[0] not in o.key_of
    # registering a block under a different prefix than its own is an error
    assert o.register(0, [1, 2, 3, 4]) == Status.INVALID_ARG
    assert o.register(0, a + [1]) == Status.INVALID_ARG              # longer than the sequence
    o.check_invariants()


def test_without_registrations_reserve_prefix_is_reserve():
    rng = np.random.default_rng(3)
    a, b = pool(200, 16, 32), pool(200, 16, 32)
    for s in range(20):
        n = int(rng.integers(0, 300))
        toks = list(rng.integers(0, 5, n))
        assert a.reserve_prefix(s, toks) == (Status.OK, 0)
        assert b.reserve(s, n) == Status.OK
        if rng.random() < 0.3:
            victim = int(rng.integers(0, s + 1))
            assert a.release(victim) == b.release(victim)
    assert a.tables == b.tables and a.free_list() == b.free_list() and a.refcounts() == b.refcounts()
    assert a.cached_list() == []


def lcp(x, y):
    n = 0
    for p, q in zip(x, y):
        if p != q:
            break
        n += 1
    return n


def run_conversations(seed, nb, B, vocab, steps, check_optimal):
    """Shared system prompts, multi-turn continuations, forks and decode steps.
    Checks invariants and every cached row after each operation; with
    `check_optimal` (no eviction possible) also that each match is as long
    as brute force over every registered token list allows."""
    rng = np.random.default_rng([seed, 17])
    o = pool(nb, B, max_seqs=24, mbps=64)
    systems = [list(rng.integers(0, vocab, int(rng.integers(B, 5 * B)))) for _ in range(3)]
    hist, done, registered = {}, [], []
    free_ids = list(range(24))
    for _ in range(steps):
        op = rng.random()
        if op < 0.3 and free_ids:                                   # new request
            if done and rng.random() < 0.5:
                base = done[int(rng.integers(len(done)))]            # next turn of a conversation
            else:
                base = systems[int(rng.integers(len(systems)))]
            toks = base + list(rng.integers(0, vocab, int(rng.integers(0, 3 * B))))
            s = free_ids.pop(0)
            st, cached = o.reserve_prefix(s, toks)
            if st == Status.NO_BLOCKS:
                free_ids.insert(0, s)
                continue
            assert st == Status.OK and cached % B == 0 and cached <= len(toks)
            if check_optimal:
                best = max([lcp(toks, r) // B for r in registered] + [0])
                assert cached == min(best, len(toks) // B) * B
            hist[s] = toks
            write(o, s, toks, cached, len(toks))
            assert o.register(s, toks) == Status.OK
            registered.append(toks[: len(toks) // B * B])
        elif op < 0.4 and hist and free_ids:                        # parallel sample
            parent = list(hist)[int(rng.integers(len(hist)))]
            s = free_ids.pop(0)
            assert o.fork(parent, s) == Status.OK
            hist[s] = list(hist[parent])
        elif op < 0.8 and hist:                                     # one decode step
            s = list(hist)[int(rng.integers(len(hist)))]
            if o.reserve(s, len(hist[s]) + 1) != Status.OK:
                continue
            hist[s].append(int(rng.integers(0, vocab)))
            write(o, s, hist[s], len(hist[s]) - 1, len(hist[s]))
            if rng.random() < 0.3:
                assert o.register(s, hist[s]) == Status.OK
                registered.append(hist[s][: len(hist[s]) // B * B])
        elif hist:                                                  # finish a request
            s = list(hist)[int(rng.integers(len(hist)))]
            assert o.release(s) == Status.OK
            done.append(hist.pop(s))
            free_ids.append(s)
        o.check_invariants()
        check_contents(o, hist)
    return o


@pytest.mark.parametrize("seed", range(6))
def test_conversations_under_pool_pressure_keep_exact_contents(seed):
    o = run_conversations(seed, nb=40, B=4, vocab=2, steps=150, check_optimal=False)
    assert o.registry                                                # the cache was used


@pytest.mark.parametrize("seed", range(4))
def test_matches_are_longest_when_nothing_is_evicted(seed):
    run_conversations(seed, nb=4000, B=4, vocab=3, steps=120, check_optimal=True)
