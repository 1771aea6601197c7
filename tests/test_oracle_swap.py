"""Pins of the oracle's swap-out / swap-in.

"Managing the KV Cache" (Offload; Hands-On Exercise) and
kv-cache-pagedattention-serving (Beyond paging: radix trees and continuous
batching) say that a preempted sequence's KV can move to host memory and be
paged back.  Fixed by the pages and the mathematics: the allocated-block
bytes of the exercise's 1,525-token request (derived from the printed
bytes-per-token figures), and that paging back restores every cached token,
so attention over the sequence is unchanged.  The image layout is checked
against the rows the test itself appended at each position.
"""
import json
import os

import numpy as np
import pytest

from oracle import PagedKVOracle, Status

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "exercise_derived.json")

SHAPES = {  # case -> (layers, kv_heads, head_dim, bytes per element)
    "bf16_gqa_b16": (80, 8, 128, 2), "bf16_gqa_b32": (80, 8, 128, 2),
    "fp8_gqa_b16": (80, 8, 128, 1), "bf16_mha64_b16": (80, 64, 128, 2),
}


def test_swap_bytes_are_the_exercise_allocated_bytes():
    g = json.load(open(GOLDEN))
    for case in g["cases"]:
        L, H, d, e = SHAPES[case["name"]]
        o = PagedKVOracle(num_layers=L, num_kv_heads=H, head_dim=d, block_size=case["block_size"],
                          num_blocks=8, max_seqs=1, max_blocks_per_seq=8,
                          kv_dtype="fp8_e4m3" if e == 1 else "bf16", stored_layers=[])
        n = g["lengths"][2]
        assert o.swap_bytes(n, e) == case["offload_allocated_bytes"]
        assert n * 2 * L * H * d * e == case["offload_useful_bytes"]
        assert o.swap_bytes(n, e) - case["offload_useful_bytes"] == (
            (case["offload_allocated_bytes"] // case["bytes_per_token"]) - n) * case["bytes_per_token"]


class Pool:
    """An oracle pool plus the rows the test appended, per (seq, layer, pos)."""

    def __init__(self, nb=64, B=16, L=3, H=2, d=8, seed=0):
        self.o = PagedKVOracle(num_layers=L, num_kv_heads=H, head_dim=d, block_size=B,
                               num_blocks=nb, max_seqs=8, max_blocks_per_seq=32, kv_dtype="bf16",
                               free_order=np.random.default_rng(seed).permutation(nb))
        self.g = np.random.default_rng([seed, 3])
        self.rows = {}

    def grow(self, s, n):
        o = self.o
        cur = o.lens.get(s, 0)
        assert o.reserve(s, cur + n) == Status.OK
        for layer in range(o.L):
            k = self.g.integers(0, 0x3F80, (n, o.H, o.d)).astype(np.uint16)   # finite bf16
            v = self.g.integers(0, 0x3F80, (n, o.H, o.d)).astype(np.uint16)
            assert o.append(layer, [s] * n, list(range(cur, cur + n)), k, v, "bf16") == Status.OK
            rk, rv = self.rows.get((s, layer), (np.zeros((0, o.H, o.d), np.uint16),) * 2)
            self.rows[(s, layer)] = (np.concatenate([rk, k]), np.concatenate([rv, v]))

    def attention(self, s, q):
        return np.stack([self.o.attention(layer, [s], q, "bf16", 0.3)[0] for layer in range(self.o.L)])


def test_image_layout_holds_each_appended_row_at_its_place():
    p = Pool()
    p.grow(0, 37)
    p.grow(1, 5)
    st, img, n = p.o.swap_out(0)
    assert st == Status.OK and n == 37
    B = p.o.B
    assert img.shape == (2, 3, 3, 2, B, 8) and img.nbytes == p.o.swap_bytes(37, 2)
    for layer in range(3):
        rk, rv = p.rows[(0, layer)]
        for t in range(37):
            assert np.array_equal(img[0, t // B, layer, :, t % B, :], rk[t])
            assert np.array_equal(img[1, t // B, layer, :, t % B, :], rv[t])


def test_round_trip_restores_attention_exactly_and_frees_blocks():
    p = Pool(nb=32, seed=1)
    for s, n in enumerate([70, 16, 33]):            # 5 + 1 + 3 blocks
        p.grow(s, n)
    q = np.random.default_rng(9).integers(0, 0x3F00, (1, 4, 8)).astype(np.uint16)
    before = p.attention(0, q)
    old = p.o.table(0)
    st, img, n = p.o.swap_out(0)
    assert st == Status.OK and n == 70 and 0 not in p.o.tables
    assert p.o.free_list()[-5:] == old and len(p.o.free_list()) == 28
    p.grow(3, 28 * 16)                              # takes every free block: old ones too
    assert set(old) <= set(p.o.table(3))
    B = p.o.B

    def holds_own_rows(s):
        tab = p.o.table(s)
        for layer in range(3):
            rk, rv = p.rows[(s, layer)]
            for t in range(len(rk)):
                assert np.array_equal(p.o.k[layer][tab[t // B], :, t % B, :], rk[t])
                assert np.array_equal(p.o.v[layer][tab[t // B], :, t % B, :], rv[t])

    for s in (1, 2, 3):
        holds_own_rows(s)
    assert p.o.swap_in(0, n, img) == Status.NO_BLOCKS
    assert p.o.release(3) == Status.OK
    assert p.o.swap_in(0, n, img) == Status.OK
    assert np.array_equal(p.attention(0, q), before)
    for s in (0, 1, 2):
        holds_own_rows(s)
    p.o.check_invariants()


def test_forked_and_registered_blocks():
    p = Pool(seed=2)
    p.grow(0, 40)
    assert p.o.fork(0, 1) == Status.OK
    q = np.random.default_rng(4).integers(0, 0x3F00, (1, 4, 8)).astype(np.uint16)
    child = p.attention(1, q)
    ref = p.o.refcounts()
    shared = p.o.table(0)
    st, img, n = p.o.swap_out(1)
    assert st == Status.OK
    assert all(p.o.refcounts()[b] == ref[b] - 1 for b in shared)
    assert p.o.swap_in(1, n, img) == Status.OK
    assert not set(p.o.table(1)) & set(shared)      # private copies
    assert all(p.o.refcounts()[b] == 1 for b in p.o.table(1))
    assert np.array_equal(p.attention(1, q), child)
    # registered blocks of a swapped-out sequence stay cached for other prompts
    toks = list(range(40))
    assert p.o.register(0, toks) == Status.OK
    st, img, n = p.o.swap_out(0)
    assert st == Status.OK and p.o.cached_list() == [shared[1], shared[0]]
    assert p.o.free_list()[-1] == shared[2]         # the partial tail is not registered
    assert p.o.match(toks) == 2
    assert p.o.swap_in(0, n, img) == Status.OK
    assert not set(p.o.table(0)) & set(shared)      # fresh blocks; the cache is kept
    assert p.o.cached_list() == [shared[1], shared[0]]
    p.o.check_invariants()


def test_empty_sequence_swaps_an_empty_image():
    p = Pool(seed=4)
    assert p.o.reserve(0, 0) == Status.OK
    st, img, n = p.o.swap_out(0)
    assert st == Status.OK and n == 0 and img.nbytes == p.o.swap_bytes(0, 2) == 0
    assert p.o.swap_in(0, 0, img) == Status.OK and p.o.lens[0] == 0 and p.o.table(0) == []
    p.o.check_invariants()


def test_swap_in_without_room_changes_nothing():
    p = Pool(nb=8, seed=3)
    p.grow(0, 64)                                   # 4 blocks
    st, img, n = p.o.swap_out(0)
    p.grow(1, 80)                                   # 5 of the 8 blocks
    before = (p.o.free_list(), p.o.refcounts(), dict(p.o.tables))
    assert p.o.swap_in(0, n, img) == Status.NO_BLOCKS
    assert (p.o.free_list(), p.o.refcounts(), dict(p.o.tables)) == before
    assert p.o.swap_in(1, n, img) == Status.SEQ_EXISTS
    assert p.o.swap_out(5) == (Status.NO_SEQ, None, 0)
