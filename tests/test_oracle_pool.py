"""Pins the oracle's block pool: free list, block tables, reference counts,
copy-on-write, and the pool scenarios the pages work through."""
import numpy as np
import pytest

from oracle import PagedKVOracle, Status


def make(num_blocks=64, B=16, max_seqs=8, mbps=64, L=1, H=1, d=4, kv="bf16", order=None):
    return PagedKVOracle(num_layers=L, num_kv_heads=H, head_dim=d, block_size=B,
                         num_blocks=num_blocks, max_seqs=max_seqs, max_blocks_per_seq=mbps,
                         kv_dtype=kv, free_order=order)


def test_825_token_request_takes_52_blocks_fifo():
    # "Managing the KV Cache", Worked Example: ceil(825/16) = 52 blocks, 7 unused slots
    order = np.random.default_rng(1).permutation(128)
    o = make(num_blocks=128, order=order)
    assert o.reserve(0, 825) is Status.OK
    assert o.table(0) == [int(b) for b in order[:52]]
    assert len(o.table(0)) * 16 - 825 == 7
    assert o.free_list() == [int(b) for b in order[52:]]
    o.check_invariants()


def test_growth_claims_one_block_per_boundary():
    # "Managing the KV Cache", Answer Key item 2: growing claims one free block at a time
    o = make(num_blocks=16)
    seen = []
    for n in range(1, 70):
        before = len(o.free)
        assert o.reserve(3, n) is Status.OK
        took = before - len(o.free)
        assert took == (1 if (n - 1) % 16 == 0 else 0)
        seen.append(took)
        o.check_invariants()
    assert sum(seen) == 5 and o.table(3) == [0, 1, 2, 3, 4]


def test_12gib_pool_47_requests_then_block_53_overflows():
    # "Managing the KV Cache", Worked Capacity Under a 12 GiB KV Budget: 2,457 blocks
    # hold 47 requests at 825 tokens; growing into block 53 needs headroom.
    order = np.random.default_rng(2).permutation(2457)
    o = PagedKVOracle(num_layers=1, num_kv_heads=1, head_dim=1, block_size=16, num_blocks=2457,
                      max_seqs=48, max_blocks_per_seq=60, kv_dtype="bf16", free_order=order)
    for s in range(47):
        assert o.reserve(s, 825) is Status.OK
    assert o.reserve(47, 825) is Status.NO_BLOCKS          # a 48th request does not fit
    assert 47 not in o.tables
    assert len(o.free) == 2457 - 47 * 52 == 13
    for n in range(826, 833):                              # fills block 52's slots, no new block
        for s in range(47):
            assert o.reserve(s, n) is Status.OK
    assert len(o.free) == 13
    for s in range(13):                                    # the 833rd token needs block 53
        assert o.reserve(s, 833) is Status.OK
    snap = (o.free_list(), o.refcounts(), {s: o.table(s) for s in o.tables}, dict(o.lens))
    assert o.reserve(13, 833) is Status.NO_BLOCKS
    assert snap == (o.free_list(), o.refcounts(), {s: o.table(s) for s in o.tables}, dict(o.lens))
    o.check_invariants()


def test_parallel_sampling_cow_seven_copies_one_in_place():
    # kv-cache-pagedattention-serving, The bonus: sharing via copy-on-write (parallel sampling);
    # "Managing the KV Cache", Block Tables and Sharing: a fresh block only on divergence
    # inside a shared tail block.
    o = make(num_blocks=200, mbps=140, max_seqs=8)
    assert o.reserve(0, 2050) is Status.OK                 # 128 full blocks + tail of 2
    o.k[0][:] = np.arange(o.k[0].size, dtype=np.uint16).reshape(o.k[0].shape)
    for c in range(1, 8):
        assert o.fork(0, c) is Status.OK
    parent_table = o.table(0)
    assert all(o.ref[b] == 8 for b in parent_table)
    tail = parent_table[-1]
    for s in range(8):
        assert o.reserve(s, 2051) is Status.OK
        o.check_invariants()
    assert len(o.cow_log) == 7
    assert all(src == tail for src, _ in o.cow_log)
    for s in range(8):
        assert o.table(s)[:128] == parent_table[:128]
        assert o.ref[o.table(s)[-1]] == 1
    assert o.table(7)[-1] == tail                          # the last sharer writes in place
    for _, dst in o.cow_log:                               # copies carry the shared contents
        assert (o.k[0][dst] == o.k[0][tail]).all()
    assert all(o.ref[b] == 8 for b in parent_table[:128])
    # growth past the next boundary: one private block each, no copies
    for s in range(8):
        assert o.reserve(s, 2065) is Status.OK
    assert len(o.cow_log) == 7


def test_full_shared_blocks_are_never_copied():
    o = make(num_blocks=20)
    assert o.reserve(0, 32) is Status.OK                   # two full blocks
    assert o.fork(0, 1) is Status.OK
    assert o.reserve(0, 33) is Status.OK and o.reserve(1, 33) is Status.OK
    assert o.cow_log == []
    assert o.table(0)[:2] == o.table(1)[:2] and o.table(0)[2] != o.table(1)[2]


def test_cow_and_growth_need_is_checked_before_any_change():
    o = make(num_blocks=4, mbps=4)
    assert o.reserve(0, 17) is Status.OK                   # 2 blocks
    assert o.fork(0, 1) is Status.OK
    assert o.reserve(2, 16) is Status.OK                   # 1 block, 1 left
    snap = (o.free_list(), o.refcounts(), o.table(0), o.table(1))
    # growing seq 1 to 33 needs a CoW block and a new block: 2 > 1 free
    assert o.reserve(1, 33) is Status.NO_BLOCKS
    assert snap == (o.free_list(), o.refcounts(), o.table(0), o.table(1))
    assert o.cow_log == []
    assert o.reserve(1, 18) is Status.OK                   # CoW alone fits
    assert len(o.cow_log) == 1


def test_release_returns_blocks_in_logical_order_once_unreferenced():
    # "Managing the KV Cache", Block Tables and Sharing: a block returns to the free
    # list once no sequence references it
    o = make(num_blocks=10)
    assert o.reserve(0, 40) is Status.OK                   # blocks 0,1,2
    assert o.fork(0, 1) is Status.OK
    assert o.release(0) is Status.OK
    assert o.free_list() == [3, 4, 5, 6, 7, 8, 9]
    assert o.release(1) is Status.OK
    assert o.free_list() == [3, 4, 5, 6, 7, 8, 9, 0, 1, 2]
    assert o.reserve(5, 16) is Status.OK and o.table(5) == [3]
    o.check_invariants()


def test_invalid_calls():
    o = make(num_blocks=8, mbps=2, max_seqs=4)
    assert o.reserve(4, 1) is Status.INVALID_ARG
    assert o.reserve(-1, 1) is Status.INVALID_ARG
    assert o.reserve(0, 33) is Status.INVALID_ARG          # beyond max blocks per sequence
    assert o.reserve(0, 10) is Status.OK
    assert o.reserve(0, 9) is Status.INVALID_ARG           # no shrinking
    assert o.fork(1, 2) is Status.NO_SEQ
    assert o.fork(0, 0) is Status.SEQ_EXISTS
    assert o.release(3) is Status.NO_SEQ
    assert o.slot(0, 10) is Status.INVALID_ARG
    assert o.fork(0, 1) is Status.OK
    assert o.slot(0, 3) is Status.SHARED_BLOCK             # writes never land in shared blocks
    assert o.append(0, [0], [3], np.zeros((1, 1, 4), np.uint16), np.zeros((1, 1, 4), np.uint16),
                    "bf16") is Status.SHARED_BLOCK


def test_append_writes_the_slot_and_nothing_else():
    o = make(num_blocks=8, H=2, d=3)
    assert o.reserve(0, 20) is Status.OK and o.reserve(1, 5) is Status.OK
    k = np.array([[[1, 2, 3], [4, 5, 6]], [[7, 8, 9], [10, 11, 12]]], np.uint16)
    v = k + 100
    assert o.append(0, [0, 1], [17, 4], k, v, "bf16") is Status.OK
    b0 = o.table(0)[1]
    b1 = o.table(1)[0]
    assert (o.k[0][b0, :, 1, :] == k[0]).all() and (o.v[0][b0, :, 1, :] == v[0]).all()
    assert (o.k[0][b1, :, 4, :] == k[1]).all()
    assert int(o.k[0].astype(np.int64).sum()) == int(k.astype(np.int64).sum())


def test_random_operation_sequences_keep_invariants():
    g = np.random.default_rng(11)
    for trial in range(20):
        nb = int(g.integers(4, 40))
        B = int(g.choice([1, 2, 4, 16]))
        o = make(num_blocks=nb, B=B, max_seqs=6, mbps=12, order=g.permutation(nb))
        for _ in range(200):
            op = g.integers(0, 4)
            s = int(g.integers(0, 6))
            if op <= 1:
                cur = o.lens.get(s, 0)
                r = o.reserve(s, cur + int(g.integers(0, 2 * B + 2)))
                assert r in (Status.OK, Status.NO_BLOCKS, Status.INVALID_ARG)
            elif op == 2:
                o.fork(int(g.integers(0, 6)), s)
            else:
                o.release(s)
            o.check_invariants()


@pytest.mark.parametrize("B", [1, 16, 32])
def test_tail_waste_bound_under_growth(B):
    # "Managing the KV Cache", Internal Fragmentation: at most B - 1 empty slots per sequence
    o = make(num_blocks=1300, B=B, mbps=500, max_seqs=3)
    for n in range(0, 400, 7):
        for s in range(3):
            assert o.reserve(s, n + s) is Status.OK
            assert 0 <= len(o.table(s)) * B - o.lens[s] <= B - 1
