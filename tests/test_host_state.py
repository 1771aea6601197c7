"""Host state checkpoint (pa_state_save / pa_state_load) of the block manager.

A restored pool must behave exactly as the saved one from the save on: the
same blocks handed out, shared, copied, cached, evicted and released.  The
pin is the oracle ("kv-cache-pagedattention-serving", PagedAttention: virtual
memory for GPUs, Beyond paging: radix trees and continuous batching), copied
at the save point: the library restored from the image and the oracle copy
are driven by the same operations and compared bit-exactly after each one.
Images that are truncated, corrupt, inconsistent or of another geometry are
refused with nothing changed.  Host-only pools; no GPU.
"""
import copy
import struct

import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa
from oracle import Status

from test_host_prefix import Both


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


class Book:
    """The driver's own bookkeeping (which sequences hold which tokens)."""

    def __init__(self, rng, B, vocab):
        self.systems = [list(rng.integers(0, vocab, int(rng.integers(B, 6 * B)))) for _ in range(4)]
        self.hist, self.done, self.free_ids = {}, [], list(range(24))


def run(x, book, rng, steps, B, vocab):
    """Random prompts with prefix reuse, registrations, forks, growth with
    copy-on-write and releases; library and oracle compared after each."""
    hist, done, free_ids = book.hist, book.done, book.free_ids
    for _ in range(steps):
        op = rng.random()
        if op < 0.3 and free_ids:
            base = (done[int(rng.integers(len(done)))] if done and rng.random() < 0.5
                    else book.systems[int(rng.integers(len(book.systems)))])
            toks = base + list(rng.integers(0, vocab, int(rng.integers(0, 3 * B))))
            s = free_ids.pop(0)
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


def snapshot(p):
    tables = {}
    for s in range(p.max_seqs):
        try:
            tables[s] = pa.pa_get_seq(p, s)
        except pa.PAError:
            tables[s] = None
    return (pa.pa_get_free_list(p), pa.pa_get_cached_blocks(p), pa.pa_get_refcounts(p), tables)


def trie_of(words):
    """Offset of the node records in a state image, their count and the live
    (not spare) nodes, following the image layout of block_manager.cpp."""
    nb, B, max_seqs = words[1], words[2], words[3]
    at = 5
    at += 1 + words[at]                  # free list
    at += 2 * nb                         # reference counts, block -> node
    for _ in range(max_seqs):
        at += 3 + words[at + 2]          # active, len, table size, table
    nn = words[at]
    nodes_at = at + 1
    at = nodes_at + 5 * nn + nn * B
    spare = set(words[at + 1: at + 1 + words[at]])
    return nodes_at, nn, [c for c in range(nn) if c not in spare]


@pytest.mark.parametrize("seed,nb,B", [(0, 40, 16), (1, 24, 16), (2, 48, 32), (3, 20, 16)])
def test_restore_replays_exactly(seed, nb, B):
    vocab = 7
    rng = np.random.default_rng([seed, 71])
    x = Both(nb, B)
    book = Book(rng, B, vocab)
    run(x, book, rng, 60, B, vocab)
    image = pa.pa_state_save(x.p)
    assert len(image) == pa.pa_state_size(x.p)
    saved_oracle, saved_book, saved_snap = copy.deepcopy(x.o), copy.deepcopy(book), snapshot(x.p)
    # go on, then come back to the save point and take the same path again
    run(x, book, np.random.default_rng([seed, 72]), 60, B, vocab)
    after_first = snapshot(x.p)
    pa.pa_state_load(x.p, image)
    x.o, book = copy.deepcopy(saved_oracle), copy.deepcopy(saved_book)
    assert snapshot(x.p) == saved_snap
    assert pa.pa_get_cow_log(x.p) == []
    x.same()
    run(x, book, np.random.default_rng([seed, 72]), 60, B, vocab)
    assert snapshot(x.p) == after_first
    # a fresh pool of the same geometry restored from the image takes it too
    y = Both(nb, B)
    pa.pa_state_load(y.p, image)
    y.o = copy.deepcopy(saved_oracle)
    y.same()
    run(y, copy.deepcopy(saved_book), np.random.default_rng([seed, 73]), 60, B, vocab)


def test_refused_images_change_nothing():
    B, vocab = 16, 7
    rng = np.random.default_rng(5)
    x = Both(32, B)
    run(x, Book(rng, B, vocab), rng, 40, B, vocab)
    image = pa.pa_state_save(x.p)
    target = Both(32, B)
    run(target, Book(np.random.default_rng(6), B, vocab), np.random.default_rng(6), 20, B, vocab)
    before = snapshot(target.p)
    words = list(struct.unpack(f"<{len(image) // 4}i", image))

    def refused(img):
        with pytest.raises(pa.PAError) as e:
            pa.pa_state_load(target.p, img)
        assert e.value.status == pa.PA_ERR_INVALID_ARG
        assert snapshot(target.p) == before

    def packed(ws):
        return struct.pack(f"<{len(ws)}i", *ws)

    refused(image[:-4])                                  # truncated
    refused(image + b"\0\0\0\0")                         # trailing words
    refused(image[:-1])                                  # not whole words
    refused(packed([0x12345678] + words[1:]))            # not a state image
    nb = words[1]
    ref0 = 5 + 1 + words[5]                              # first reference count
    bad = list(words)
    bad[ref0] += 1                                       # a count its tables do not support
    refused(packed(bad))
    bad = list(words)
    bad[ref0 + nb] = nb + 7                              # a block names a node that does not exist
    refused(packed(bad))
    # the prefix trie inside the image: a live node's child count, a parent
    # cycle and a key that is not the hash of (parent, tokens)
    nodes_at, nn, live = trie_of(words)
    assert live, "the drive registered no prefix"
    c = live[0]
    for field, value in ((2, words[nodes_at + 5 * c + 2] + 1), (0, c), (3, words[nodes_at + 5 * c + 3] ^ 1)):
        bad = list(words)
        bad[nodes_at + 5 * c + field] = value
        refused(packed(bad))
    other = Both(33, B)                                  # another geometry
    with pytest.raises(pa.PAError) as e:
        pa.pa_state_load(other.p, image)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    # and the untouched target still works against its own oracle
    target.same()
    pa.pa_state_load(target.p, image)                    # the valid image loads


def test_empty_pool_round_trip():
    x = Both(8, 16)
    image = pa.pa_state_save(x.p)
    pa.pa_alloc_blocks(x.p, 0, 40)
    x.o.reserve(0, 40)
    x.same()
    pa.pa_state_load(x.p, image)
    assert pa.pa_get_free_list(x.p) == list(range(8))
    assert pa.pa_get_refcounts(x.p) == [0] * 8
