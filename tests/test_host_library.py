"""CPU tests of libpa.so: symbol exports, argument validation, and the
host block manager checked bit-exact against the oracle's pool model.

These need no GPU: a pool created without device buffers ("host-only")
runs the block manager alone; nothing here launches a kernel.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa
from oracle import PagedKVOracle, Status

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STATUS = {
    pa.PA_OK: Status.OK, pa.PA_ERR_INVALID_ARG: Status.INVALID_ARG,
    pa.PA_ERR_NO_BLOCKS: Status.NO_BLOCKS, pa.PA_ERR_NO_SEQ: Status.NO_SEQ,
    pa.PA_ERR_SEQ_EXISTS: Status.SEQ_EXISTS, pa.PA_ERR_SHARED_BLOCK: Status.SHARED_BLOCK,
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "pa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 18
    assert sorted(names) == sorted(pa.EXPORTS)
    L = ctypes.CDLL(pa.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    assert pa.pa_status_string(pa.PA_ERR_NO_BLOCKS) == "PA_ERR_NO_BLOCKS"
    assert pa.pa_status_string(12345) == "PA_UNKNOWN_STATUS"


def host_pool(nb=64, B=16, max_seqs=8, mbps=64, order=None):
    return pa.pa_pool_create(num_layers=1, num_kv_heads=1, block_size=B, num_blocks=nb,
                             max_seqs=max_seqs, max_blocks_per_seq=mbps, host_only=True,
                             free_order=order)


def oracle_pool(nb=64, B=16, max_seqs=8, mbps=64, order=None):
    return PagedKVOracle(num_layers=1, num_kv_heads=1, head_dim=1, block_size=B, num_blocks=nb,
                         max_seqs=max_seqs, max_blocks_per_seq=mbps, kv_dtype="bf16",
                         free_order=order)


def status_of(fn, *args):
    try:
        fn(*args)
        return Status.OK
    except pa.PAError as e:
        return STATUS[e.status]


def same_state(p, o):
    assert pa.pa_get_free_list(p) == o.free_list()
    assert pa.pa_get_refcounts(p) == o.refcounts()
    for s in range(p.max_seqs):
        if s in o.tables:
            n, tab = pa.pa_get_seq(p, s)
            assert n == o.lens[s] and tab == o.table(s), s
        else:
            with pytest.raises(pa.PAError) as ei:
                pa.pa_get_seq(p, s)
            assert ei.value.status == pa.PA_ERR_NO_SEQ
    assert pa.pa_get_cow_log(p) == o.cow_log


def test_worked_example_and_cow_match_oracle():
    order = np.random.default_rng(0).permutation(300)
    p, o = host_pool(nb=300, mbps=140, order=order), oracle_pool(nb=300, mbps=140, order=order)
    for s, n in ((0, 825), (1, 200), (2, 103), (3, 16)):
        assert status_of(pa.pa_alloc_blocks, p, s, n) is o.reserve(s, n) is Status.OK
    same_state(p, o)
    assert pa.pa_get_seq(p, 0)[1] == [int(b) for b in order[:52]]
    # parallel sampling: fork a partly filled prompt and diverge
    for c in (4, 5, 6, 7):
        assert status_of(pa.pa_fork_cow, p, 1, c) is o.fork(1, c) is Status.OK
    same_state(p, o)
    for s in (1, 4, 5, 6, 7):
        assert status_of(pa.pa_alloc_blocks, p, s, 201) is o.reserve(s, 201) is Status.OK
    same_state(p, o)
    assert len(o.cow_log) == 4
    for s in (4, 1, 0):
        assert status_of(pa.pa_free, p, s) is o.release(s) is Status.OK
        same_state(p, o)


def test_alloc_n_stops_at_first_failure_and_leaves_rest_untouched():
    p, o = host_pool(nb=10, mbps=10), oracle_pool(nb=10, mbps=10)
    with pytest.raises(pa.PAError) as ei:
        pa.pa_alloc_blocks_n(p, [0, 1, 2, 3], [64, 32, 80, 1])
    assert ei.value.status == pa.PA_ERR_NO_BLOCKS and ei.value.n_done == 2
    assert o.reserve(0, 64) is Status.OK and o.reserve(1, 32) is Status.OK
    assert o.reserve(2, 80) is Status.NO_BLOCKS
    same_state(p, o)
    assert pa.pa_alloc_blocks_n(p, [3, 2], [1, 16]) == 2


def test_12gib_pool_overflow_into_block_53_matches_oracle():
    order = np.random.default_rng(5).permutation(2457)
    p = host_pool(nb=2457, max_seqs=48, mbps=60, order=order)
    o = oracle_pool(nb=2457, max_seqs=48, mbps=60, order=order)
    seqs = list(range(47))
    pa.pa_alloc_blocks_n(p, seqs, [825] * 47)
    for s in seqs:
        o.reserve(s, 825)
    for n in range(826, 833):
        pa.pa_alloc_blocks_n(p, seqs, [n] * 47)
        for s in seqs:
            o.reserve(s, n)
    with pytest.raises(pa.PAError) as ei:
        pa.pa_alloc_blocks_n(p, seqs, [833] * 47)
    assert ei.value.status == pa.PA_ERR_NO_BLOCKS and ei.value.n_done == 13
    for s in range(13):
        assert o.reserve(s, 833) is Status.OK
    assert o.reserve(13, 833) is Status.NO_BLOCKS
    same_state(p, o)


def test_random_operations_match_oracle_bit_exact():
    g = np.random.default_rng(123)
    for trial in range(25):
        nb = int(g.integers(4, 60))
        B = int(g.choice([16, 32]))
        order = g.permutation(nb)
        p, o = host_pool(nb=nb, B=B, max_seqs=6, mbps=10, order=order), oracle_pool(
            nb=nb, B=B, max_seqs=6, mbps=10, order=order)
        for _ in range(150):
            op = int(g.integers(0, 5))
            s = int(g.integers(-1, 7))
            if op <= 1:
                n = o.lens.get(s, 0) + int(g.integers(0, 2 * B + 3)) if 0 <= s < 6 else 5
                assert status_of(pa.pa_alloc_blocks, p, s, n) is o.reserve(s, n)
            elif op == 2:
                c = int(g.integers(-1, 7))
                assert status_of(pa.pa_fork_cow, p, s, c) is o.fork(s, c)
            elif op == 3:
                assert status_of(pa.pa_free, p, s) is o.release(s)
            else:
                seqs = [int(x) for x in g.integers(0, 6, size=3)]
                lens = [o.lens.get(x, 0) + int(g.integers(0, B)) for x in seqs]
                try:
                    done = pa.pa_alloc_blocks_n(p, seqs, lens)
                except pa.PAError as e:
                    done = e.n_done
                for k, (x, n) in enumerate(zip(seqs, lens)):
                    r = o.reserve(x, n)
                    if r is not Status.OK:
                        assert k == done
                        break
                else:
                    assert done == len(seqs)
            same_state(p, o)
            o.check_invariants()


def test_debug_fail_after_injects_no_blocks_without_state_change():
    p, o = host_pool(nb=20), oracle_pool(nb=20)
    pa.pa_debug_fail_after(p, 2)
    pa.pa_alloc_blocks(p, 0, 32)                       # 2 blocks: allowed
    o.reserve(0, 32)
    with pytest.raises(pa.PAError) as ei:
        pa.pa_alloc_blocks(p, 1, 1)
    assert ei.value.status == pa.PA_ERR_NO_BLOCKS
    same_state(p, o)
    pa.pa_alloc_blocks(p, 0, 32)                       # needs nothing: fine
    pa.pa_debug_fail_after(p, -1)
    pa.pa_alloc_blocks(p, 1, 1)
    o.reserve(1, 1)
    same_state(p, o)


def test_invalid_descriptors_rejected():
    base = dict(num_layers=1, num_kv_heads=1, block_size=16, num_blocks=8, max_seqs=2,
                max_blocks_per_seq=4, host_only=True)
    for bad in (dict(block_size=8), dict(num_blocks=0), dict(max_seqs=0), dict(head_dim=64),
                dict(free_order=[0, 1, 2, 3, 4, 5, 6, 6]), dict(free_order=[0, 1, 2, 3, 4, 5, 6, 8]),
                dict(kv_dtype="fp16", act_dtype="bf16"), dict(min_partition_tokens=24)):
        with pytest.raises(pa.PAError) as ei:
            pa.pa_pool_create(**{**base, **bad})
        assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_device_calls_rejected_on_host_only_pool():
    p = host_pool()
    pa.pa_alloc_blocks(p, 0, 5)
    L = pa.lib()
    seq = (ctypes.c_int32 * 1)(0)
    pos = (ctypes.c_int32 * 1)(0)
    st = L.pa_append_kv(p.handle, 0, 1, seq, pos, ctypes.c_void_p(16), ctypes.c_void_p(16), None)
    assert st == pa.PA_ERR_INVALID_ARG
    st = L.pa_decode_attention(p.handle, 0, 1, seq, 1, ctypes.c_void_p(16), ctypes.c_void_p(16),
                               ctypes.c_float(1.0), 0, None)
    assert st == pa.PA_ERR_INVALID_ARG
    bits = ctypes.c_uint32()
    assert L.pa_check_device_errors(p.handle, None, ctypes.byref(bits)) == pa.PA_ERR_INVALID_ARG


def test_device_pool_descriptor_validation_without_gpu():
    # Creation only validates: pointers are never dereferenced, so fake
    # addresses exercise the checks on a machine without a GPU.
    L = pa.lib()
    d = pa.binding.pa_pool_desc()
    d.num_layers, d.num_kv_heads, d.head_dim, d.block_size = 2, 2, 128, 16
    d.num_blocks, d.max_seqs, d.max_blocks_per_seq = 8, 2, 4
    d.kv_dtype = d.act_dtype = pa.binding.PA_BF16
    need = L.pa_workspace_size(ctypes.byref(d))
    assert need > 0
    h = ctypes.c_void_p()
    d.k_cache, d.v_cache = 4096, 0
    assert L.pa_pool_create(ctypes.byref(d), ctypes.byref(h)) == pa.PA_ERR_INVALID_ARG
    d.v_cache = 4104                                   # not 16-byte aligned
    assert L.pa_pool_create(ctypes.byref(d), ctypes.byref(h)) == pa.PA_ERR_INVALID_ARG
    d.v_cache = 8192
    d.workspace, d.workspace_bytes = 1 << 20, need - 1  # too small
    assert L.pa_pool_create(ctypes.byref(d), ctypes.byref(h)) == pa.PA_ERR_INVALID_ARG
    d.workspace_bytes = need
    assert L.pa_pool_create(ctypes.byref(d), ctypes.byref(h)) == pa.PA_OK
    L.pa_pool_destroy(h)
    d.kv_dtype = pa.binding.PA_FP8_E4M3                # FP8 without scales
    assert L.pa_pool_create(ctypes.byref(d), ctypes.byref(h)) == pa.PA_ERR_INVALID_ARG
    d.num_blocks = 1 << 26                              # TMA row coordinate would overflow
    d.kv_dtype = pa.binding.PA_BF16
    assert L.pa_pool_create(ctypes.byref(d), ctypes.byref(h)) == pa.PA_ERR_INVALID_ARG


def test_workspace_size_grows_with_fixed_partitions():
    d = pa.binding.pa_pool_desc()
    d.num_layers, d.num_kv_heads, d.head_dim, d.block_size = 1, 8, 128, 16
    d.num_blocks, d.max_seqs, d.max_blocks_per_seq = 100, 64, 4096
    small = pa.pa_workspace_size(d)
    d.min_partition_tokens = 16
    big = pa.pa_workspace_size(d)
    assert big > small
    assert big >= 64 * 8 * 4096 * 8 * 130 * 4
