"""GPU parity of swap-out / swap-in ("Managing the KV Cache", Offload;
kv-cache-pagedattention-serving, Beyond paging: radix trees and continuous
batching): the host image's valid slots bit-exact against the oracle's, the
blocks overwritten by other work while the sequence is out, and after paging
back the cache, tables and decode output equal to the oracle's.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle import Status
from paged_harness import Pair, to_dev
from workloads import Purpose, normal_bits, rng, workload

pytestmark = pytest.mark.gpu


def host_image(pool, n):
    return torch.empty(pa.pa_swap_bytes(pool, n), dtype=torch.uint8, pin_memory=True)


def check_image(P, img, image, n):
    """Valid slots (t < n) of the library's host image equal the oracle's."""
    B = P.oracle.B
    got = img.numpy().view(image.dtype).reshape(image.shape)
    for j in range(image.shape[1]):
        m = min(B, n - j * B)
        assert np.array_equal(got[:, j, :, :, :m, :], image[:, j, :, :, :m, :]), j


def fill_free_blocks(P, seq, layers):
    """A new sequence takes every free block and writes all of them."""
    w = P.w
    n = len(P.oracle.free_list()) * w.block_size
    pa.pa_alloc_blocks(P.pool, seq, n)
    assert P.oracle.reserve(seq, n) == Status.OK
    g = rng(w.seed, 88, Purpose.MISC, seq)
    for layer in layers:
        k = normal_bits(g, (n, w.num_kv_heads, w.head_dim), w.act_dtype)
        v = normal_bits(g, (n, w.num_kv_heads, w.head_dim), w.act_dtype)
        P.append(layer, [seq] * n, list(range(n)), k, v)
    return n


def test_round_trip_three_layers_blocks_overwritten_meanwhile():
    w = dataclasses.replace(workload("tiny"), num_layers=3, max_seqs=8, max_blocks_per_seq=128)
    P = Pair(w, min_partition=16)
    P.prefill()
    seqs, pos = P.reserve_step(0)
    for layer in range(3):
        P.append_step(0, layer, seqs, pos)
    n0, old = P.oracle.lens[0], P.oracle.table(0)
    img = host_image(P.pool, n0)
    pa.pa_swap_out(P.pool, 0, img)
    st, image, n = P.oracle.swap_out(0)
    assert st == Status.OK and n == n0
    torch.cuda.synchronize()
    check_image(P, img, image, n)
    P.check_metadata()
    fill_free_blocks(P, 4, range(3))
    assert set(old) <= set(P.oracle.table(4))
    for layer in range(3):
        P.check_cache(layer)
    pa.pa_free(P.pool, 4)
    assert P.oracle.release(4) == Status.OK
    pa.pa_swap_in(P.pool, 0, n, img)
    assert P.oracle.swap_in(0, n, image) == Status.OK
    P.check_metadata()
    for layer in range(3):
        P.check_cache(layer)
        for part in (0, -1):
            q, out = P.decode(0, layer, seqs, part)
            torch.cuda.synchronize()
            P.check_attention(layer, seqs, q, out)
    assert P.device_errors() == 0


def test_forked_child_fp8_pages_back_private():
    w = dataclasses.replace(workload("fp8_long", tokens=512), max_seqs=9)
    P = Pair(w, min_partition=16)
    P.prefill()
    pa.pa_fork_cow(P.pool, 2, 8)
    assert P.oracle.fork(2, 8) == Status.OK
    shared = P.oracle.table(2)
    n = P.oracle.lens[8]
    img = host_image(P.pool, n)
    pa.pa_swap_out(P.pool, 8, img)
    st, image, _ = P.oracle.swap_out(8)
    assert st == Status.OK
    torch.cuda.synchronize()
    check_image(P, img, image, n)
    assert all(pa.pa_get_refcounts(P.pool)[b] == 1 for b in shared)
    pa.pa_swap_in(P.pool, 8, n, img)
    assert P.oracle.swap_in(8, n, image) == Status.OK
    assert not set(P.oracle.table(8)) & set(shared)
    P.check_metadata()
    P.check_cache(0)
    seqs = [2, 8, 5]
    q_bits = normal_bits(rng(w.seed, 88, Purpose.Q), (3, w.num_q_heads, w.head_dim), w.act_dtype)
    q = to_dev(q_bits, w.act_dtype)
    for part in (0, 512, -1):
        out = torch.empty_like(q)
        pa.pa_decode_attention(P.pool, 0, seqs, q, out, w.scale, part)
        torch.cuda.synchronize()
        P.check_attention(0, seqs, q_bits, out)
    assert P.device_errors() == 0


def test_refusals_change_nothing():
    w = dataclasses.replace(workload("tiny"), max_seqs=8, max_blocks_per_seq=128)
    P = Pair(w, min_partition=16)
    P.prefill()
    need = pa.pa_swap_bytes(P.pool, 825)
    small = torch.empty(need - 1, dtype=torch.uint8, pin_memory=True)
    with pytest.raises(pa.PAError) as e:
        pa.pa_swap_out(P.pool, 0, small)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    # device memory as the image is refused on the host, before any copy
    dev = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = pa.lib().pa_swap_out(P.pool.handle, 0, ctypes.c_void_p(dev.data_ptr()), need,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_ERR_INVALID_ARG
    P.check_metadata()
    img = host_image(P.pool, 825)
    pa.pa_swap_out(P.pool, 0, img)
    _, image, n = P.oracle.swap_out(0)
    fill_free_blocks(P, 4, [0])
    with pytest.raises(pa.PAError) as e:
        pa.pa_swap_in(P.pool, 0, n, img)
    assert e.value.status == pa.PA_ERR_NO_BLOCKS
    assert P.oracle.swap_in(0, n, image) == Status.NO_BLOCKS
    with pytest.raises(pa.PAError) as e:
        pa.pa_swap_in(P.pool, 1, n, img)
    assert e.value.status == pa.PA_ERR_SEQ_EXISTS
    P.check_metadata()
    P.check_cache(0)
    # an empty sequence swaps an empty image, with no copy
    pa.pa_alloc_blocks(P.pool, 5, 0)
    assert P.oracle.reserve(5, 0) == Status.OK
    empty = torch.empty(0, dtype=torch.uint8, pin_memory=True)
    pa.pa_swap_out(P.pool, 5, empty)
    st, image, n = P.oracle.swap_out(5)
    assert st == Status.OK and n == 0 and image.nbytes == 0
    pa.pa_swap_in(P.pool, 5, 0, empty)
    assert P.oracle.swap_in(5, 0, image) == Status.OK
    P.check_metadata()
    assert pa.pa_launch_count(P.pool) > 0 and P.device_errors() == 0
