"""Pools of 32-token blocks ("Managing the KV Cache", Deliberately Broken Cases
and Answer Key: the block size is an engine and kernel choice, 16 is not
universal).  The block manager, the append, copy-on-write and swapping take
block_size 32; the decode kernel takes 16 only and refuses 32 on the host
with nothing launched.  Tables, counts and every valid cache slot are compared
bit-exact with the oracle at block size 32."""
import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle import Status
from paged_harness import Pair
from workloads import Purpose, normal_bits, rng, workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv", ["bf16", "fp8_e4m3"])
def test_block32_append_cow_swap(kv):
    w = dataclasses.replace(workload("tiny"), block_size=32, kv_dtype=kv, max_seqs=6,
                            max_blocks_per_seq=40, num_blocks=96)
    p = Pair(w)
    p.prefill()
    p.check_metadata()
    p.check_cache(0)
    # a step for every sequence: 825 -> 826 crosses nothing, 16 -> 17 stays in block 0
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    # fork sequence 1 (201 tokens) into 4; both grow into the shared 9-token tail
    pa.pa_fork_cow(p.pool, 1, 4)
    assert p.oracle.fork(1, 4) == Status.OK
    g = rng(w.seed, 32, Purpose.MISC)
    for s in (4, 1):
        n = p.oracle.lens[s]
        pa.pa_alloc_blocks(p.pool, s, n + 1)
        assert p.oracle.reserve(s, n + 1) == Status.OK
        k = normal_bits(g, (1, w.num_kv_heads, w.head_dim), w.act_dtype)
        v = normal_bits(g, (1, w.num_kv_heads, w.head_dim), w.act_dtype)
        p.append(0, [s], [n], k, v)
    assert len(p.oracle.cow_log) == 1                        # 201 % 32 != 0: one copy
    p.check_metadata()
    p.check_cache(0)
    # the decode kernel takes block_size 16 only: refused, nothing launched
    before = pa.pa_launch_count(p.pool)
    q = torch.zeros((1, w.num_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_attention(p.pool, 0, [0], q, torch.empty_like(q), w.scale)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert pa.pa_launch_count(p.pool) == before
    # swap sequence 0 out and back: whole 32-token blocks
    n0 = p.oracle.lens[0]
    img = torch.empty(pa.pa_swap_bytes(p.pool, n0), dtype=torch.uint8, pin_memory=True)
    pa.pa_swap_out(p.pool, 0, img)
    st, image, n = p.oracle.swap_out(0)
    assert st == Status.OK and img.numel() == image.nbytes
    torch.cuda.synchronize()
    got = img.numpy().view(image.dtype).reshape(image.shape)
    for j in range(image.shape[1]):
        m = min(32, n - 32 * j)
        assert np.array_equal(got[:, j, :, :, :m, :], image[:, j, :, :, :m, :]), j
    pa.pa_swap_in(p.pool, 0, n, img)
    assert p.oracle.swap_in(0, n, image) == Status.OK
    p.check_metadata()
    p.check_cache(0)
    assert p.device_errors() == 0
