"""Pools of 32-token blocks ("Managing the KV Cache", Deliberately Broken Cases
and Answer Key: the block size is an engine and kernel choice, 16 is not
universal).  The block manager, the append, copy-on-write, swapping and the
decode take block_size 32 (the decode kernel reads a 32-token block as its two
16-token halves through the same table entry).  Tables, counts and every valid
cache slot are compared bit-exact with the oracle at block size 32, attention
within the stated tolerance, in every split mode, with the fused append and
with forks whose shared prompt is read once."""
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
    p = Pair(w, min_partition=32)
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
    # decode every sequence (4 shares 1's blocks up to the copied tail)
    seqs = [0, 1, 2, 3, 4]
    q_bits = normal_bits(g, (len(seqs), w.num_q_heads, w.head_dim), w.act_dtype)
    for part in (0, -1, 32):
        q, out = p.decode(0, 0, seqs, part, q_bits=q_bits)
        p.check_attention(0, seqs, q, out)
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


LENS32 = [1, 15, 16, 17, 31, 32, 33, 48, 63, 64, 65, 100, 511, 513]


def ragged32(G, kv):
    act = "fp16" if kv == "fp16" else "bf16"
    n = len(LENS32)
    return dataclasses.replace(
        workload("tiny"), name="ragged32", cfg=10, block_size=32, num_kv_heads=2,
        num_q_heads=2 * G, kv_dtype=kv, act_dtype=act, num_blocks=96, max_seqs=n,
        max_blocks_per_seq=20, seq_ids=tuple(range(n)),
        prefill_lens={i: m for i, m in enumerate(LENS32)}, steps=2)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("kv", ["bf16", "fp16", "fp8_e4m3"])
def test_block32_decode_ragged_lengths(G, kv):
    """Lengths on both sides of every 16- and 32-token boundary, all split
    modes, then the next step's append fused into the decode."""
    w = ragged32(G, kv)
    p = Pair(w, min_partition=32)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    p.check_cache(0)
    for part in (0, -1, 32, 64):
        q, out = p.decode(0, 0, seqs, part)
        p.check_attention(0, seqs, q, out)
    seqs, pos = p.reserve_step(1)
    q, out = p.append_decode(1, 0, seqs, pos, 0)
    p.check_metadata()
    p.check_cache(0)
    p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


@pytest.mark.parametrize("G", [1, 2, 4])
def test_block32_forks_read_their_prompt_once(G):
    """A 300-token prompt (9 full 32-token blocks + 12 tokens) forked into
    8 / G samples: the shared blocks form sibling sets; two steps grow the
    samples (copy-on-write of the shared tail on the first)."""
    members = 8 // G
    seqs = tuple(range(members + 2))
    lens = {0: 300, members: 45, members + 1: 700}
    forks = tuple((0, c) for c in range(1, members))
    w = dataclasses.replace(
        workload("tiny"), name="family32", cfg=11, block_size=32, num_kv_heads=2,
        num_q_heads=2 * G, num_blocks=80, max_seqs=len(seqs), max_blocks_per_seq=30,
        seq_ids=seqs, prefill_lens=lens, forks=forks, steps=2)
    p = Pair(w, min_partition=32)
    p.prefill()
    for step in (0, 1):
        seqs_, pos = p.reserve_step(step)
        q, out = p.append_decode(step, 0, seqs_, pos, 0)
        sets, _ = pa.pa_last_decode_plan(p.pool)
        assert sets >= 1
        p.check_metadata()
        p.check_cache(0)
        p.check_attention(0, seqs_, q, out)
    assert len(p.oracle.cow_log) == members - 1
    assert p.device_errors() == 0
