"""The tcgen05 decode kernel (query group of 8 over a 16-bit cache).

The 80-layer model of "Managing the KV Cache" (Worked Capacity Under a 12 GiB
KV Budget) has 64 query heads over 8 KV heads: each KV tile meets 8 query rows,
a dense 8-column contraction that this kernel runs on the 5th-generation
tensor cores with tensor-memory accumulators.  Every case is compared with
the oracle ("kv-cache-pagedattention-serving", PagedAttention: attention over
the blocks through the table) within the stated tolerance, and the kernel
that ran is checked (pa_last_decode_kernel).

Lengths cover empty and full 16-token blocks and 128-token tiles on both
sides of every boundary; all split modes; the fused append; 32-token blocks;
NaN in stale slots; placement bit-identity; a corrupt table entry; the
80-layer configuration at full size on sampled layers.
"""
import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from paged_harness import Pair, assert_close, from_dev
from oracle.numerics import bits_to_f64
from workloads import step_q_bits, workload

pytestmark = pytest.mark.gpu

LENS = [1, 2, 15, 16, 17, 127, 128, 129, 255, 256, 257, 600, 1000, 2049]


def group8(kv="bf16", block=16, lens=LENS, cfg=20):
    act = "fp16" if kv == "fp16" else "bf16"
    n = len(lens)
    return dataclasses.replace(
        workload("tiny"), name="tc8", cfg=cfg, num_kv_heads=3, num_q_heads=24, kv_dtype=kv,
        act_dtype=act, block_size=block,
        num_blocks=sum(-(-(m + 2) // block) for m in lens) + 16, max_seqs=n,
        max_blocks_per_seq=-(-(max(lens) + 2) // block) + 1, seq_ids=tuple(range(n)),
        prefill_lens={i: m - 1 if m > 1 else 1 for i, m in enumerate(lens)}, steps=2)


def tc_pair(w, **kw):
    p = Pair(w, min_partition=max(16, w.block_size), **kw)
    pa.pa_set_decode_path(p.pool, "tcgen05")
    return p


@pytest.mark.parametrize("kv", ["bf16", "fp16"])
def test_tcgen05_ragged_lengths_all_modes(kv):
    w = group8(kv)
    p = tc_pair(w)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    for part in (0, -1, 16, 128, 512):
        q, out = p.decode(0, 0, seqs, part)
        assert pa.pa_last_decode_kernel(p.pool) == "tcgen05"
        p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp16"])
def test_tcgen05_matches_warp_kernel(kv):
    w = group8(kv, cfg=21)
    p = tc_pair(w)
    p.prefill()
    seqs = list(w.seq_ids)
    q_bits = step_q_bits(w, 0, 0)
    _, a = p.decode(0, 0, seqs, 0, q_bits=q_bits)
    pa.pa_set_decode_path(p.pool, "warp")
    _, b = p.decode(0, 0, seqs, 0, q_bits=q_bits)
    assert pa.pa_last_decode_kernel(p.pool) == "warp"
    assert_close(bits_to_f64(from_dev(a), w.act_dtype), bits_to_f64(from_dev(b), w.act_dtype), kv,
                 "tcgen05 vs warp-level kernel")


@pytest.mark.parametrize("kv", ["bf16", "fp16"])
def test_tcgen05_fused_append(kv):
    w = group8(kv, cfg=22)
    p = tc_pair(w)
    p.prefill()
    for step in (0, 1):
        seqs, pos = p.reserve_step(step)
        q, out = p.append_decode(step, 0, seqs, pos, 0)
        assert pa.pa_last_decode_kernel(p.pool) == "tcgen05"
        p.check_metadata()
        p.check_cache(0)
        p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_tcgen05_block32():
    w = group8("bf16", block=32, cfg=23)
    p = tc_pair(w)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    for part in (0, -1, 32, 512):
        q, out = p.decode(0, 0, seqs, part)
        p.check_attention(0, seqs, q, out)
    seqs, pos = p.reserve_step(1)
    q, out = p.append_decode(1, 0, seqs, pos, 0)
    p.check_cache(0)
    p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_tcgen05_nan_in_stale_slots():
    w = group8("bf16", cfg=24)
    p = tc_pair(w)
    for t in (p.pool.k_cache, p.pool.v_cache, p.pool.workspace):
        t.view(torch.uint8).fill_(0xFF)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    for part in (0, -1, 128):
        q, out = p.decode(0, 0, seqs, part)
        p.check_attention(0, seqs, q, out)
    seqs, pos = p.reserve_step(1)
    q, out = p.append_decode(1, 0, seqs, pos, 0)
    p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_tcgen05_placement_bit_identity():
    w = group8("bf16", cfg=25)
    outs = []
    for seed in (0, 1):
        order = np.random.default_rng(300 + seed).permutation(w.num_blocks)
        p = tc_pair(w, free_order=order, oracle_seqs=[])
        p.prefill()
        q, out = p.decode(0, 0, list(w.seq_ids), 0)
        outs.append(from_dev(out))
    assert np.array_equal(outs[0], outs[1])


def test_tcgen05_corrupt_table_entry_is_reported():
    w = group8("bf16", cfg=26)
    p = tc_pair(w, oracle_seqs=[])
    p.prefill()
    seqs = list(w.seq_ids)
    # sequence 12 (1000 tokens): one entry of the device mirror points outside the pool
    meta = p.pool.workspace[256:].view(torch.int32)
    meta[12 * w.max_blocks_per_seq + 5] = w.num_blocks + 5
    q, out = p.decode(0, 0, seqs, 0)
    torch.cuda.synchronize()
    assert np.isfinite(bits_to_f64(from_dev(out), w.act_dtype)).all()
    assert p.device_errors() & pa.PA_DEVERR_BAD_BLOCK


def test_tcgen05_gqa70b_full_size_sampled_layers():
    """The 80-layer configuration at full size (47 sequences of 825 tokens,
    the 2,457 + 34-block pool), two of its layers written and decoded, the
    step's append fused; every output checked."""
    w = workload("gqa70b_headroom", steps=2)
    p = tc_pair(w, layers=[0, 79])
    p.prefill(gpu_layers=[0, 79])
    for step in (0, 1):
        seqs, pos = p.reserve_step(step)
        for layer in (0, 79):
            q, out = p.append_decode(step, layer, seqs, pos, 0)
            assert pa.pa_last_decode_kernel(p.pool) == "tcgen05"
            p.check_cache(layer)
            p.check_attention(layer, seqs, q, out)
    assert p.device_errors() == 0
