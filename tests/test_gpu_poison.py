"""Stale slot contents never reach the output.

Only a sequence's last block may be partly filled ("Managing the KV Cache",
Internal Fragmentation): the slots past its length hold whatever an earlier
owner of the block left there.  The decode masks those slots, so their bits --
here NaN in every dtype -- must not leak into any output, in any split mode.

The byte 0xFF is a NaN in each storage format: bf16 0xFFFF and fp16 0xFFFF
have an all-ones exponent and a non-zero fraction, E4M3 0xFF is S.1111.111.
The pool (and the workspace, whose contents the header says need no
initialisation) is filled with it before the prefill, and blocks released by
finished sequences are filled with it again before new sequences take them.
Lengths sit on both sides of block (16-token) and 512-token partition
boundaries, exact multiples of 16 included.  Every output must be finite and
match the oracle; cache contents of valid slots stay bit-exact.

Also: outputs are bit-identical under another physical placement of the
blocks at the full 8B-class size (64 sequences of 128..4096 tokens)
("kv-cache-pagedattention-serving", PagedAttention: blocks may sit anywhere
in GPU memory).
"""
import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle import Status
from paged_harness import Pair, from_dev
from workloads import Purpose, normal_bits, rng, workload

pytestmark = pytest.mark.gpu

# lengths after the first step's append
FINAL = [2, 16, 17, 32, 48, 511, 512, 513, 1024, 1025, 528, 496, 15, 1023]
# lengths of the sequences that take the released blocks
REFILL = [31, 512, 64, 3, 257, 1008]
NAN_BYTE = 0xFF


def poison(t: torch.Tensor):
    t.view(torch.uint8).fill_(NAN_BYTE)


def poisoned_pair(G, kv):
    act = "fp16" if kv == "fp16" else "bf16"
    n = len(FINAL) + len(REFILL)
    w = dataclasses.replace(
        workload("tiny"), name="poison", cfg=13, num_kv_heads=2, num_q_heads=2 * G, kv_dtype=kv,
        act_dtype=act, num_blocks=sum(-(-m // 16) for m in FINAL) + 8,
        max_seqs=n, max_blocks_per_seq=70, seq_ids=tuple(range(len(FINAL))),
        prefill_lens={i: m - 1 for i, m in enumerate(FINAL)}, steps=2)
    p = Pair(w, min_partition=16)
    poison(p.pool.k_cache)
    poison(p.pool.v_cache)
    poison(p.pool.workspace)
    return w, p


def decode_all_modes(p, step, seqs):
    for part in (0, -1, 16, 512):
        q, out = p.decode(step, 0, seqs, part)
        p.check_attention(0, seqs, q, out)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("kv", ["bf16", "fp16", "fp8_e4m3"])
def test_nan_in_stale_slots_never_leaks(G, kv):
    w, p = poisoned_pair(G, kv)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    p.check_cache(0)
    decode_all_modes(p, 0, seqs)
    # release every other sequence, fill the released blocks with NaN, and
    # start new sequences in them (8 blocks were never used: the rest of the
    # new sequences' blocks are released ones)
    freed = seqs[::2]
    for s in freed:
        pa.pa_free(p.pool, s)
        assert p.oracle.release(s) is Status.OK
    free = torch.tensor(pa.pa_get_free_list(p.pool), dtype=torch.int64, device="cuda")
    p.pool.k_cache.view(torch.uint8)[:, free] = NAN_BYTE
    p.pool.v_cache.view(torch.uint8)[:, free] = NAN_BYTE
    g = rng(w.seed, w.cfg, Purpose.MISC, G)
    new = list(range(len(FINAL), len(FINAL) + len(REFILL)))
    for s, m in zip(new, REFILL):
        pa.pa_alloc_blocks(p.pool, s, m)
        assert p.oracle.reserve(s, m) is Status.OK
        k = normal_bits(g, (m, w.num_kv_heads, 128), w.act_dtype)
        v = normal_bits(g, (m, w.num_kv_heads, 128), w.act_dtype)
        p.append(0, [s] * m, list(range(m)), k, v)
    live = [s for s in seqs if s not in freed] + new
    p.check_metadata()
    p.check_cache(0, live)
    q_bits = normal_bits(g, (len(live), w.num_q_heads, 128), w.act_dtype)
    for part in (0, -1, 16, 512):
        q, out = p.decode(1, 0, live, part, q_bits=q_bits)
        p.check_attention(0, live, q, out)
    assert p.device_errors() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp8_e4m3"])
def test_nan_in_stale_slots_fused_append(kv):
    """The fused append writes the new row into a NaN-filled slot and the
    staged tile; the slots after it stay NaN and stay masked."""
    w, p = poisoned_pair(8, kv)
    p.prefill()
    for step in (0, 1):
        seqs, pos = p.reserve_step(step)
        q, out = p.append_decode(step, 0, seqs, pos, 0)
        p.check_cache(0)
        p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


@pytest.mark.parametrize("partition", [0, -1, 512])
def test_placement_bit_identity_full_8b_class(partition):
    w = workload("gqa8b", steps=1)
    outs = []
    for seed in (0, 1):
        order = np.random.default_rng(200 + seed).permutation(w.num_blocks)
        p = Pair(w, free_order=order, oracle_seqs=[])
        p.prefill()
        seqs, pos = p.reserve_step(0)
        p.append_step(0, 0, seqs, pos)
        q, out = p.decode(0, 0, seqs, partition)
        outs.append(from_dev(out))
        assert p.device_errors() == 0
        del p
        torch.cuda.empty_cache()
    assert np.array_equal(outs[0], outs[1])
