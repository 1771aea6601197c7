"""The no-allocation decode entry point.

pa_decode_attention_noalloc serves callers that cannot allocate device
memory -- a serving engine's plugin or custom-operator interface that keeps
every free byte of HBM for the engine's own KV pool and hands a kernel only
its input and output buffers, or a process under a hard memory cap -- and so
cannot give the library a pool workspace.  It takes the caller's device block
tables and host lengths and keeps its split-KV scratch in a static device
array.  These tests check, on two calls in a row (the second reuses the
scratch the first left behind):

* its output against the oracle, within the tolerance every parity test uses
  (1e-2 absolute + 1e-2 relative for 16-bit KV, 5e-2 for FP8 KV), and against
  pa_decode_attention's on the same cache, for query groups 1, 2, 4 and 8 and
  bf16 / FP8 caches;
* a call with the full 512 sequences, enough work that every decode worker
  of the GPU takes part;
* a corrupt block-table entry: read as block 0 with no fault and reported by
  pa_noalloc_check_errors, which also clears the bits;
* more sequences than the scratch holds: refused on the host.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle.numerics import bits_to_f64
from paged_harness import Pair, TOL, assert_close, from_dev, to_dev
from workloads import Purpose, rng, step_q_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()
    assert torch.cuda.is_available()
    pa.pa_noalloc_check_errors(0)  # start from a clear error word


def device_tables(p, seqs):
    mbps = p.w.max_blocks_per_seq
    tables = np.zeros((len(seqs), mbps), np.int32)
    lens = []
    for i, s in enumerate(seqs):
        n, tab = pa.pa_get_seq(p.pool, s)
        tables[i, : len(tab)] = tab
        lens.append(n)
    return torch.from_numpy(tables).cuda(), lens


def run_twice(p, seqs, q_bits, tables, lens):
    """Two no-allocation calls; returns the first output's bits after
    checking that the second is bit-identical."""
    w = p.w
    q = to_dev(q_bits, w.act_dtype)
    outs = []
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_attention_noalloc(p.pool.desc, 0, tables, lens, q, out, w.scale)
        torch.cuda.synchronize()
        outs.append(from_dev(out))
    assert np.array_equal(outs[0], outs[1])
    return outs[0]


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("kv", ["bf16", "fp8_e4m3"])
def test_noalloc_matches_oracle_and_pool_entry_point_twice(kv, G):
    w = dataclasses.replace(workload("gqa8b", num_seqs=24, steps=1), num_q_heads=8 * G,
                            kv_dtype=kv)
    p = Pair(w)
    p.prefill()
    seqs = list(w.seq_ids)
    q_bits = step_q_bits(w, 0, 0)
    _, ref_dev = p.decode(0, 0, seqs, 0, q_bits=q_bits)
    ref_pool = bits_to_f64(from_dev(ref_dev), w.act_dtype)
    tables, lens = device_tables(p, seqs)
    got = bits_to_f64(run_twice(p, seqs, q_bits, tables, lens), w.act_dtype)
    assert_close(got, p.oracle_attention(0, seqs, q_bits), kv, "no-allocation vs oracle")
    assert_close(got, ref_pool, kv, "no-allocation vs pa_decode_attention")
    assert pa.pa_noalloc_check_errors(0) == 0
    assert p.device_errors() == 0


def test_noalloc_full_512_sequences():
    """512 sequences of 1..600 tokens, 2 KV heads, G = 4: the work spans every
    decode worker the GPU holds, so the scratch's slot and counter arrays are
    used up to the worker capacity."""
    n = 512
    lens0 = rng(0, 12, Purpose.LENS).integers(1, 601, size=n)
    need = int(sum((int(m) + 15) // 16 for m in lens0))
    w = dataclasses.replace(workload("tiny"), name="noalloc512", cfg=12, num_blocks=need + 64,
                            max_seqs=n, max_blocks_per_seq=40, seq_ids=tuple(range(n)),
                            prefill_lens={i: int(m) for i, m in enumerate(lens0)})
    p = Pair(w)
    p.prefill()
    seqs = list(w.seq_ids)
    q_bits = step_q_bits(w, 0, 0)
    tables, lens = device_tables(p, seqs)
    got = bits_to_f64(run_twice(p, seqs, q_bits, tables, lens), w.act_dtype)
    assert_close(got, p.oracle_attention(0, seqs, q_bits), w.kv_dtype, "no-allocation, 512 sequences")
    assert pa.pa_noalloc_check_errors(0) == 0


def test_noalloc_reports_a_corrupt_table_entry():
    w = workload("tiny")
    p = Pair(w)
    p.prefill()
    seqs = list(w.seq_ids)
    q_bits = step_q_bits(w, 0, 0)
    tables, lens = device_tables(p, seqs)
    bad = tables.clone()
    bad[2, 3] = w.num_blocks + 5            # sequence 2 (103 tokens), its 4th block
    out = torch.full_like(to_dev(q_bits, w.act_dtype), float("nan"))
    pa.pa_decode_attention_noalloc(p.pool.desc, 0, bad, lens, to_dev(q_bits, w.act_dtype), out,
                                   w.scale)
    torch.cuda.synchronize()
    got = bits_to_f64(from_dev(out), w.act_dtype)
    assert np.isfinite(got).all()           # the bad id was read as block 0, nothing faulted
    ref = p.oracle_attention(0, seqs, q_bits)
    keep = [0, 1, 3]                        # the other sequences are untouched
    assert_close(got[keep], ref[keep], w.kv_dtype, "sequences with valid tables")
    bits = pa.pa_noalloc_check_errors(0)
    assert bits & pa.PA_DEVERR_BAD_BLOCK
    assert pa.pa_noalloc_check_errors(0) == 0   # read clears the word
    # a clean call afterwards reports nothing and matches the oracle
    got = bits_to_f64(run_twice(p, seqs, q_bits, tables, lens), w.act_dtype)
    assert_close(got, ref, w.kv_dtype, "after the corrupt call")
    assert pa.pa_noalloc_check_errors(0) == 0


def test_noalloc_rejects_more_sequences_than_its_scratch_holds():
    w = workload("tiny")
    p = Pair(w, oracle_seqs=[])
    p.prefill()
    n = 513
    lens = (ctypes.c_int32 * n)(*([1] * n))
    q = torch.zeros((1, w.num_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    tab = torch.zeros((1, w.max_blocks_per_seq), dtype=torch.int32, device="cuda")
    st = pa.lib().pa_decode_attention_noalloc(
        ctypes.byref(p.pool.desc), 0, n, ctypes.c_void_p(tab.data_ptr()), lens, w.num_q_heads,
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(q.data_ptr()), ctypes.c_float(w.scale), None)
    assert st == pa.PA_ERR_INVALID_ARG
    assert "512" in pa.pa_last_error()
    assert TOL["bf16"] == (1e-2, 1e-2)
