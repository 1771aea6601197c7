"""The no-allocation decode entry point against the pool-based one.

pa_decode_attention_noalloc serves callers that cannot allocate device
memory (a host engine that keeps all HBM for itself and hands a kernel only
its input and output buffers): it takes the caller's device block tables and
host lengths and keeps its split-KV scratch in a static device array.  Its
output must match pa_decode_attention's on the same cache, within the
tolerance the other tests use (1e-2), on two calls in a row (the second call
reuses the scratch the first one left behind).

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from paged_harness import Pair, from_dev, to_dev
from oracle.numerics import bits_to_f64
from workloads import step_q_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()
    assert torch.cuda.is_available()


def test_noalloc_matches_pool_entry_point_twice():
    w = workload("gqa8b", num_seqs=24, steps=1)
    p = Pair(w, oracle_seqs=[])
    p.prefill()
    seqs = list(w.seq_ids)
    q_bits = step_q_bits(w, 0, 0)
    _, ref = p.decode(0, 0, seqs, 0, q_bits=q_bits)
    q = to_dev(q_bits, w.act_dtype)
    torch.cuda.synchronize()

    mbps = w.max_blocks_per_seq
    tables = np.zeros((len(seqs), mbps), np.int32)
    lens = []
    for i, s in enumerate(seqs):
        n, tab = pa.pa_get_seq(p.pool, s)
        tables[i, : len(tab)] = tab
        lens.append(n)
    dtab = torch.from_numpy(tables).cuda()
    ref_f = bits_to_f64(from_dev(ref), w.act_dtype)
    outs = []
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_attention_noalloc(p.pool.desc, 0, dtab, lens, q, out, w.scale)
        torch.cuda.synchronize()
        got = bits_to_f64(from_dev(out), w.act_dtype)
        assert np.isfinite(got).all()
        assert np.abs(got - ref_f).max() <= 1e-2
        outs.append(from_dev(out))
    assert np.array_equal(outs[0], outs[1])


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
