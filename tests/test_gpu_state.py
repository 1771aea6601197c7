"""Resume from a host state checkpoint on the GPU.

Pool A prefills and decodes; its host state image is loaded into pool B,
created over A's own cache buffers (the KV cache is the caller's memory).
B's device copy of the block tables is rewritten from the image with its
first launch, so B must decode exactly as A does, bit for bit, in every split
mode, and both must match the oracle; then both take the next step (the
append fused into the decode) and still agree.  ("kv-cache-pagedattention-
serving", PagedAttention: virtual memory for GPUs: attention over the blocks
through the table.)
"""
import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from paged_harness import Pair, from_dev, to_dev
from test_gpu_siblings import family_workload
from workloads import step_kv_bits, step_q_bits, workload

pytestmark = pytest.mark.gpu


def twin(p):
    """A second pool over p's cache buffers, restored from p's state image."""
    pool = p.pool
    b = pa.pa_pool_create(num_layers=pool.num_layers, num_kv_heads=pool.num_kv_heads,
                          block_size=pool.block_size, num_blocks=pool.num_blocks,
                          max_seqs=pool.max_seqs, max_blocks_per_seq=pool.max_blocks_per_seq,
                          kv_dtype=pool.kv_dtype, act_dtype=pool.act_dtype,
                          k_cache=pool.k_cache, v_cache=pool.v_cache,
                          k_scale=pool.scales[0], v_scale=pool.scales[1],
                          k_inv_scale=pool.scales[2], v_inv_scale=pool.scales[3])
    pa.pa_state_load(b, pa.pa_state_save(pool))
    return b


def case(name):
    if name == "fp8_family":   # FP8 scales carried over; forks, sibling sets, a lone sequence
        return family_workload(4, "fp8_e4m3", [(203, 3)], [300], steps=2)
    return workload(name, steps=2)


@pytest.mark.parametrize("name", ["tiny", "mha7b_share", "fp8_family"])
def test_restored_pool_decodes_like_the_saved_one(name):
    w = case(name)
    layers = [0] if w.num_layers > 1 else None
    p = Pair(w, layers=layers) if layers else Pair(w)
    if layers:
        p.prefill(gpu_layers=layers)
    else:
        p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    b = twin(p)
    assert pa.pa_get_free_list(b) == pa.pa_get_free_list(p.pool)
    assert pa.pa_get_refcounts(b) == pa.pa_get_refcounts(p.pool)
    for part in (0, -1, 512):
        q_bits, out_a = p.decode(0, 0, seqs, part)
        q = to_dev(q_bits, w.act_dtype)
        out_b = torch.empty_like(q)
        pa.pa_decode_attention(b, 0, seqs, q, out_b, w.scale, part)
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out_a), from_dev(out_b)), part
        p.check_attention(0, seqs, q_bits, out_a)
    # the next step on both pools: the same reservations, the append fused
    # into the decode (A writes the rows; B's call writes the same values)
    seqs, pos = p.reserve_step(1)
    lens = [int(x) + 1 for x in pos]
    pa.pa_alloc_blocks_n(b, seqs, lens)
    assert pa.pa_get_free_list(b) == pa.pa_get_free_list(p.pool)
    for s in seqs:
        assert pa.pa_get_seq(b, s) == pa.pa_get_seq(p.pool, s)
    q_bits, out_a = p.append_decode(1, 0, seqs, pos, 0)
    k, v = step_kv_bits(w, 1, 0)
    q = to_dev(step_q_bits(w, 1, 0), w.act_dtype)
    out_b = torch.empty_like(q)
    pa.pa_decode_attention_append(b, 0, seqs, to_dev(k, w.act_dtype), to_dev(v, w.act_dtype), q,
                                  out_b, w.scale, 0)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(out_a), from_dev(out_b))
    p.check_cache(0)
    p.check_attention(0, seqs, q_bits, out_a)
    assert p.device_errors() == 0
    assert pa.pa_check_device_errors(b) == 0
