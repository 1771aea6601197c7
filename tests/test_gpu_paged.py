"""GPU parity tests: the CUDA path (through the C ABI) against the oracle.

Metadata and cache contents bit-exact; attention within the stated
tolerance (1e-2 absolute + 1e-2 relative for 16-bit KV, 5e-2 absolute for FP8 KV).  Marked `gpu`.
"""
import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from oracle import PagedKVOracle, Status, fp8
from paged_harness import Pair, assert_close, from_dev, to_dev
from workloads import normal_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("partition", [0, -1, 16])
def test_tiny_workload_end_to_end(partition):
    w = workload("tiny")
    p = Pair(w, min_partition=16)
    p.prefill()
    p.check_metadata()
    p.check_cache(0)
    seqs, pos = p.reserve_step(0)
    p.check_metadata()
    p.append_step(0, 0, seqs, pos)
    p.check_cache(0)
    q, out = p.decode(0, 0, seqs, partition)
    p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_tiny_partition_modes_agree_closely():
    w = workload("tiny")
    p = Pair(w, min_partition=16)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    outs = [p.decode(0, 0, seqs, part)[1].float() for part in (0, -1, 16, 512)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 1e-2


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("kv", ["bf16", "fp16"])
def test_groups_and_ragged_lengths(G, kv):
    """Lengths 1..70 cover empty tails, full blocks and several tiles."""
    H = 2
    lens = [1, 2, 15, 16, 17, 31, 32, 33, 47, 64, 70, 5]
    g = np.random.default_rng(G)
    nb = 80
    order = g.permutation(nb)
    pool = pa.pa_pool_create(num_layers=2, num_kv_heads=H, block_size=16, num_blocks=nb,
                             max_seqs=len(lens), max_blocks_per_seq=8, kv_dtype=kv,
                             free_order=order, min_partition_tokens=16)
    o = PagedKVOracle(num_layers=2, num_kv_heads=H, head_dim=128, block_size=16, num_blocks=nb,
                      max_seqs=len(lens), max_blocks_per_seq=8, kv_dtype=kv, free_order=order)
    for s, n in enumerate(lens):
        pa.pa_alloc_blocks(pool, s, n)
        assert o.reserve(s, n) is Status.OK
        for layer in (0, 1):
            k = normal_bits(g, (n, H, 128), kv)
            v = normal_bits(g, (n, H, 128), kv)
            pa.pa_append_kv(pool, layer, [s] * n, list(range(n)), to_dev(k, kv), to_dev(v, kv))
            assert o.append(layer, [s] * n, list(range(n)), k, v, kv) is Status.OK
    seqs = list(range(len(lens)))
    q_bits = normal_bits(g, (len(lens), H * G, 128), kv)
    q = to_dev(q_bits, kv)
    for layer in (0, 1):
        ref = o.attention(layer, seqs, q_bits, kv, 0.0883883461356163)
        for part in (0, -1, 16, 32):
            out = torch.empty_like(q)
            pa.pa_decode_attention(pool, layer, seqs, q, out, 0.0883883461356163, part)
            from oracle.numerics import bits_to_f64
            assert_close(bits_to_f64(from_dev(out), kv), ref, kv, f"layer {layer}, partition {part}")
    assert pa.pa_check_device_errors(pool) == 0


def test_single_token_output_is_the_value_row_exactly():
    H, G = 2, 4
    pool = pa.pa_pool_create(num_layers=1, num_kv_heads=H, block_size=16, num_blocks=8,
                             max_seqs=3, max_blocks_per_seq=2, kv_dtype="bf16")
    g = np.random.default_rng(3)
    vbits = []
    for s in range(3):
        pa.pa_alloc_blocks(pool, s, 1)
        k = normal_bits(g, (1, H, 128), "bf16")
        v = normal_bits(g, (1, H, 128), "bf16")
        vbits.append(v)
        pa.pa_append_kv(pool, 0, [s], [0], to_dev(k, "bf16"), to_dev(v, "bf16"))
    q = to_dev(normal_bits(g, (3, H * G, 128), "bf16"), "bf16")
    for part in (0, -1):
        out = torch.empty_like(q)
        pa.pa_decode_attention(pool, 0, [0, 1, 2], q, out, 0.088, part)
        got = from_dev(out)
        for s in range(3):
            for qh in range(H * G):
                assert np.array_equal(got[s, qh], vbits[s][0, qh // G])


def test_identical_keys_and_constant_values():
    H, G, n = 1, 8, 300
    pool = pa.pa_pool_create(num_layers=1, num_kv_heads=H, block_size=16, num_blocks=40,
                             max_seqs=2, max_blocks_per_seq=20, kv_dtype="bf16")
    g = np.random.default_rng(4)
    krow = normal_bits(g, (1, H, 128), "bf16")
    k = np.repeat(krow, n, axis=0)
    v = normal_bits(g, (n, H, 128), "bf16")
    pa.pa_alloc_blocks(pool, 0, n)
    pa.pa_append_kv(pool, 0, [0] * n, list(range(n)), to_dev(k, "bf16"), to_dev(v, "bf16"))
    c = np.full((n, H, 128), 0x3FC0, np.uint16)  # bf16 1.5
    pa.pa_alloc_blocks(pool, 1, n)
    pa.pa_append_kv(pool, 0, [1] * n, list(range(n)), to_dev(v, "bf16"), to_dev(c, "bf16"))
    q = to_dev(normal_bits(g, (2, H * G, 128), "bf16"), "bf16")
    out = torch.empty_like(q)
    pa.pa_decode_attention(pool, 0, [0, 1], q, out, 0.088, 0)
    from oracle.numerics import bits_to_f64
    mean_v = bits_to_f64(v, "bf16")[:, 0].mean(axis=0)
    got = bits_to_f64(from_dev(out), "bf16")
    assert_close(got[0], mean_v, "bf16", "identical keys")
    assert np.array_equal(from_dev(out)[1], np.full((H * G, 128), 0x3FC0, np.uint16))


@pytest.mark.parametrize("partition", [0, -1, 32])
def test_placement_invariance_bit_identical(partition):
    w = workload("tiny")
    outs = []
    for seed in (0, 1):
        order = np.random.default_rng(100 + seed).permutation(w.num_blocks)
        p = Pair(w, free_order=order, min_partition=16)
        p.prefill()
        seqs, pos = p.reserve_step(0)
        p.append_step(0, 0, seqs, pos)
        q, out = p.decode(0, 0, seqs, partition)
        outs.append(from_dev(out))
        assert pa.pa_get_seq(p.pool, 0)[1] != [] and p.device_errors() == 0
    assert np.array_equal(outs[0], outs[1])


def test_append_fp8_encoder_exhaustive():
    """All 65,536 bf16 patterns x several scales through the append kernel."""
    H = 1
    T = 512  # 512 rows x 128 = 65,536 values
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(T, H, 128)
    for inv in (1.0, 1 / 0.37, 448.0 / 4.0, 2.0 ** -5):
        inv32 = np.array([[inv]], np.float32)
        scale = (np.float32(1) / inv32).astype(np.float32)
        dev = [torch.from_numpy(a).cuda() for a in (scale, scale, inv32, inv32)]
        pool = pa.pa_pool_create(num_layers=1, num_kv_heads=H, block_size=16, num_blocks=T // 16,
                                 max_seqs=1, max_blocks_per_seq=T // 16, kv_dtype="fp8_e4m3",
                                 act_dtype="bf16", k_scale=dev[0], v_scale=dev[1],
                                 k_inv_scale=dev[2], v_inv_scale=dev[3])
        pa.pa_alloc_blocks(pool, 0, T)
        pa.pa_append_kv(pool, 0, [0] * T, list(range(T)), to_dev(bits, "bf16"), to_dev(bits, "bf16"))
        _, table = pa.pa_get_seq(pool, 0)
        t = np.arange(T)
        blk = torch.from_numpy(np.asarray(table, np.int64)[t // 16]).cuda()
        got = pool.k_cache[0][blk, :, torch.from_numpy(t % 16).cuda(), :].cpu().numpy()
        x = (bits.astype(np.uint32) << 16).view(np.float32)
        want = fp8.quantize(x, inv32[0, 0])
        nan = fp8.is_nan_code(want)
        assert fp8.is_nan_code(got[nan]).all()
        assert np.array_equal(got[~nan], want[~nan]), inv


def test_append_fp16_bit_exact_and_cow_copies_all_layers():
    g = np.random.default_rng(21)
    L, H, n = 3, 4, 37
    order = g.permutation(12)
    pool = pa.pa_pool_create(num_layers=L, num_kv_heads=H, block_size=16, num_blocks=12,
                             max_seqs=3, max_blocks_per_seq=4, kv_dtype="fp16", free_order=order)
    o = PagedKVOracle(num_layers=L, num_kv_heads=H, head_dim=128, block_size=16, num_blocks=12,
                      max_seqs=3, max_blocks_per_seq=4, kv_dtype="fp16", free_order=order)
    pa.pa_alloc_blocks(pool, 0, n)
    assert o.reserve(0, n) is Status.OK
    for layer in range(L):
        k = normal_bits(g, (n, H, 128), "fp16")
        v = normal_bits(g, (n, H, 128), "fp16")
        pa.pa_append_kv(pool, layer, [0] * n, list(range(n)), to_dev(k, "fp16"), to_dev(v, "fp16"))
        assert o.append(layer, [0] * n, list(range(n)), k, v, "fp16") is Status.OK
    pa.pa_fork_cow(pool, 0, 1)
    assert o.fork(0, 1) is Status.OK
    pa.pa_alloc_blocks(pool, 1, n + 1)      # tail block shared and partly filled: copy
    assert o.reserve(1, n + 1) is Status.OK
    assert pa.pa_get_cow_log(pool) == o.cow_log and len(o.cow_log) == 1
    for layer in range(L):
        for s in (0, 1):
            _, tab = pa.pa_get_seq(pool, s)
            for j, b in enumerate(tab):
                assert np.array_equal(from_dev(pool.k_cache[layer, b]), o.k[layer][b]) or j * 16 >= n
        src, dst = o.cow_log[0]
        # the whole copied block matches, in every layer, K and V
        assert np.array_equal(from_dev(pool.k_cache[layer, dst]), o.k[layer][dst])
        assert np.array_equal(from_dev(pool.v_cache[layer, dst]), o.v[layer][dst])
    assert pa.pa_check_device_errors(pool) == 0


def test_gqa8b_steps_with_growth():
    """8B-class GQA layer: 64 sequences, lengths 128..4096, growth across
    block boundaries; every 10th step checked in full."""
    w = workload("gqa8b", steps=21)
    p = Pair(w)
    p.prefill()
    p.check_metadata()
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        p.append_step(step, 0, seqs, pos)
        q, out = p.decode(step, 0, seqs, 0)
        if step % 10 == 0:
            p.check_metadata()
            p.check_cache(0)
            p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_mha_sharing_cow_reduced_layers():
    """Parallel sampling n=8 over 2,050-token prompts: 28 copy-on-writes at the
    first divergent append, then growth; 4 of 32 layers compared."""
    w = workload("mha7b_share", steps=3)
    layers = [0, 13, 31]
    p = Pair(w, layers=layers)
    p.prefill(gpu_layers=layers)      # other layers stay zero: only compared layers need data
    p.check_metadata()
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        p.check_metadata()
        if step == 0:
            assert len(p.oracle.cow_log) == 28
            for layer in layers:
                p.check_cache(layer)
        for layer in range(w.num_layers):
            k, v = __import__("workloads").step_kv_bits(w, step, layer)
            p.append(layer, seqs, pos, k, v)
            q, out = p.decode(step, layer, seqs, 0)
            if layer in layers:
                p.check_cache(layer)
                p.check_attention(layer, seqs, q, out)
    assert p.device_errors() == 0


def test_gqa70b_exact_pool_overflow_then_headroom():
    w = workload("gqa70b")
    p = Pair(w, layers=[0])
    # metadata only on the exact pool: the 14th sequence cannot get block 53
    order = w.free_order()
    host = pa.pa_pool_create(num_layers=w.num_layers, num_kv_heads=w.num_kv_heads, block_size=16,
                             num_blocks=w.num_blocks, max_seqs=w.max_seqs,
                             max_blocks_per_seq=w.max_blocks_per_seq, host_only=True,
                             free_order=order)
    o = PagedKVOracle(num_layers=1, num_kv_heads=1, head_dim=1, block_size=16,
                      num_blocks=w.num_blocks, max_seqs=w.max_seqs,
                      max_blocks_per_seq=w.max_blocks_per_seq, kv_dtype="bf16", free_order=order)
    seqs = list(w.seq_ids)
    pa.pa_alloc_blocks_n(host, seqs, [825] * 47)
    for s in seqs:
        o.reserve(s, 825)
    for step in range(7):
        pa.pa_alloc_blocks_n(host, seqs, [826 + step] * 47)
        for s in seqs:
            o.reserve(s, 826 + step)
    with pytest.raises(pa.PAError) as ei:
        pa.pa_alloc_blocks_n(host, seqs, [833] * 47)
    assert ei.value.status == pa.PA_ERR_NO_BLOCKS and ei.value.n_done == 13
    for s in range(13):
        o.reserve(s, 833)
    assert o.reserve(13, 833) is Status.NO_BLOCKS
    assert pa.pa_get_free_list(host) == o.free_list() == []
    del p


def test_bad_block_id_is_caught_by_the_kernel_check():
    w = workload("tiny")
    p = Pair(w)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    p.decode(0, 0, seqs, 0)
    assert p.device_errors() == 0
    # corrupt one entry of the device copy of seq 1's block table
    mbps = w.max_blocks_per_seq
    meta = p.pool.workspace[256:].view(torch.int32)
    meta[1 * mbps + 3] = w.num_blocks + 5
    p.decode(0, 0, seqs, 0)
    assert p.device_errors() & pa.PA_DEVERR_BAD_BLOCK
    assert p.device_errors() == 0


def test_errors_leave_state_unchanged():
    w = workload("tiny")
    p = Pair(w)
    p.prefill()
    before = (pa.pa_get_free_list(p.pool), pa.pa_get_refcounts(p.pool))
    with pytest.raises(pa.PAError) as ei:
        pa.pa_alloc_blocks(p.pool, 0, 100000)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PAError) as ei:
        pa.pa_append_kv(p.pool, 0, [0], [900], to_dev(np.zeros((1, 2, 128), np.uint16), "bf16"),
                        to_dev(np.zeros((1, 2, 128), np.uint16), "bf16"))
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    q = torch.zeros((1, 6, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PAError):
        pa.pa_decode_attention(p.pool, 0, [0], q, torch.empty_like(q), 0.1)   # G = 3
    assert before == (pa.pa_get_free_list(p.pool), pa.pa_get_refcounts(p.pool))


def test_empty_calls_launch_nothing_and_change_nothing():
    """Zero sequences or tokens: every call succeeds, launches no kernel and
    leaves tables, counts, free list and cache as they were."""
    w = workload("tiny")
    p = Pair(w)
    p.prefill()
    before = (pa.pa_get_free_list(p.pool), pa.pa_get_refcounts(p.pool), pa.pa_launch_count(p.pool))
    q = torch.zeros((0, 8, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    for part in (0, -1, 512):
        pa.pa_decode_attention(p.pool, 0, [], q, torch.empty_like(q), w.scale, part)
        pa.pa_decode_attention_append(p.pool, 0, [], kv, kv, q, torch.empty_like(q), w.scale, part)
    pa.pa_append_kv(p.pool, 0, [], [], kv, kv)
    assert pa.pa_alloc_blocks_n(p.pool, [], []) == 0
    torch.cuda.synchronize()
    assert before == (pa.pa_get_free_list(p.pool), pa.pa_get_refcounts(p.pool), pa.pa_launch_count(p.pool))
    p.check_metadata()
    p.check_cache(0)
    assert p.device_errors() == 0


@pytest.mark.parametrize("partition", [512, 0, -1])
def test_fp8_long_context_reduced(partition):
    """FP8-E4M3 KV with per-(layer, head) scales, 64 q / 8 KV heads, 8 sequences
    (2,048 tokens here; the full 32,768 below), split-KV partitions + reduce."""
    w = workload("fp8_long", tokens=2048)
    p = Pair(w)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    p.check_metadata()
    p.check_cache(0)
    q, out = p.decode(0, 0, seqs, partition)
    p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_fp8_long_context_full_size_sampled():
    """8 x 32,768 tokens, 512-token partitions (4,096 work units + reduce); the
    oracle keeps the contents of two sequences and checks all their heads."""
    w = workload("fp8_long")
    sample = [0, 5]
    p = Pair(w, oracle_seqs=sample)
    p.prefill()
    seqs, pos = p.reserve_step(0)
    p.append_step(0, 0, seqs, pos)
    p.check_metadata()
    p.check_cache(0, seqs=sample)
    for part in (512, 0):
        q, out = p.decode(0, 0, seqs, part)
        p.check_attention(0, seqs, q, out, only=sample)
    assert p.device_errors() == 0


def test_gqa70b_headroom_sampled_layers():
    """80 layers, 64 q / 8 KV heads, 47 sequences growing from 825 into block 53
    on the 2,491-block pool; three layers carry data and are compared at steps
    1, 8 and 16, layer 0 at every step."""
    w = workload("gqa70b_headroom")
    layers = [0, 40, 79]
    p = Pair(w, layers=layers)
    p.prefill(gpu_layers=layers)
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        for layer in range(w.num_layers):
            p.append_step(step, layer, seqs, pos)      # oracle keeps only the compared layers
            if layer in layers and (layer == 0 or step in (0, 7, 15)):
                q, out = p.decode(step, layer, seqs, 0)
                p.check_attention(layer, seqs, q, out)
            else:
                p.decode(step, layer, seqs, 0)
        if step in (0, 7, 15):
            p.check_metadata()
            for layer in layers:
                p.check_cache(layer)
    assert pa.pa_get_free_list(p.pool) == []
    assert p.device_errors() == 0
