"""GPU parity of pa_decode_attention_append: the step's append of every
sequence's last token fused into the decode launch.  Cache contents are
compared bit-exactly with the oracle (which appends the same rows), the
output within the decode tolerance, in every split mode, for 16-bit and FP8
KV, plain and sibling-set plans."""
import numpy as np
import pytest
import torch

import pagedattention_decode_03_b200 as pa
from paged_harness import Pair, to_dev
from test_gpu_siblings import family_workload
from workloads import step_kv_bits, step_q_bits, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()
    assert torch.cuda.is_available()


def run(p, w, parts):
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        for part in parts:                 # same rows written again: same bits
            q, out = p.append_decode(step, 0, seqs, pos, part)
            p.check_attention(0, seqs, q, out)
        p.check_cache(0)
    p.check_metadata()
    assert p.device_errors() == 0


def test_fused_tiny_all_modes():
    w = workload("tiny", steps=3)
    p = Pair(w, min_partition=16)
    p.prefill()
    run(p, w, (0, -1, 16))


@pytest.mark.parametrize("kv", ["bf16", "fp16", "fp8_e4m3"])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_fused_families(G, kv):
    """Forks (copy-on-write at the first append), sibling sets (G < 8) and
    unrelated sequences; lengths cross block boundaries during the steps."""
    w = family_workload(G, kv, [(203, 8 // G + 1), (47, 2)], [300, 15, 16], steps=18)
    p = Pair(w, min_partition=16)
    p.prefill()
    run(p, w, (0, 32))


def test_fused_equals_separate_calls_bitwise():
    """Same output bits as pa_append_kv + pa_decode_attention."""
    w = workload("gqa8b", num_seqs=12, steps=2)
    outs = []
    for fused in (False, True):
        p = Pair(w)
        p.prefill()
        seqs, pos = p.reserve_step(0)
        if fused:
            _, out = p.append_decode(0, 0, seqs, pos, 0)
        else:
            p.append_step(0, 0, seqs, pos)
            _, out = p.decode(0, 0, seqs, 0)
        p.check_cache(0)
        outs.append(out.view(torch.int16).cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


def test_fused_host_errors_launch_nothing():
    w = family_workload(4, "bf16", [(40, 2)], [20], steps=1)
    p = Pair(w, min_partition=16)
    p.prefill()
    H, Hq = w.num_kv_heads, w.num_q_heads
    kn = torch.zeros((3, H, 128), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((3, Hq, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    n0 = pa.pa_launch_count(p.pool)
    # the forked pair still shares its partly filled tail block: no reservation yet
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_attention_append(p.pool, 0, [0, 1], kn[:2], kn[:2], q[:2], out[:2], w.scale)
    assert e.value.status == pa.PA_ERR_SHARED_BLOCK
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_attention_append(p.pool, 0, [2, 2], kn[:2], kn[:2], q[:2], out[:2], w.scale)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert pa.pa_launch_count(p.pool) == n0
    p.check_metadata()


def test_fused_gqa8b_full_size():
    """The benchmark's step at full size: 64 sequences of 128..4096 tokens,
    append fused into the decode, growth across block boundaries; every 5th
    step checked in full (cache bit-exact, every output within tolerance)."""
    w = workload("gqa8b", steps=11)
    p = Pair(w)
    p.prefill()
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        q, out = p.append_decode(step, 0, seqs, pos, 0)
        if step % 5 == 0:
            p.check_metadata()
            p.check_cache(0)
            p.check_attention(0, seqs, q, out)
    assert p.device_errors() == 0


def test_fused_gqa70b_layers():
    """80 layers on the 2,491-block pool, every layer's append fused into its
    decode as in the benchmark step; layers 0 and 79 carry data and are
    compared at steps 1, 8 and 16 (layer 0 at every step)."""
    w = workload("gqa70b_headroom")
    layers = [0, 79]
    p = Pair(w, layers=layers)
    p.prefill(gpu_layers=layers)
    for step in range(w.steps):
        seqs, pos = p.reserve_step(step)
        for layer in range(w.num_layers):
            q, out = p.append_decode(step, layer, seqs, pos, 0)
            if layer in layers and (layer == 0 or step in (0, 7, 15)):
                p.check_attention(layer, seqs, q, out)
        if step in (0, 7, 15):
            p.check_metadata()
            for layer in layers:
                p.check_cache(layer)
    assert p.device_errors() == 0
