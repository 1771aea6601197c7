"""Host-side checks of swap-out / swap-in (no GPU): the host image size is the
allocated-block bytes of "Managing the KV Cache", Hands-On Exercise (the
1,525-token request, derived from the printed bytes per token), and the
device calls are refused on host-only pools.
"""
import json
import os

import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "exercise_derived.json")
SHAPES = {  # case -> (layers, kv_heads, kv dtype)
    "bf16_gqa_b16": (80, 8, "bf16"), "bf16_gqa_b32": (80, 8, "bf16"),
    "fp8_gqa_b16": (80, 8, "fp8_e4m3"), "bf16_mha64_b16": (80, 64, "bf16"),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


def test_swap_bytes_match_the_exercise():
    g = json.load(open(GOLDEN))
    n = g["lengths"][2]
    for case in g["cases"]:
        L, H, kv = SHAPES[case["name"]]
        p = pa.pa_pool_create(num_layers=L, num_kv_heads=H, block_size=case["block_size"],
                              num_blocks=128, max_seqs=2, max_blocks_per_seq=128, kv_dtype=kv,
                              host_only=True)
        assert pa.pa_swap_bytes(p, n) == case["offload_allocated_bytes"]
        assert pa.pa_swap_bytes(p, 0) == 0
        # 1,536 tokens fill whole blocks at B = 16 and 32; one more costs a block
        B = case["block_size"]
        assert pa.pa_swap_bytes(p, 1537) - pa.pa_swap_bytes(p, 1536) == B * case["bytes_per_token"]
        with pytest.raises(pa.PAError) as e:
            pa.pa_swap_bytes(p, -1)
        assert e.value.status == pa.PA_ERR_INVALID_ARG


def test_swap_calls_refused_on_host_only_pool():
    p = pa.pa_pool_create(num_layers=2, num_kv_heads=2, block_size=16, num_blocks=16,
                          max_seqs=2, max_blocks_per_seq=8, host_only=True)
    pa.pa_alloc_blocks(p, 0, 20)
    img = np.zeros(pa.pa_swap_bytes(p, 20), np.uint8)
    for call in (lambda: pa.pa_swap_out(p, 0, img), lambda: pa.pa_swap_in(p, 1, 20, img)):
        with pytest.raises(pa.PAError) as e:
            call()
        assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert pa.pa_get_seq(p, 0)[0] == 20                    # nothing changed
    with pytest.raises(ValueError):
        pa.pa_swap_out(p, 0, img[::2])
