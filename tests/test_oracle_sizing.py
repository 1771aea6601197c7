"""Pins the oracle's sizing arithmetic to the numbers the pages print."""
import json
import math
import os

import pytest

from oracle import sizing


@pytest.fixture(scope="module")
def printed(golden_dir):
    with open(os.path.join(golden_dir, "printed_sizing.json")) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def exercise(golden_dir):
    with open(os.path.join(golden_dir, "exercise_derived.json")) as f:
        return json.load(f)


def test_bytes_per_token_printed(printed):
    for row in printed["bytes_per_token"]:
        got = sizing.kv_bytes_per_token(row["layers"], row["kv_heads"], row["head_dim"], row["bytes"])
        if "value" in row:
            assert got == row["value"], row["cite"]
        if "mib" in row:
            assert got / 2**20 == row["mib"], row["cite"]
        if "approx_mb" in row:
            # the page rounds 524,288 B to half a megabyte
            assert got == 524288 and abs(got / 2**20 - row["approx_mb"]) < 1e-12, row["cite"]


def test_bytes_per_token_ratios():
    # GQA versus MHA at 64 KV heads: the per-token footprint differs by the KV-head
    # ratio, 8x ("Managing the KV Cache", Reproduce Bytes per Token)
    gqa = sizing.kv_bytes_per_token(80, 8, 128, 2)
    mha = sizing.kv_bytes_per_token(80, 64, 128, 2)
    assert mha == 8 * gqa
    # FP8 halves the logical payload
    assert sizing.kv_bytes_per_token(80, 8, 128, 1) * 2 == gqa


def test_worked_825(printed):
    w = printed["worked_825"]
    c = sizing.contiguous_request(w["used"], w["reserved"])
    assert c["unused_slots"] == w["contiguous_unused"]
    assert round(100 * c["unused_fraction"], 2) == w["contiguous_unused_percent"]
    p = sizing.paged_request(w["used"], w["block_size"])
    assert p["blocks"] == w["paged_blocks"]
    assert p["slots"] == w["paged_slots"]
    assert p["unused_slots"] == w["paged_unused"]
    assert round(p["internal_waste_percent"], 4) == w["paged_waste_percent"]
    assert round(w["reserved"] / p["slots"], 4) == w["ratio"]


def test_capacity_12gib(printed):
    c12 = printed["capacity_12gib"]
    assert 12 * 2**30 == c12["budget_bytes"]
    bpt = sizing.kv_bytes_per_token(80, 8, 128, 2)
    cap = sizing.capacity(c12["budget_bytes"], bpt, 16, 825, 2048)
    assert cap["token_slots"] == c12["token_slots"]
    assert cap["pool_blocks"] == c12["pool_blocks"]
    assert cap["block_backed_slots"] == c12["block_backed_slots"]
    assert cap["contiguous_requests"] == c12["contiguous_requests"]
    assert cap["paged_requests"] == c12["paged_requests"]
    assert round(cap["capacity_ratio"], 4) == c12["capacity_ratio"]
    leftover = c12["budget_bytes"] - cap["pool_blocks"] * 16 * bpt
    assert leftover == c12["leftover_mib"] * 2**20
    assert round(leftover / bpt, 1) == c12["leftover_tokens_approx"]
    # a 48th request does not fit at the 825-token snapshot
    per_req = sizing.paged_request(825, 16)["slots"]
    assert 48 * per_req == c12["slots_for_48"] > cap["block_backed_slots"]
    fp8 = sizing.kv_bytes_per_token(80, 8, 128, 1)
    assert sizing.token_slots(c12["budget_bytes"], fp8) == c12["fp8_ideal_token_slots"]


def test_broken_cases(printed):
    b = printed["broken_cases"]
    p32 = sizing.paged_request(825, 32)
    assert p32["blocks"] == b["b32_blocks_825"] and p32["slots"] == b["b32_slots_825"]
    assert sizing.paged_request(200, 16)["slots"] == b["slots_200_b16"]
    assert sizing.paged_request(200, 32)["slots"] == b["slots_200_b32"]
    wrong = sizing.kv_bytes_per_token(80, b["wrong_head_count_q_heads"], 128, 2)
    assert sizing.token_slots(12 * 2**30, wrong) == b["wrong_head_count_token_slots"]


def test_rough_figures(printed):
    r70, r8b, prefix = printed["rough_figures"]
    bpt = sizing.kv_bytes_per_token(80, 8, 128, 2)
    assert abs(bpt / 1000 - r70["per_token_kb_approx"]) / r70["per_token_kb_approx"] < 0.1
    assert abs(bpt * r70["tokens"] / 1e9 - r70["total_gb_approx"]) / r70["total_gb_approx"] < 0.1
    assert sizing.kv_bytes_per_token(32, 32, 128, 2) * r8b["tokens"] == 2 * 2**30
    # block-granular prefix reuse: only whole blocks of the prompt can be shared
    assert (prefix["prompt"] // prefix["block_size"]) * prefix["block_size"] == prefix["reusable"]


def test_exercise_derived(exercise):
    for case in exercise["cases"]:
        got = sizing.group_packing(exercise["budget_bytes"], case["bytes_per_token"],
                                   case["block_size"], exercise["lengths"], 1525)
        for key in ("blocks_per_group", "slots_per_group", "useful_slots", "tail_waste",
                    "pool_blocks", "groups", "offload_useful_bytes", "offload_allocated_bytes"):
            assert got[key] == case[key], (case["name"], key)


@pytest.mark.parametrize("block_size", [1, 2, 7, 16, 32])
def test_tail_waste_bound_closed_form(block_size):
    # "Managing the KV Cache", Internal Fragmentation: waste <= block_size - 1,
    # and zero exactly on block boundaries
    for n in range(1, 300):
        p = sizing.paged_request(n, block_size)
        assert 0 <= p["unused_slots"] <= block_size - 1
        assert (p["unused_slots"] == 0) == (n % block_size == 0)
        assert p["blocks"] == math.ceil(n / block_size)


def test_calculator_rejects_bad_sizes():
    with pytest.raises(ValueError):
        sizing.blocks_for(10, 0)
    with pytest.raises(ValueError):
        sizing.blocks_for(-1, 16)
