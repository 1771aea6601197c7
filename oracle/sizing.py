"""KV-cache sizing arithmetic (oracle).

Test infrastructure only: imported by tests and the benchmark's CPU leg.

All quantities are plain integer arithmetic on the definitions the pages
state; no rounding beyond the floors and ceilings they name.
"""
from __future__ import annotations


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_element: int) -> int:
    """Two tensors (K and V) x layers x KV heads x head_dim x element bytes.

    "Managing the KV Cache", Reproduce Bytes per Token; "KV cache", The
    maths (cache size per token); kv-cache-pagedattention-serving, What the
    KV cache actually is.
    """
    return 2 * layers * kv_heads * head_dim * bytes_per_element


def blocks_for(tokens: int, block_size: int) -> int:
    """Blocks a sequence of `tokens` occupies: ceil(tokens / block_size).

    "Managing the KV Cache", Worked Example: The 825-Token Request.
    """
    if tokens < 0 or block_size <= 0:
        raise ValueError("invalid sequence or block size")
    return -(-tokens // block_size)


def paged_request(tokens: int, block_size: int) -> dict:
    """Paged allocation of one request: blocks, slots, unused slots, waste %.

    "Managing the KV Cache", Worked Example: Paged Allocation With 16-Token
    Blocks.
    """
    blocks = blocks_for(tokens, block_size)
    slots = blocks * block_size
    unused = slots - tokens
    return {
        "blocks": blocks,
        "slots": slots,
        "unused_slots": unused,
        "internal_waste_percent": 100.0 * unused / slots if slots else 0.0,
    }


def contiguous_request(used_tokens: int, reserved_tokens: int) -> dict:
    """Contiguous max-length reservation of one request.

    "Managing the KV Cache", Worked Example: Contiguous Reservation.
    """
    unused = reserved_tokens - used_tokens
    return {
        "slots": reserved_tokens,
        "unused_slots": unused,
        "unused_fraction": unused / reserved_tokens,
    }


def token_slots(budget_bytes: int, bytes_per_token: int) -> int:
    """Whole token slots in a byte budget: floor(budget / bytes_per_token).

    "Managing the KV Cache", Worked Capacity Under a 12 GiB KV Budget.
    """
    return budget_bytes // bytes_per_token


def pool_blocks(budget_bytes: int, bytes_per_token: int, block_size: int) -> int:
    """Complete blocks in a byte budget: floor(budget / (bytes/token x B)).

    "Managing the KV Cache", Worked Capacity Under a 12 GiB KV Budget (the
    pool holds complete blocks only; the leftover cannot form a block).
    """
    return budget_bytes // (bytes_per_token * block_size)


def capacity(budget_bytes: int, bytes_per_token: int, block_size: int,
             used_tokens: int, reserved_tokens: int) -> dict:
    """Snapshot request capacity, contiguous versus paged.

    contiguous = floor(token_slots / reserved); paged = floor(pool_blocks /
    blocks per request).  "Managing the KV Cache", Worked Capacity Under a
    12 GiB KV Budget and Build the Capacity Calculator.
    """
    slots = token_slots(budget_bytes, bytes_per_token)
    blocks = pool_blocks(budget_bytes, bytes_per_token, block_size)
    per_req = blocks_for(used_tokens, block_size)
    contiguous = slots // reserved_tokens
    paged = blocks // per_req
    return {
        "token_slots": slots,
        "pool_blocks": blocks,
        "block_backed_slots": blocks * block_size,
        "contiguous_requests": contiguous,
        "paged_requests": paged,
        "capacity_ratio": paged / contiguous,
    }


def group_packing(budget_bytes: int, bytes_per_token: int, block_size: int,
                  lengths: list[int], offload_tokens: int) -> dict:
    """Whole groups of requests packed into a pool (no sharing, own tails).

    "Managing the KV Cache", Hands-On Exercise: allocated slots per group,
    useful slots, tail waste per group, complete groups that fit, and the
    useful versus allocated bytes of offloading one request.
    """
    blocks = sum(blocks_for(n, block_size) for n in lengths)
    slots = blocks * block_size
    useful = sum(lengths)
    pool = pool_blocks(budget_bytes, bytes_per_token, block_size)
    return {
        "blocks_per_group": blocks,
        "slots_per_group": slots,
        "useful_slots": useful,
        "tail_waste": slots - useful,
        "pool_blocks": pool,
        "groups": pool // blocks,
        "offload_useful_bytes": offload_tokens * bytes_per_token,
        "offload_allocated_bytes": blocks_for(offload_tokens, block_size) * block_size * bytes_per_token,
    }
