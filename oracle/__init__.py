"""CPU oracle for paged single-query decode attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the smoke check
(`__graft_entry__.smoke`) and the benchmark's CPU-baseline leg may import
anything in this package.  The library path never calls it and never falls
back to it.

The oracle is a plain, slow, float64 model of what the pages define, written
so a reader can check it against them by eye:

* ``sizing``   -- KV bytes per token, block/slot counts, pool capacity
                  ("Managing the KV Cache": Reproduce Bytes per Token, Worked
                  Example: The 825-Token Request, Worked Capacity Under a
                  12 GiB KV Budget, Build the Capacity Calculator, Hands-On
                  Exercise);
* ``fp8``      -- OCP FP8 E4M3 encode (round-to-nearest-even, saturate to
                  +-448) and exact decode ("Managing the KV Cache": Quantized
                  KV names the format, the OCP 8-bit floating point
                  specification defines it);
* ``numerics`` -- bf16 / fp16 bit patterns to float64;
* ``paged``    -- the block pool (free list, per-sequence block tables,
                  reference counts, copy-on-write of a shared tail block),
                  the cache contents, and attention computed by first
                  gathering each sequence's blocks into a contiguous buffer
                  ("KV cache": The maths; "Managing the KV Cache": Block
                  Tables and Sharing; kv-cache-pagedattention-serving:
                  PagedAttention: virtual memory for GPUs, The bonus:
                  sharing via copy-on-write).

It shares no code with the CUDA path and imports nothing from it.
Every function is pinned by tests under ``tests/`` against values the pages
print, closed forms, brute force on tiny inputs and library routines.
"""
from . import fp8, numerics, paged, sizing  # noqa: F401
from .paged import PagedKVOracle, Status  # noqa: F401
