"""The five paged-decode workloads, as concrete seeded shapes.

Each workload fixes the model shape (layers, query / KV heads, head_dim),
the storage dtypes, the pool size, the per-sequence lengths before the first
decode step, the fork structure (parallel sampling) and the number of decode
steps.  Sizes follow the worked examples of the pages:

* tiny: 4 sequences {825, 200, 103, 16}, 8 q / 2 KV heads, 128-block pool
  ("Managing the KV Cache", Worked Example: The 825-Token Request);
* gqa8b: 64 sequences, lengths uniform in [128, 4096], 32 q / 8 KV heads,
  pool sized 1.25x the need at the end of the run;
* gqa70b: 80 layers, 64 q / 8 KV heads, 47 sequences at 825 tokens in the
  2,457-block pool of the 12 GiB budget ("Worked Capacity Under a 12 GiB KV
  Budget"); a +34-block headroom variant lets all 47 grow into block 53;
* mha7b_share: 32 layers, 32/32 heads, fp16, 4 prompts of 2,050 tokens each
  forked 7 times (parallel sampling n=8, "The bonus: sharing via
  copy-on-write");
* fp8_long: 64 q / 8 KV heads, FP8-E4M3 KV with per-(layer, head) scales,
  8 sequences of 32,768 tokens, 512-token split-KV partitions.

No paging arithmetic lives here beyond sizing the pool buffer; the block
counts used for pool sizing are plain ceilings of lengths.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .gen import Purpose, rng


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: int
    num_layers: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    act_dtype: str            # "bf16" | "fp16": q, out, k_new, v_new
    kv_dtype: str             # "bf16" | "fp16" | "fp8_e4m3": the pool
    num_blocks: int
    max_seqs: int
    max_blocks_per_seq: int
    seq_ids: tuple            # decode order (ascending)
    prefill_lens: dict = field(hash=False)   # seq -> tokens written before forks
    forks: tuple = ()         # (parent, child) pairs, applied after prefill
    steps: int = 1
    partition_tokens: int = 0  # 0 = library chooses, -1 = never split, >0 fixed
    seed: int = 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(head_dim), rounded to fp32."""
        return float(np.float32(1.0 / math.sqrt(self.head_dim)))

    def lens_before_step(self, step: int) -> dict:
        """Sequence lengths before decode step `step` (0-based)."""
        base = dict(self.prefill_lens)
        for parent, child in self.forks:
            base[child] = base[parent]
        return {s: base[s] + step for s in self.seq_ids}

    def free_order(self) -> np.ndarray:
        return rng(self.seed, self.cfg, Purpose.PERM).permutation(self.num_blocks).astype(np.int32)


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _tiny(seed: int, steps: int) -> Workload:
    lens = [825, 200, 103, 16]
    mbps = max(_ceil_div(n + steps, 16) for n in lens) + 1
    return Workload(
        name="tiny", cfg=1, num_layers=1, num_q_heads=8, num_kv_heads=2, head_dim=128,
        block_size=16, act_dtype="bf16", kv_dtype="bf16", num_blocks=128, max_seqs=4,
        max_blocks_per_seq=mbps, seq_ids=(0, 1, 2, 3),
        prefill_lens={i: n for i, n in enumerate(lens)}, steps=steps, seed=seed)


def _gqa8b(seed: int, steps: int, num_seqs: int = 64) -> Workload:
    lens = rng(seed, 2, Purpose.LENS).integers(128, 4096, size=num_seqs, endpoint=True)
    need = sum(_ceil_div(int(n) + steps, 16) for n in lens)
    mbps = max(_ceil_div(int(n) + steps, 16) for n in lens)
    return Workload(
        name="gqa8b", cfg=2, num_layers=1, num_q_heads=32, num_kv_heads=8, head_dim=128,
        block_size=16, act_dtype="bf16", kv_dtype="bf16",
        num_blocks=_ceil_div(5 * need, 4), max_seqs=num_seqs, max_blocks_per_seq=mbps,
        seq_ids=tuple(range(num_seqs)),
        prefill_lens={i: int(n) for i, n in enumerate(lens)}, steps=steps, seed=seed)


def _gqa70b(seed: int, steps: int, headroom: bool) -> Workload:
    n_seqs = 47
    nb = 2457
    if headroom:
        nb = max(nb, n_seqs * _ceil_div(825 + steps, 16))
    return Workload(
        name="gqa70b_headroom" if headroom else "gqa70b", cfg=3, num_layers=80,
        num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
        act_dtype="bf16", kv_dtype="bf16", num_blocks=nb, max_seqs=n_seqs,
        max_blocks_per_seq=_ceil_div(825 + steps, 16) + 1, seq_ids=tuple(range(n_seqs)),
        prefill_lens={i: 825 for i in range(n_seqs)}, steps=steps, seed=seed)


def _mha7b_share(seed: int, steps: int) -> Workload:
    prompts, n, plen = 4, 8, 2050
    forks = tuple((8 * p, 8 * p + c) for p in range(prompts) for c in range(1, n))
    shared_full = plen // 16
    private = _ceil_div(plen + steps, 16) - shared_full
    need = prompts * shared_full + prompts * n * private
    return Workload(
        name="mha7b_share", cfg=4, num_layers=32, num_q_heads=32, num_kv_heads=32,
        head_dim=128, block_size=16, act_dtype="fp16", kv_dtype="fp16",
        num_blocks=_ceil_div(5 * need, 4), max_seqs=prompts * n,
        max_blocks_per_seq=_ceil_div(plen + steps, 16) + 1,
        seq_ids=tuple(range(prompts * n)),
        prefill_lens={8 * p: plen for p in range(prompts)}, forks=forks, steps=steps,
        seed=seed)


def _fp8_long(seed: int, steps: int, num_seqs: int = 8, tokens: int = 32768) -> Workload:
    per_seq = _ceil_div(tokens + steps, 16)
    return Workload(
        name="fp8_long", cfg=5, num_layers=1, num_q_heads=64, num_kv_heads=8, head_dim=128,
        block_size=16, act_dtype="bf16", kv_dtype="fp8_e4m3",
        num_blocks=_ceil_div(5 * num_seqs * per_seq, 4), max_seqs=num_seqs,
        max_blocks_per_seq=per_seq + 1, seq_ids=tuple(range(num_seqs)),
        prefill_lens={i: tokens for i in range(num_seqs)}, steps=steps,
        partition_tokens=512, seed=seed)


WORKLOADS = {
    "tiny": lambda seed=0, steps=1, **kw: _tiny(seed, steps),
    "gqa8b": lambda seed=0, steps=100, **kw: _gqa8b(seed, steps, **kw),
    "gqa70b": lambda seed=0, steps=16, **kw: _gqa70b(seed, steps, headroom=False),
    "gqa70b_headroom": lambda seed=0, steps=16, **kw: _gqa70b(seed, steps, headroom=True),
    "mha7b_share": lambda seed=0, steps=64, **kw: _mha7b_share(seed, steps),
    "fp8_long": lambda seed=0, steps=1, **kw: _fp8_long(seed, steps, **kw),
}


def workload(name: str, **kw) -> Workload:
    return WORKLOADS[name](**kw)
