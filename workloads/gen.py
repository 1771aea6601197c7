"""Seeded random draws for the paged decode workloads.

Every array is drawn from ``numpy.random.default_rng([seed, cfg, purpose,
...])`` so each consumer can regenerate exactly the slice it needs (one
layer, one sequence, one step) without materialising the whole workload.
Values are N(0, 1) in fp32, rounded to the activation dtype with IEEE
round-to-nearest-even (bf16 through torch's conversion, fp16 through numpy's)
and returned as raw uint16 bit patterns.
"""
from __future__ import annotations

import enum
import hashlib

import numpy as np
import torch

_E4M3_MAX = 448.0  # largest finite OCP FP8 E4M3 value; used only to size the scale


class Purpose(enum.IntEnum):
    LENS = 0
    PERM = 1
    PREFILL_K = 2
    PREFILL_V = 3
    Q = 4
    K_NEW = 5
    V_NEW = 6
    MISC = 7
    PREFIX_KV = 8


def rng(seed: int, cfg: int, purpose: int, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(cfg), int(purpose), *[int(e) for e in extra]])


def _round_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "fp16":
        return x.astype(np.float16).view(np.uint16)
    raise ValueError(f"unsupported activation dtype {dtype!r}")


def normal_bits(g: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0,1) fp32 draws rounded to `dtype`, as uint16 bit patterns."""
    return _round_bits(g.standard_normal(shape, dtype=np.float32), dtype)


def prefill_kv_bits(w, layer: int, seq: int, tokens: int | None = None):
    """K and V rows written for `seq` before the first decode step.

    Shape [tokens, num_kv_heads, head_dim], activation dtype bits.
    """
    n = w.prefill_lens[seq] if tokens is None else tokens
    shape = (n, w.num_kv_heads, w.head_dim)
    k = normal_bits(rng(w.seed, w.cfg, Purpose.PREFILL_K, layer, seq), shape, w.act_dtype)
    v = normal_bits(rng(w.seed, w.cfg, Purpose.PREFILL_V, layer, seq), shape, w.act_dtype)
    return k, v


def step_q_bits(w, step: int, layer: int) -> np.ndarray:
    """Decode queries of step `step`: [num_seqs, num_q_heads, head_dim] bits."""
    shape = (len(w.seq_ids), w.num_q_heads, w.head_dim)
    return normal_bits(rng(w.seed, w.cfg, Purpose.Q, step, layer), shape, w.act_dtype)


def step_kv_bits(w, step: int, layer: int):
    """K/V rows appended at step `step`: [num_seqs, num_kv_heads, head_dim] bits each."""
    shape = (len(w.seq_ids), w.num_kv_heads, w.head_dim)
    k = normal_bits(rng(w.seed, w.cfg, Purpose.K_NEW, step, layer), shape, w.act_dtype)
    v = normal_bits(rng(w.seed, w.cfg, Purpose.V_NEW, step, layer), shape, w.act_dtype)
    return k, v


def prefix_kv_bits(w, layer: int, tokens, lo: int, hi: int):
    """K and V rows of positions lo..hi-1 of the token history `tokens`.

    Each row is drawn from a generator seeded by the whole token prefix that
    ends at its position, so two histories that start with the same tokens
    get the same rows there, as a model's KV would.  Shape [hi - lo,
    num_kv_heads, head_dim], activation dtype bits, each.
    """
    shape = (max(hi - lo, 0), w.num_kv_heads, w.head_dim)
    k = np.zeros(shape, np.uint16)
    v = np.zeros(shape, np.uint16)
    toks = np.asarray(tokens, np.int64)
    for t in range(lo, hi):
        digest = hashlib.blake2b(toks[: t + 1].tobytes(), digest_size=8).digest()
        g = rng(w.seed, w.cfg, Purpose.PREFIX_KV, layer, int.from_bytes(digest, "little"))
        k[t - lo] = normal_bits(g, shape[1:], w.act_dtype)
        v[t - lo] = normal_bits(g, shape[1:], w.act_dtype)
    return k, v


def _to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32)
    return bits.view(np.float16).astype(np.float32)


def fp8_scales(w, steps: int | None = None):
    """Per-(layer, kv_head) calibration scales for an FP8 pool.

    scale = amax(|x|) / 448 over every K (resp. V) value the workload writes
    for that layer and head (prefill plus `steps` decode steps), in fp32;
    inv_scale = fp32(1 / scale), computed once here so every consumer uses
    the same bits.  Returns (k_scale, v_scale, k_inv, v_inv), each
    float32 [num_layers, num_kv_heads].
    """
    steps = w.steps if steps is None else steps
    L, H = w.num_layers, w.num_kv_heads
    amax_k = np.zeros((L, H), np.float32)
    amax_v = np.zeros((L, H), np.float32)
    for layer in range(L):
        for seq, n in w.prefill_lens.items():
            k, v = prefill_kv_bits(w, layer, seq, n)
            amax_k[layer] = np.maximum(amax_k[layer], np.abs(_to_f32(k, w.act_dtype)).max(axis=(0, 2)))
            amax_v[layer] = np.maximum(amax_v[layer], np.abs(_to_f32(v, w.act_dtype)).max(axis=(0, 2)))
        for step in range(steps):
            k, v = step_kv_bits(w, step, layer)
            amax_k[layer] = np.maximum(amax_k[layer], np.abs(_to_f32(k, w.act_dtype)).max(axis=(0, 2)))
            amax_v[layer] = np.maximum(amax_v[layer], np.abs(_to_f32(v, w.act_dtype)).max(axis=(0, 2)))
    k_scale = (amax_k / np.float32(_E4M3_MAX)).astype(np.float32)
    v_scale = (amax_v / np.float32(_E4M3_MAX)).astype(np.float32)
    k_inv = (np.float32(1.0) / k_scale).astype(np.float32)
    v_inv = (np.float32(1.0) / v_scale).astype(np.float32)
    return k_scale, v_scale, k_inv, v_inv
