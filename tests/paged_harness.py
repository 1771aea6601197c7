"""Drives the CUDA path (through the C-ABI binding) and the oracle side by side
on one seeded workload, and compares them.

Both sides receive the same seeded inputs from ``workloads``; neither sees
the other's outputs.  Comparisons:

* block tables, lengths, reference counts, free list, copy-on-write log:
  bit-exact;
* cache contents of every valid slot (t < len) of the compared layers:
  bit-exact (bf16 / fp16 bits, or FP8 codes);
* attention output, element by element: |gpu - oracle| <= 1e-2 + 1e-2 |oracle|
  for 16-bit KV ("1e-2 absolute and 1e-2 relative"; a bf16 output alone
  is rounded by up to 2^-9 |oracle|, 1.6e-2 at |oracle| = 8), and
  |gpu - oracle| <= 5e-2 for FP8 KV (the oracle runs on the dequantised values).
"""
from __future__ import annotations

import numpy as np
import torch

import pagedattention_decode_03_b200 as pa
from oracle import PagedKVOracle, Status
from oracle.numerics import bits_to_f64
from workloads import fp8_scales, prefill_kv_bits, step_kv_bits, step_q_bits

# (absolute, relative) bound per KV dtype
TOL = {"bf16": (1e-2, 1e-2), "fp16": (1e-2, 1e-2), "fp8_e4m3": (5e-2, 0.0)}


def assert_close(got, ref, kv_dtype, what="attention"):
    """Every element within TOL[kv_dtype]; returns the largest |got - ref|."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    atol, rtol = TOL[kv_dtype]
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    if not (err <= bound).all():
        at = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: |err| {err[at]:.3e} > bound {bound[at]:.3e} at {at} "
                             f"(oracle {ref[at]:+.5f}, got {got[at]:+.5f})")
    return float(err.max()) if err.size else 0.0


def to_dev(bits: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    t = t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)
    return t.to(device)


def from_dev(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


class Pair:
    """A GPU pool and an oracle built from the same workload description."""

    def __init__(self, w, *, layers=None, num_blocks=None, free_order=None, min_partition=0,
                 scales_steps=None, oracle_seqs=None):
        self.w = w
        # sequences whose cache contents the oracle keeps (all by default); the
        # oracle's pool metadata always follows every sequence
        self.oracle_seqs = None if oracle_seqs is None else set(oracle_seqs)
        nb = num_blocks or w.num_blocks
        order = w.free_order() if free_order is None else np.asarray(free_order)
        if len(order) != nb:
            order = np.random.default_rng([w.seed, w.cfg, 99]).permutation(nb)
        self.layers = list(range(w.num_layers)) if layers is None else list(layers)
        self.scales = None
        kw = {}
        if w.kv_dtype == "fp8_e4m3":
            ks, vs, ki, vi = fp8_scales(w, scales_steps)
            self.scales = (ks, vs, ki, vi)
            dev = [torch.from_numpy(a).cuda() for a in (ks, vs, ki, vi)]
            kw = dict(k_scale=dev[0], v_scale=dev[1], k_inv_scale=dev[2], v_inv_scale=dev[3])
        self.pool = pa.pa_pool_create(
            num_layers=w.num_layers, num_kv_heads=w.num_kv_heads, block_size=w.block_size,
            num_blocks=nb, max_seqs=w.max_seqs, max_blocks_per_seq=w.max_blocks_per_seq,
            kv_dtype=w.kv_dtype, act_dtype=w.act_dtype, free_order=order,
            min_partition_tokens=min_partition, **kw)
        self.oracle = PagedKVOracle(
            num_layers=w.num_layers, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
            block_size=w.block_size, num_blocks=nb, max_seqs=w.max_seqs,
            max_blocks_per_seq=w.max_blocks_per_seq, kv_dtype=w.kv_dtype, free_order=order,
            stored_layers=self.layers)

    # ------------------------------------------------------------ driving
    def append(self, layer, seqs, positions, k_bits, v_bits, gpu=True):
        if gpu:
            pa.pa_append_kv(self.pool, layer, seqs, positions, to_dev(k_bits, self.w.act_dtype),
                            to_dev(v_bits, self.w.act_dtype))
        if layer in self.layers:
            ki = vi = None
            if self.scales is not None:
                ki, vi = self.scales[2], self.scales[3]
            if self.oracle_seqs is not None:
                keep = [t for t, s in enumerate(seqs) if s in self.oracle_seqs]
                if not keep:
                    return
                seqs = [seqs[t] for t in keep]
                positions = [positions[t] for t in keep]
                k_bits, v_bits = k_bits[keep], v_bits[keep]
            st = self.oracle.append(layer, seqs, positions, k_bits, v_bits, self.w.act_dtype, ki, vi)
            assert st is Status.OK, st

    def prefill(self, gpu_layers=None):
        """Reserve and write every prefill token; forks afterwards."""
        w = self.w
        gpu_layers = range(w.num_layers) if gpu_layers is None else gpu_layers
        for s in sorted(w.prefill_lens):
            n = w.prefill_lens[s]
            pa.pa_alloc_blocks(self.pool, s, n)
            assert self.oracle.reserve(s, n) is Status.OK
            for layer in range(w.num_layers):
                on_gpu = layer in gpu_layers
                if not on_gpu and layer not in self.layers:
                    continue
                k, v = prefill_kv_bits(w, layer, s)
                for c0 in range(0, n, 8192):
                    c1 = min(n, c0 + 8192)
                    self.append(layer, [s] * (c1 - c0), list(range(c0, c1)), k[c0:c1], v[c0:c1],
                                gpu=on_gpu)
        for parent, child in w.forks:
            pa.pa_fork_cow(self.pool, parent, child)
            assert self.oracle.fork(parent, child) is Status.OK

    def reserve_step(self, step):
        w = self.w
        lens = w.lens_before_step(step)
        seqs = list(w.seq_ids)
        new = [lens[s] + 1 for s in seqs]
        pa.pa_alloc_blocks_n(self.pool, seqs, new)
        for s, n in zip(seqs, new):
            assert self.oracle.reserve(s, n) is Status.OK
        return seqs, [lens[s] for s in seqs]

    def append_step(self, step, layer, seqs, positions):
        k, v = step_kv_bits(self.w, step, layer)
        self.append(layer, seqs, positions, k, v)

    def decode(self, step, layer, seqs, partition_tokens=0, q_bits=None):
        w = self.w
        q_bits = step_q_bits(w, step, layer) if q_bits is None else q_bits
        q = to_dev(q_bits, w.act_dtype)
        out = torch.empty_like(q)
        pa.pa_decode_attention(self.pool, layer, seqs, q, out, w.scale, partition_tokens)
        return q_bits, out

    def append_decode(self, step, layer, seqs, positions, partition_tokens=0):
        """The step's append of every sequence's last token and the decode in one
        call (pa_decode_attention_append); the oracle appends the same rows."""
        w = self.w
        k, v = step_kv_bits(w, step, layer)
        q_bits = step_q_bits(w, step, layer)
        q = to_dev(q_bits, w.act_dtype)
        out = torch.empty_like(q)
        pa.pa_decode_attention_append(self.pool, layer, seqs, to_dev(k, w.act_dtype),
                                      to_dev(v, w.act_dtype), q, out, w.scale, partition_tokens)
        self.append(layer, seqs, positions, k, v, gpu=False)
        return q_bits, out

    def oracle_attention(self, layer, seqs, q_bits):
        ks = vs = None
        if self.scales is not None:
            ks, vs = self.scales[0], self.scales[1]
        return self.oracle.attention(layer, seqs, q_bits, self.w.act_dtype, self.w.scale, ks, vs)

    # --------------------------------------------------------- comparing
    def check_metadata(self):
        o, p = self.oracle, self.pool
        assert pa.pa_get_free_list(p) == o.free_list()
        assert pa.pa_get_refcounts(p) == o.refcounts()
        for s in o.tables:
            n, tab = pa.pa_get_seq(p, s)
            assert n == o.lens[s] and tab == o.table(s), s
        assert pa.pa_get_cow_log(p) == o.cow_log

    def check_cache(self, layer, seqs=None):
        """Bit-exact comparison of every valid slot of `layer`."""
        o = self.oracle
        seqs = list(o.tables) if seqs is None else seqs
        kc, vc = self.pool.k_cache[layer], self.pool.v_cache[layer]
        for s in seqs:
            n = o.lens[s]
            t = np.arange(n)
            blocks = torch.from_numpy(np.asarray(o.table(s), np.int64)[t // o.B]).cuda()
            offs = torch.from_numpy(t % o.B).cuda()
            gk = kc[blocks, :, offs, :]
            gv = vc[blocks, :, offs, :]
            if self.w.kv_dtype == "fp8_e4m3":
                gk, gv = gk.cpu().numpy(), gv.cpu().numpy()
            else:
                gk, gv = from_dev(gk), from_dev(gv)
            blk = np.asarray(o.table(s), np.int64)[t // o.B]
            assert np.array_equal(gk, o.k[layer][blk, :, t % o.B, :]), ("K", layer, s)
            assert np.array_equal(gv, o.v[layer][blk, :, t % o.B, :]), ("V", layer, s)

    def check_attention(self, layer, seqs, q_bits, out, only=None):
        """Compare the decode output of items `only` (all by default);
        returns the largest |gpu - oracle|."""
        got = bits_to_f64(from_dev(out), self.w.act_dtype)
        if only is not None:
            seqs = [seqs[i] for i in only]
            q_bits = q_bits[list(only)]
            got = got[list(only)]
        ref = self.oracle_attention(layer, seqs, q_bits)
        return assert_close(got, ref, self.w.kv_dtype, f"attention, layer {layer}")

    def device_errors(self):
        return pa.pa_check_device_errors(self.pool)
