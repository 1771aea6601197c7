"""Benchmark of the paged decode-attention hot path on B200.

One step = one decode step of the workload: reserve one more slot per
sequence (block manager; a block on boundary crossings, copy-on-write where
a shared tail is written), then for every layer append the step's K/V row
per sequence and run decode attention for every sequence -- all through the
C ABI (libpa.so).  Default workload: the 70B-class GQA model of "Managing
the KV Cache" (Worked Capacity Under a 12 GiB KV Budget): 80 layers, 64 query /
8 KV heads, head_dim 128, bf16, 16-token blocks, 47 sequences of 825 tokens in
the 2,457-block pool plus the headroom that lets all of them grow into block
53, 16 decode steps; `--workload` selects the other configurations.

Metric: achieved HBM GB/s of the step's algorithmic bytes (KV read by the
decode + Q + O + block-table entries + appended rows read and written),
with its fraction of the measured B200 copy bandwidth, and decode tokens/s
(sequences x steps / time).  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun each rank runs its own replica of the workload on its own GPU
(the path has no exchange step: replicas only, weak scaling); the timed
region is bracketed by a barrier and synchronize, and the time is the max
over ranks.  `--impl reference` times the CPU oracle (float64 NumPy) on the
host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attn: achieved HBM GB/s (% of B200 peak), decode tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: the workload's own decode step count)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gqa70b_headroom",
                    choices=["tiny", "gqa8b", "gqa70b_headroom", "mha7b_share", "fp8_long"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition", type=int, default=None,
                    help="partition_tokens for decode (default: the workload's)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-swap", action="store_true",
                    help="skip the swap-out / swap-in transfer measurement")
    ap.add_argument("--separate-append", action="store_true",
                    help="append with pa_append_kv and decode with pa_decode_attention (two launches "
                         "per layer) instead of the fused pa_decode_attention_append")
    ap.add_argument("--decode-path", default="auto", choices=["auto", "warp", "tcgen05"],
                    help="decode kernel for a query group of 8 over 16-bit KV (pa_set_decode_path)")
    ap.add_argument("--layers", type=int, default=None,
                    help="profiling: keep only the first N layers (a smaller case of the same "
                         "kernels; the JSON line then names the reduced workload)")
    return ap.parse_args()


DEFAULT_STEPS = {"tiny": 1, "gqa8b": 100, "gqa70b_headroom": 16, "mha7b_share": 64, "fp8_long": 1}
# timed steps when --steps is not given: the workload's decode steps, and
# enough launches for a stable mean where a workload has a single step
BENCH_STEPS = {"tiny": 100, "gqa8b": 100, "gqa70b_headroom": 16, "mha7b_share": 64, "fp8_long": 20}


def pool_steps(a):
    """Decode steps the pool is sized for (same in both arms): the timed run
    plus the end-to-end run, and never fewer than the workload's own count."""
    return max(DEFAULT_STEPS[a.workload], 2 * (a.warmup + a.steps))


def make_workload(a, seed):
    import dataclasses
    import workloads
    w = workloads.workload(a.workload, seed=seed, steps=pool_steps(a))
    if a.layers:
        w = dataclasses.replace(w, num_layers=max(1, min(a.layers, w.num_layers)))
    return w


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def describe(w, partition):
    return {
        "workload": f"{w.name}: {len(w.seq_ids)} seqs, {w.num_layers} layer(s), "
                    f"{w.num_q_heads} q / {w.num_kv_heads} KV heads, d{w.head_dim}, "
                    f"{w.kv_dtype} KV, block {w.block_size}",
        "seqs": len(w.seq_ids),
        "layers": w.num_layers,
        "q_heads": w.num_q_heads,
        "kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim,
        "block_size": w.block_size,
        "kv_dtype": w.kv_dtype,
        "pool_blocks": w.num_blocks,
        "partition_tokens": partition,
        "l2": "inputs larger than L2 (KV working set >> 126 MB); no flush",
    }


def step_bytes(w, lens_before):
    """Algorithmic HBM bytes of one step (all layers), and of its decode alone.

    decode: every cached token's K and V row once per (seq, KV head) + Q + O +
    one block-table entry per block; append: new K/V rows read + written.
    Shared blocks (parallel sampling) are counted once (distinct bytes).
    """
    kvb = 1 if w.kv_dtype == "fp8_e4m3" else 2
    n = len(w.seq_ids)
    row = 2 * w.num_kv_heads * w.head_dim * kvb           # K and V of one token, one layer
    tokens = sum(lens_before[s] + 1 for s in w.seq_ids)
    if w.forks:
        # distinct tokens: shared prompt blocks once per family
        fam = {}
        for parent, child in w.forks:
            fam.setdefault(parent, []).append(child)
        shared_full = 0
        for parent in fam:
            shared_full += (w.prefill_lens[parent] // w.block_size) * w.block_size * len(fam[parent])
        tokens -= shared_full
    blocks = sum(math.ceil((lens_before[s] + 1) / w.block_size) for s in w.seq_ids)
    qo = 2 * n * w.num_q_heads * w.head_dim * 2
    decode = tokens * row + qo + 4 * blocks
    append = n * 2 * w.num_kv_heads * w.head_dim * (2 + kvb)
    return w.num_layers * (decode + append), w.num_layers * decode


def logical_decode_bytes(w, lens_before):
    kvb = 1 if w.kv_dtype == "fp8_e4m3" else 2
    row = 2 * w.num_kv_heads * w.head_dim * kvb
    return w.num_layers * sum((lens_before[s] + 1) * row for s in w.seq_ids)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        # the step loop holds the interpreter between its library calls: switch
        # threads often enough that the sampler runs every few hundred us
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(0.0002)
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._nvml = None
        return self

    def _run(self):
        nv = self._nvml
        names = {
            0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
            0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, nm in names.items():
                    if r & bit:
                        self.reasons.add(nm)
            except Exception:
                break
            time.sleep(0.0005)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()
        sys.setswitchinterval(self._switch)

    def summary(self):
        return {
            "sm_mhz": statistics.median(self.samples) if self.samples else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(self.reasons),
            "samples": len(self.samples),
        }


def traffic_record(kernel_key):
    """ncu DRAM bytes per decode launch, if recorded for this exact kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    r = rec.get(kernel_key)
    if not r or r.get("source_sha") != source_sha():
        return None
    return r


def source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "pagedattention_decode_03_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h", ".cpp")):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


# ======================================================================== ours
class Runner:
    """Pool + per-step inputs for one replica, driven through the C ABI."""

    def __init__(self, w, device, partition, seed):
        import torch
        import pagedattention_decode_03_b200 as pa
        self.torch, self.pa, self.w = torch, pa, w
        self.dev = device
        self.partition = partition
        self.fused = True
        gen = torch.Generator(device=device)
        gen.manual_seed(1000 + seed)
        act = torch.bfloat16 if w.act_dtype == "bf16" else torch.float16
        self.act = act
        L, H, Hq, d = w.num_layers, w.num_kv_heads, w.num_q_heads, w.head_dim
        kw = {}
        if w.kv_dtype == "fp8_e4m3":
            # calibration as the tests use it: separate K and V scales per
            # (layer, head), amax/448 over every value the replica writes
            # (prefill and the step inputs below)
            amax_k = torch.zeros((L, H), dtype=torch.float32, device=device)
            amax_v = torch.zeros((L, H), dtype=torch.float32, device=device)
        self.scales = None
        # prefill data per (layer, seq) generated on the device
        self.prefill_data = {}
        for layer in range(L):
            for s, n in w.prefill_lens.items():
                k = torch.randn((n, H, d), generator=gen, device=device, dtype=torch.float32).to(act)
                v = torch.randn((n, H, d), generator=gen, device=device, dtype=torch.float32).to(act)
                self.prefill_data[(layer, s)] = (k, v)
                if w.kv_dtype == "fp8_e4m3":
                    amax_k[layer] = torch.maximum(amax_k[layer], k.float().abs().amax(dim=(0, 2)))
                    amax_v[layer] = torch.maximum(amax_v[layer], v.float().abs().amax(dim=(0, 2)))
        # per-step inputs: a few distinct sets, cycled
        n = len(w.seq_ids)
        self.nsets = 4
        self.q = [torch.randn((L, n, Hq, d), generator=gen, device=device).to(act) for _ in range(self.nsets)]
        self.kn = [torch.randn((L, n, H, d), generator=gen, device=device).to(act) for _ in range(self.nsets)]
        self.vn = [torch.randn((L, n, H, d), generator=gen, device=device).to(act) for _ in range(self.nsets)]
        if w.kv_dtype == "fp8_e4m3":
            for kn, vn in zip(self.kn, self.vn):
                amax_k = torch.maximum(amax_k, kn.float().abs().amax(dim=(1, 3)))
                amax_v = torch.maximum(amax_v, vn.float().abs().amax(dim=(1, 3)))
            ks = (amax_k / 448.0).float().contiguous()
            vs = (amax_v / 448.0).float().contiguous()
            self.scales = (ks, vs, (1.0 / ks).float().contiguous(), (1.0 / vs).float().contiguous())
            kw = dict(k_scale=self.scales[0], v_scale=self.scales[1],
                      k_inv_scale=self.scales[2], v_inv_scale=self.scales[3])
        order = w.free_order()
        self.pool = pa.pa_pool_create(
            num_layers=L, num_kv_heads=H, block_size=w.block_size, num_blocks=w.num_blocks,
            max_seqs=w.max_seqs, max_blocks_per_seq=w.max_blocks_per_seq, kv_dtype=w.kv_dtype,
            act_dtype=w.act_dtype, free_order=order, device=device,
            min_partition_tokens=min(512, partition) if partition and partition > 0 else 0, **kw)
        for s in sorted(w.prefill_lens):
            plen = w.prefill_lens[s]
            pa.pa_alloc_blocks(self.pool, s, plen)
            for layer in range(L):
                k, v = self.prefill_data.pop((layer, s))
                pa.pa_append_kv(self.pool, layer, [s] * plen, list(range(plen)), k, v)
        for parent, child in w.forks:
            pa.pa_fork_cow(self.pool, parent, child)
        torch.cuda.synchronize(device)
        self.out = torch.empty((L, len(w.seq_ids), Hq, d), dtype=act, device=device)
        # per-layer device addresses, computed once (no tensor views inside the timed loop)
        self._ptrs = {}
        self.seqs = np.asarray(w.seq_ids, np.int32)
        self.lens = np.asarray([w.lens_before_step(0)[s] for s in w.seq_ids], np.int32)
        self.step_idx = 0
        self.L = pa.lib()
        self.i32p = ctypes.POINTER(ctypes.c_int32)

    def lens_dict(self):
        return {s: int(n) for s, n in zip(self.w.seq_ids, self.lens)}

    def step(self, stream, q=None, kn=None, vn=None, out=None, dec_events=None):
        """One decode step through the C ABI (host arrays prebuilt)."""
        w, L = self.w, self.L
        k = self.step_idx % self.nsets
        q = self.q[k] if q is None else q
        kn = self.kn[k] if kn is None else kn
        vn = self.vn[k] if vn is None else vn
        out = self.out if out is None else out
        key = (q.data_ptr(), kn.data_ptr(), vn.data_ptr(), out.data_ptr())
        ptrs = self._ptrs.get(key)
        if ptrs is None:
            ptrs = [tuple(ctypes.c_void_p(t[layer].data_ptr()) for t in (q, kn, vn, out))
                    for layer in range(w.num_layers)]
            self._ptrs[key] = ptrs
        n = len(self.seqs)
        new = self.lens + 1
        done = ctypes.c_int32()
        sp = self.seqs.ctypes.data_as(self.i32p)
        st = L.pa_alloc_blocks_n(self.pool.handle, n, sp, new.ctypes.data_as(self.i32p), stream,
                                 ctypes.byref(done))
        if st != 0:
            raise RuntimeError(f"pa_alloc_blocks_n: {self.pa.pa_last_error()}")
        pos = self.lens.ctypes.data_as(self.i32p)
        scale = ctypes.c_float(w.scale)
        if dec_events is not None:   # the layer loop, back to back: launch overlap intact
            dec_events[0].record()
        for layer in range(w.num_layers):
            pq, pk, pv, po = ptrs[layer]
            if not self.fused:
                st = L.pa_append_kv(self.pool.handle, layer, n, sp, pos, pk, pv, stream)
                if st != 0:
                    raise RuntimeError(f"pa_append_kv: {self.pa.pa_last_error()}")
            if self.fused:   # append of the step's token and decode in one launch
                st = L.pa_decode_attention_append(self.pool.handle, layer, n, sp, pk, pv, w.num_q_heads,
                                                  pq, po, scale, self.partition, stream)
            else:
                st = L.pa_decode_attention(self.pool.handle, layer, n, sp, w.num_q_heads, pq, po, scale,
                                           self.partition, stream)
            if st != 0:
                raise RuntimeError(f"pa_decode_attention: {self.pa.pa_last_error()}")
        if dec_events is not None:
            dec_events[1].record()
        self.lens = new
        self.step_idx += 1


def reduce_ranks(vals, op, device, world):
    """Max or sum of per-rank floats over all ranks (identity for one rank)."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(
        t, op=torch.distributed.ReduceOp.MAX if op == "max" else torch.distributed.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def steps_of(a):
    return BENCH_STEPS[a.workload] if a.steps is None else a.steps


def run_ours(a, rank, world, local_rank):
    import torch
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    # All work of the replica runs on a stream of its own, as in a serving
    # engine: the library then launches each kernel with programmatic stream
    # serialization, so a decode launch's prologue overlaps the tail of the
    # previous one (on the legacy default stream every launch waits for the
    # previous kernel to end).
    with torch.cuda.stream(torch.cuda.Stream(device)):
        return _run_ours(a, rank, world, local_rank, device)


def _run_ours(a, rank, world, local_rank, device):
    import torch
    from pagedattention_decode_03_b200 import build as _b
    if rank == 0 or world == 1:
        _b.build()
    if world > 1:
        torch.distributed.barrier()
    w = make_workload(a, a.seed + rank)
    partition = w.partition_tokens if a.partition is None else a.partition
    r = Runner(w, device, partition, a.seed + rank)
    r.fused = not a.separate_append
    r.pa.pa_set_decode_path(r.pool, a.decode_path)
    stream_obj = torch.cuda.current_stream(device)
    stream = ctypes.c_void_p(stream_obj.cuda_stream)
    pa = r.pa

    for _ in range(a.warmup):
        r.step(stream)
    torch.cuda.synchronize(device)

    lens0 = r.lens_dict()
    bytes_step = [step_bytes(w, {s: lens0[s] + i for s in lens0}) for i in range(a.steps)]
    total_bytes = sum(b for b, _ in bytes_step)
    # bytes of the kernels inside the layer loop: the decode plus, when fused,
    # the step's append (separate appends are launched inside the loop too)
    loop_bytes = [b for b, _ in bytes_step]
    logical = sum(logical_decode_bytes(w, {s: lens0[s] + i for s in lens0}) for i in range(a.steps))
    # the layer loop of every step is bracketed by two events: inside it the
    # decode launches run back to back, each overlapping its neighbour's
    # prologue as in an untimed step (an event between two launches would
    # stop the second from starting early)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(a.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = pa.pa_launch_count(r.pool)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index) as clk:
        start.record()
        host_t = []
        for i in range(a.steps):
            h0 = time.perf_counter()
            r.step(stream, dec_events=ev[i])
            host_t.append(time.perf_counter() - h0)
        host_ms = sum(host_t) * 1e3   # host time to enqueue the K steps
        end.record()
        torch.cuda.synchronize(device)
    launches = pa.pa_launch_count(r.pool) - launches0
    ms = start.elapsed_time(end)
    loop_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bits = pa.pa_check_device_errors(r.pool)
    # every rank takes the same collectives, errors included
    ms, bits = reduce_ranks([ms, float(bits)], "max", device, world)
    total_bytes, = reduce_ranks([float(total_bytes)], "sum", device, world)
    if bits:
        raise RuntimeError(f"device error bits 0x{int(bits):x}")

    # ---- end to end: host (pinned) inputs in, output back, every step.  Copies
    # overlap the compute as a serving loop would: step i+1's inputs travel to a
    # second device set on one copy stream while step i computes, and step i's
    # output travels back on another while step i+1 computes; events order every
    # reuse of a buffer.  The first step's inputs and the last step's output are
    # inside the timed region, not overlapped.
    e2e = None
    if not a.no_e2e:
        comp = torch.cuda.current_stream(device)
        cs_in, cs_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        hq = torch.empty_like(r.q[0], device="cpu").pin_memory()
        hk = torch.empty_like(r.kn[0], device="cpu").pin_memory()
        hv = torch.empty_like(r.vn[0], device="cpu").pin_memory()
        ho = torch.empty_like(r.out, device="cpu").pin_memory()
        hq.copy_(r.q[0].cpu()); hk.copy_(r.kn[0].cpu()); hv.copy_(r.vn[0].cpu())
        din = [(torch.empty_like(r.q[0]), torch.empty_like(r.kn[0]), torch.empty_like(r.vn[0])) for _ in range(2)]
        dout = [torch.empty_like(r.out) for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]    # set j's inputs are on the device
        ev_done = [torch.cuda.Event() for _ in range(2)]  # the step that used set j has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]   # output j is back on the host

        def h2d(j, after=None):
            with torch.cuda.stream(cs_in):
                if after is not None:
                    cs_in.wait_event(after)
                cs_in.wait_event(ev_done[j])
                for d, h in zip(din[j], (hq, hk, hv)):
                    d.copy_(h, non_blocking=True)
                ev_in[j].record(cs_in)

        def d2h(j):
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(ev_done[j])
                ho.copy_(dout[j], non_blocking=True)
                ev_out[j].record(cs_out)

        def run_steps(k, s0=None):
            h2d(0, s0)
            for i in range(k):
                j = i & 1
                if i + 1 < k:
                    h2d(1 - j)
                comp.wait_event(ev_in[j])
                comp.wait_event(ev_out[j])   # output j's previous trip back is done
                r.step(stream, *din[j], dout[j])
                ev_done[j].record(comp)
                d2h(j)
            comp.wait_event(ev_out[(k - 1) & 1])

        run_steps(a.warmup)
        torch.cuda.synchronize(device)
        lens1 = r.lens_dict()
        e2e_bytes = sum(step_bytes(w, {s: lens1[s] + i for s in lens1})[0] for i in range(a.steps))
        if world > 1:
            torch.distributed.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(device)
        s0.record(comp)
        run_steps(a.steps, s0)
        s1.record(comp)
        torch.cuda.synchronize(device)
        e_ms, = reduce_ranks([s0.elapsed_time(s1)], "max", device, world)
        e2e_bytes, = reduce_ranks([float(e2e_bytes)], "sum", device, world)
        e2e = {"value": e2e_bytes / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel()) * 2,
               "d2h_bytes_per_step": ho.numel() * 2, "ms_per_step": e_ms / a.steps,
               "copies": "pinned host <-> device on two copy streams, overlapping the previous / next step"}

    peak, peak_src = peaks()
    value = total_bytes / (ms * 1e-3) / 1e9          # bytes of all ranks / max time
    launch_ms = sum(loop_ms) / (len(loop_ms) * w.num_layers)     # per layer
    launch_bytes = sum(loop_bytes) / (len(loop_bytes) * w.num_layers)
    achieved = launch_bytes / (launch_ms * 1e-3) / 1e9
    kern = pa.pa_last_decode_kernel(r.pool)
    tr = traffic_record(f"{w.name}:decode" + ("_tcgen05" if kern == "tcgen05" else ""))
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "pct_of_peak": round(100 * value / world / peak, 1),
        "decode_tokens_per_s": round(world * len(w.seq_ids) * a.steps / (ms * 1e-3), 1),
        "n_gpus": world,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": round(ms / a.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.kv_dtype if w.kv_dtype != "fp8_e4m3" else "fp8_e4m3 KV / bf16 act",
        "data": "synthetic (seeded N(0,1) K/V/Q, seeded lengths and block placement)",
        "device": torch.cuda.get_device_name(device),
        "config": {**describe(w, partition), "parallelism": f"replicas x{world} (no exchange step)"},
        "roofline": {
            "kernel": ("decode attention" + (" with the step's append fused" if r.fused else
                                             ", after a separate append launch") +
                       " (decode kernel, + reduce kernel for fixed partitions): every step's layer "
                       "loop timed as a whole, per layer"),
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            # ncu dram read+write of one captured launch of this kernel, scaled to this
            # launch's algorithmic bytes (same workload, a few tokens shorter)
            "traffic": (int(tr["ratio_to_algorithmic"] * launch_bytes) if tr else None),
            "traffic_over_algorithmic": tr["ratio_to_algorithmic"] if tr else None,
            "algorithmic_bytes_per_launch": int(launch_bytes),
            "launch_ms": round(launch_ms, 5),
            "ncu_launch_us": tr.get("duration_us") if tr else None,
        },
        "logical_decode_gbs": round(world * logical / (ms * 1e-3) / 1e9, 1),
        "gpu_launches": int(launches),
        "step_loop_ms": {"min": round(min(loop_ms), 4), "median": round(statistics.median(loop_ms), 4),
                         "max": round(max(loop_ms), 4)},
        "host_enqueue_ms_per_step": round(host_ms / a.steps, 4),
        # the first timed step starts with an empty launch queue, so its host
        # time is the enqueue cost itself; later steps can wait for queue room
        "host_enqueue_first_step_ms": round(host_t[0] * 1e3, 4),
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    line["config"]["append"] = ("fused into the decode launch (pa_decode_attention_append)" if r.fused
                                else "separate launch (pa_append_kv)")
    line["config"]["decode_kernel"] = kern
    if w.name == "tiny":
        line["graph_batch"] = graph_batch(r, 1000)
    if rank == 0 and not a.no_cpu:
        line["cpu_baseline"] = cpu_baseline(w, a.cpu_seconds, lens0)
    if rank == 0 and not a.no_swap:
        line["swap"] = swap_probe(device)
    return line


def swap_probe(device, reps=5):
    """Host transfer of one preempted sequence, outside the timed step: the
    1,525-token request of "Managing the KV Cache", Hands-On Exercise, in a pool
    of its 80-layer, 8-KV-head bf16 model, swapped out to pinned host memory and
    back (pa_swap_out / pa_swap_in: whole allocated blocks, every layer, K and
    V), timed with CUDA events on the launching stream after one warm-up round
    trip.  Reports the allocated bytes moved, the useful-state bytes they hold
    and the achieved GB/s each way; an error is reported, not raised."""
    import torch
    import pagedattention_decode_03_b200 as pa
    n, L, H = 1525, 80, 8
    nb = -(-n // 16)
    pool = img = None
    try:
        pool = pa.pa_pool_create(num_layers=L, num_kv_heads=H, block_size=16, num_blocks=nb,
                                 max_seqs=1, max_blocks_per_seq=nb, kv_dtype="bf16", device=device)
        pa.pa_alloc_blocks(pool, 0, n)
        size = pa.pa_swap_bytes(pool, n)
        img = torch.empty(size, dtype=torch.uint8, pin_memory=True)
        s = torch.cuda.current_stream(device)
        t_out, t_in = [], []
        for rep in range(reps + 1):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record(s)
            pa.pa_swap_out(pool, 0, img, s)
            ev[1].record(s)
            pa.pa_swap_in(pool, 0, n, img, s)
            ev[2].record(s)
            torch.cuda.synchronize(device)
            if rep:
                t_out.append(ev[0].elapsed_time(ev[1]))
                t_in.append(ev[1].elapsed_time(ev[2]))
        out_ms, in_ms = statistics.median(t_out), statistics.median(t_in)
        # the roofline of a swap is the host link: one contiguous copy of the
        # same bytes each way between a device buffer and the pinned image
        dev = torch.empty(size, dtype=torch.uint8, device=device)
        l_out, l_in = [], []
        for rep in range(reps + 1):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record(s)
            img.copy_(dev, non_blocking=True)
            ev[1].record(s)
            dev.copy_(img, non_blocking=True)
            ev[2].record(s)
            torch.cuda.synchronize(device)
            if rep:
                l_out.append(ev[0].elapsed_time(ev[1]))
                l_in.append(ev[1].elapsed_time(ev[2]))
        del dev
        link_out = size / (statistics.median(l_out) * 1e-3) / 1e9
        link_in = size / (statistics.median(l_in) * 1e-3) / 1e9
        out_gbs, in_gbs = size / (out_ms * 1e-3) / 1e9, size / (in_ms * 1e-3) / 1e9
        return {"tokens": n, "layers": L, "kv_heads": H, "dtype": "bf16",
                "allocated_bytes": size, "useful_bytes": n * 2 * L * H * 128 * 2,
                "out_ms": round(out_ms, 3), "in_ms": round(in_ms, 3),
                "out_gbs": round(out_gbs, 2), "in_gbs": round(in_gbs, 2),
                "roofline": {"bound": "host link", "unit": "GB/s",
                             "peak_out": round(link_out, 2), "peak_in": round(link_in, 2),
                             "peak_source": "measured: one contiguous cudaMemcpyAsync of the same "
                                            "bytes each way, device buffer <-> pinned host",
                             "frac_out": round(out_gbs / link_out, 4),
                             "frac_in": round(in_gbs / link_in, 4)},
                "host_memory": "pinned", "reps": reps}
    except Exception as ex:  # a failed probe must not cost the benchmark line
        return {"error": f"{type(ex).__name__}: {ex}"[:300]}
    finally:
        if pool is not None:
            torch.cuda.synchronize(device)
            pa.pa_pool_destroy(pool)
        del img


def graph_batch(r, reps):
    """GPU time of one decode launch of a launch-bound workload: `reps` decodes of
    layer 0 (same lengths, no appends) captured in one CUDA graph and replayed
    once.  L2-warm (the tiny KV pool stays in L2), so it shows the launch and
    ramp cost, not HBM bandwidth."""
    import torch
    w, L = r.w, r.L
    n = len(r.seqs)
    sp = r.seqs.ctypes.data_as(r.i32p)
    q, out = ctypes.c_void_p(r.q[0][0].data_ptr()), ctypes.c_void_p(r.out[0].data_ptr())
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        cs = ctypes.c_void_p(side.cuda_stream)
        for _ in range(reps):
            st = L.pa_decode_attention(r.pool.handle, 0, n, sp, w.num_q_heads, q, out,
                                       ctypes.c_float(w.scale), r.partition, cs)
            if st != 0:
                raise RuntimeError(f"pa_decode_attention (graph capture): {r.pa.pa_last_error()}")
    torch.cuda.synchronize()
    g.replay()                      # warm-up replay
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return {"launches": reps, "us_per_decode": round(e0.elapsed_time(e1) * 1e3 / reps, 2),
            "note": "L2-warm: one decode of layer 0 replayed from a CUDA graph"}


# ==================================================================== oracle
def _oracle_setup(w, lens_before, seqs):
    """Oracle pool holding the sample sequences at `lens_before`."""
    from oracle import PagedKVOracle
    from workloads import prefill_kv_bits, step_kv_bits
    order = w.free_order()
    o = PagedKVOracle(num_layers=w.num_layers, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                      block_size=w.block_size, num_blocks=w.num_blocks, max_seqs=w.max_seqs,
                      max_blocks_per_seq=w.max_blocks_per_seq, kv_dtype=w.kv_dtype,
                      free_order=order, stored_layers=[0])
    ki = vi = None
    if w.kv_dtype == "fp8_e4m3":
        from workloads import fp8_scales
        sc = fp8_scales(w, 0)
        ki, vi = sc[2], sc[3]
        o._scales = sc
    for s in seqs:
        n = w.prefill_lens.get(s, lens_before[s])
        o.reserve(s, n)
        k, v = prefill_kv_bits(w, 0, s, n)
        o.append(0, [s] * n, list(range(n)), k, v, w.act_dtype, ki, vi)
    return o


class OracleSample:
    """The oracle holding a bounded sample of the workload: the first (up to)
    16 sequences, layer 0.  One step = reserve + append + float64 attention
    for those sequences, as the GPU step does for all of them."""

    def __init__(self, w, lens_before):
        seqs = list(w.seq_ids)[: max(1, min(len(w.seq_ids), 16))]
        if w.forks:
            seqs = [s for s in seqs if s in w.prefill_lens][:4]
        self.w, self.seqs = w, seqs
        self.o = _oracle_setup(w, lens_before, seqs)
        self.lens = {s: self.o.lens[s] for s in seqs}
        self.idx = [w.seq_ids.index(s) for s in seqs]
        self.sub = _subset(w, seqs)
        self.k = 0

    def step(self):
        from workloads import step_kv_bits, step_q_bits
        w, o, seqs = self.w, self.o, self.seqs
        ki = vi = ks = vs = None
        if w.kv_dtype == "fp8_e4m3":
            ks, vs, ki, vi = o._scales
        for s in seqs:
            o.reserve(s, self.lens[s] + 1)
        k, v = step_kv_bits(w, self.k, 0)
        o.append(0, seqs, [self.lens[s] for s in seqs], k[self.idx], v[self.idx], w.act_dtype, ki, vi)
        q = step_q_bits(w, self.k, 0)[self.idx]
        o.attention(0, seqs, q, w.act_dtype, w.scale, ks, vs)
        nbytes = step_bytes(self.sub, self.lens)[0] / w.num_layers
        for s in seqs:
            self.lens[s] += 1
        self.k += 1
        return nbytes


def _threads():
    from threadpoolctl import threadpool_info
    return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])


def cpu_baseline(w, seconds, lens_before, kind="oracle"):
    """Time the float64 oracle on the host cores on a bounded sample."""
    smp = OracleSample(w, lens_before)
    t0 = time.perf_counter()
    steps = 0
    nbytes = 0.0
    while (time.perf_counter() - t0 < seconds and steps < 200) or steps == 0:
        nbytes += smp.step()
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": _threads(),
            "host_cpus": os.cpu_count(), "kind": kind,
            "sample": f"{steps} decode step(s) of layer 0 for {len(smp.seqs)} of {len(w.seq_ids)} "
                      f"sequences (reserve + append + float64 attention), {dt:.1f} s"}


def _subset(w, seqs):
    import dataclasses
    return dataclasses.replace(w, seq_ids=tuple(seqs), forks=(),
                               prefill_lens={s: w.prefill_lens.get(s, 0) for s in seqs})


def run_reference(a):
    import workloads
    w = make_workload(a, a.seed)
    partition = w.partition_tokens if a.partition is None else a.partition
    lens0 = w.lens_before_step(0)
    smp = OracleSample(w, lens0)
    for _ in range(a.warmup):
        smp.step()
    nbytes = 0.0
    t0 = time.perf_counter()
    for _ in range(a.steps):
        nbytes += smp.step()
    dt = time.perf_counter() - t0
    value = round(nbytes / dt / 1e9, 4)
    sample = (f"each step: one decode step of layer 0 for {len(smp.seqs)} of {len(w.seq_ids)} "
              f"sequences (reserve + append + float64 attention)")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": a.gpus, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(1000 * dt / a.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) K/V/Q, seeded lengths and block placement)",
        "config": {**describe(w, partition), "parallelism": "host cores"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": _threads(), "host_cpus": os.cpu_count(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    a = parse()
    a.steps = steps_of(a)
    if a.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(a)), flush=True)
        return
    import torch
    import datetime
    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(a, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
