"""Pins the oracle's decode attention.

* brute force: scalar loops that walk each sequence's block table slot by
  slot (no gather, no matrix products) and build the softmax with math.exp;
* special cases with closed forms: one token (output = that V row
  exactly), identical keys (output = mean of V), constant V (output = V);
* a library cross-check: torch's scaled_dot_product_attention in float64
  over the gathered, GQA-expanded K/V;
* placement invariance: permuting physical block ids (pool contents and
  tables together) changes nothing ("kv-cache-pagedattention-serving",
  PagedAttention: blocks stored anywhere in physical GPU memory).
"""
import math

import numpy as np
import pytest
import torch

from oracle import PagedKVOracle, Status, fp8
from workloads import normal_bits


def _bf16_scalar(bits):
    import struct
    return struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0]


def _fp16_scalar(bits):
    import struct
    return struct.unpack("<e", struct.pack("<H", int(bits)))[0]


def _scalar(bits, dtype):
    """One 16-bit pattern to a Python float, by the struct codecs (binary32
    upper half for bf16, binary16 for fp16), independent of the oracle."""
    return _bf16_scalar(bits) if dtype == "bf16" else _fp16_scalar(bits)


def build(lens, H=2, G=2, d=8, B=4, nb=40, kv="bf16", act="bf16", seed=0, order=None):
    g = np.random.default_rng(seed)
    o = PagedKVOracle(num_layers=2, num_kv_heads=H, head_dim=d, block_size=B, num_blocks=nb,
                      max_seqs=len(lens), max_blocks_per_seq=64, kv_dtype=kv,
                      free_order=g.permutation(nb) if order is None else order)
    k_inv = v_inv = k_scale = v_scale = None
    if kv == "fp8_e4m3":
        k_scale = np.full((2, H), 0.011, np.float32) * (1 + np.arange(H, dtype=np.float32))
        v_scale = np.full((2, H), 0.009, np.float32) * (1 + np.arange(H, dtype=np.float32))
        k_inv = (np.float32(1) / k_scale).astype(np.float32)
        v_inv = (np.float32(1) / v_scale).astype(np.float32)
    for s, n in enumerate(lens):
        assert o.reserve(s, n) is Status.OK
        for layer in range(2):
            k = normal_bits(g, (n, H, d), act)
            v = normal_bits(g, (n, H, d), act)
            assert o.append(layer, [s] * n, list(range(n)), k, v, act, k_inv, v_inv) is Status.OK
    q = normal_bits(g, (len(lens), H * G, d), act)
    return o, q, (k_scale, v_scale)


def brute_force(o, layer, lens, q_bits, scale, scales=(None, None), act="bf16"):
    """Scalar-loop attention straight off the pool, one slot at a time."""
    k_scale, v_scale = scales
    n_seq, hq, d = q_bits.shape
    G = hq // o.H
    out = np.zeros((n_seq, hq, d))
    sc = float(np.float32(scale))
    for s in range(n_seq):
        for qh in range(hq):
            h = qh // G
            qv = [_scalar(q_bits[s, qh, j], act) for j in range(d)]
            logits = []
            for t in range(lens[s]):
                blk = o.tables[s][t // o.B]
                row = o.k[layer][blk, h, t % o.B]
                if o.kv_dtype == "fp8_e4m3":
                    kv = [float(fp8.decode([row[j]])[0]) * float(k_scale[layer][h]) for j in range(d)]
                else:
                    kv = [_scalar(row[j], o.kv_dtype) for j in range(d)]
                acc = 0.0
                for j in range(d):
                    acc += qv[j] * kv[j]
                logits.append(acc * sc)
            mx = max(logits)
            w = [math.exp(x - mx) for x in logits]
            tot = sum(w)
            for t in range(lens[s]):
                blk = o.tables[s][t // o.B]
                row = o.v[layer][blk, h, t % o.B]
                for j in range(d):
                    if o.kv_dtype == "fp8_e4m3":
                        vj = float(fp8.decode([row[j]])[0]) * float(v_scale[layer][h])
                    else:
                        vj = _scalar(row[j], o.kv_dtype)
                    out[s, qh, j] += w[t] / tot * vj
    return out


@pytest.mark.parametrize("G", [1, 2, 4])
def test_matches_scalar_brute_force(G):
    lens = [1, 3, 4, 5, 13]
    o, q, _ = build(lens, G=G, seed=G)
    for layer in (0, 1):
        got = o.attention(layer, range(len(lens)), q, "bf16", 0.35)
        want = brute_force(o, layer, lens, q, 0.35)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("G", [1, 4])
def test_fp16_matches_scalar_brute_force(G):
    lens = [1, 6, 11]
    o, q, _ = build(lens, G=G, kv="fp16", act="fp16", seed=20 + G)
    for layer in (0, 1):
        got = o.attention(layer, range(len(lens)), q, "fp16", 0.35)
        want = brute_force(o, layer, lens, q, 0.35, act="fp16")
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_fp8_matches_scalar_brute_force():
    lens = [2, 7, 9]
    o, q, scales = build(lens, G=2, kv="fp8_e4m3", seed=5)
    got = o.attention(1, range(3), q, "bf16", 0.35, *scales)
    want = brute_force(o, 1, lens, q, 0.35, scales)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_single_token_returns_that_value_row_exactly():
    o, q, _ = build([1, 1], G=4, seed=3)
    out = o.attention(0, [0, 1], q, "bf16", 0.088)
    for s in range(2):
        K, V = o.gather(0, s)
        for qh in range(8):
            assert (out[s, qh] == V[0, qh // 4]).all()


def test_identical_keys_give_mean_of_values():
    o, q, _ = build([37], H=1, G=2, seed=4)
    blk_rows = [(o.tables[0][t // o.B], t % o.B) for t in range(37)]
    for b, r in blk_rows:
        o.k[0][b, 0, r] = o.k[0][blk_rows[0][0], 0, blk_rows[0][1]]
    out = o.attention(0, [0], q, "bf16", 1.0)
    _, V = o.gather(0, 0)
    for qh in range(2):
        np.testing.assert_allclose(out[0, qh], V[:, 0].mean(axis=0), rtol=0, atol=1e-14)


def test_constant_values_pass_through():
    o, q, _ = build([29, 6], H=2, G=2, seed=6)
    c = np.uint16(0x3FC0)  # bf16 1.5
    for layer in (0,):
        o.v[layer][:] = c
    out = o.attention(0, [0, 1], q, "bf16", 0.2)
    np.testing.assert_allclose(out, 1.5, rtol=0, atol=1e-14)


def test_matches_torch_sdpa_float64():
    lens = [17, 64, 5, 33]
    o, q, _ = build(lens, H=2, G=4, d=16, B=16, nb=30, seed=9)
    got = o.attention(1, range(4), q, "bf16", 0.25)
    qf = (q.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for s, n in enumerate(lens):
        K, V = o.gather(1, s)
        Kx = torch.from_numpy(np.repeat(K.transpose(1, 0, 2), 4, axis=0))   # [Hq, n, d]
        Vx = torch.from_numpy(np.repeat(V.transpose(1, 0, 2), 4, axis=0))
        qs = torch.from_numpy(qf[s][:, None, :])                             # [Hq, 1, d]
        ref = torch.nn.functional.scaled_dot_product_attention(qs, Kx, Vx, scale=float(np.float32(0.25)))
        np.testing.assert_allclose(got[s], ref[:, 0].numpy(), rtol=1e-12, atol=1e-13)


def test_placement_invariance_exact():
    lens = [9, 31, 2]
    nb = 24
    o1, q, _ = build(lens, nb=nb, seed=12, order=np.arange(nb))
    perm = np.random.default_rng(13).permutation(nb)
    o2 = PagedKVOracle(num_layers=2, num_kv_heads=o1.H, head_dim=o1.d, block_size=o1.B,
                       num_blocks=nb, max_seqs=3, max_blocks_per_seq=64, kv_dtype="bf16",
                       free_order=perm)
    for s, n in enumerate(lens):
        assert o2.reserve(s, n) is Status.OK
    for s in range(3):
        for j, b in enumerate(o1.tables[s]):
            b2 = o2.tables[s][j]
            for layer in (0, 1):
                o2.k[layer][b2] = o1.k[layer][b]
                o2.v[layer][b2] = o1.v[layer][b]
    assert o1.tables != o2.tables
    for layer in (0, 1):
        a = o1.attention(layer, range(3), q, "bf16", 0.3)
        b = o2.attention(layer, range(3), q, "bf16", 0.3)
        assert (a == b).all()
