"""Paged KV pool, cache contents and decode attention (oracle).

Test infrastructure only: imported by tests, the smoke check and the
benchmark's CPU leg.  Nothing here is called by the library.

What the pages define, and how this model reads it:

* The cache is cut into fixed-size blocks of `block_size` token slots that
  live anywhere in one physical pool; each sequence owns a block table
  mapping logical block j to a physical block ("KV cache", The maths and
  its paging paragraph; kv-cache-pagedattention-serving, PagedAttention:
  virtual memory for GPUs).
* Blocks are handed out only as a sequence grows, one free block per block
  boundary crossed ("Managing the KV Cache", Answer Key item 2), and go
  back to the free list once no sequence references them ("Managing the KV
  Cache", Block Tables and Sharing).
* Several sequences may reference the same immutable blocks through
  reference counts; a fresh block is taken only when a sequence is about to
  write into a tail block that others still share, and the shared block is
  copied first (copy-on-write; "Managing the KV Cache", Block Tables and
  Sharing; kv-cache-pagedattention-serving, The bonus: sharing via
  copy-on-write).
* Attention for a sequence runs over every cached token of that sequence
  in logical order ("kv-cache-pagedattention-serving", PagedAttention:
  virtual memory for GPUs).  This oracle deliberately gathers the blocks
  into a contiguous buffer first, which is the plain definition the fused
  kernel must reproduce.

Readings where the pages are silent:

* free list is FIFO: allocate from the head, release to the tail, in
  logical-block order; its initial order is given by the caller;
* a reservation that needs both a copy-on-write block and new blocks takes
  the copy-on-write block first; the number of blocks needed is checked
  before anything changes, so a failed reservation leaves no trace;
* the copy-on-write copy covers the whole block for every layer, K and V;
* a query of head i attends through KV head floor(i / G), G = H_q / H_kv;
* no mask beyond the sequence length; the scale is a caller argument.

Block-granular prefix caching (kv-cache-pagedattention-serving, Beyond
paging: radix trees and continuous batching; "Managing the KV Cache", Block
Tables and Sharing and Answer Key item 4): a full block whose KV the caller
has written may be registered under the token prefix it ends, i.e. all
tokens from the sequence start to the block's last slot (the KV of a token
depends on every token before it).  A new prompt reuses, from its first
block on, each full block whose whole prefix is registered, and stops at the
first one that is not; so a 103-token prompt reuses at most 96 tokens with
16-token blocks.  Registered blocks stay reference counted; when no sequence
references one it is kept, with its contents, on a least-recently-used list
and is evicted only when a block is needed and the free list is empty.
Readings where the pages are silent:

* a registered block is immutable: writing a slot of it is refused like a
  write into a shared block;
* the first registration of a prefix wins; registering another block with
  the same prefix leaves that block unregistered;
* when a release drops several registered blocks to zero references, they
  join the recently-used end in reverse logical order, so a longer prefix
  is evicted before the shorter prefix it extends (a block is only reached
  through its predecessors);
* a prompt whose every token falls in registered blocks reuses all of them
  (whether the last token is recomputed to get logits is a scheduler's
  choice, outside the pool).

Swap-out / swap-in ("Managing the KV Cache", Offload and Hands-On Exercise;
kv-cache-pagedattention-serving, Beyond paging: radix trees and continuous
batching): a preempted sequence's KV moves to host memory and its blocks go
back to the pool; paging it back takes fresh blocks and restores every
cached token.  Readings where the pages are silent:

* the transfer moves whole allocated blocks (the exercise asks for both the
  useful-state and the allocated-block byte counts; a block-granular copy
  moves the latter), every layer, K and V, as raw storage bits;
* the host image is laid out [K, V][logical block][layer][kv_head][slot][dim];
* swap-out releases the sequence exactly as a release does; swap-in creates
  it again with private blocks (sharing with forks is not restored).
"""
from __future__ import annotations

import collections
import enum

import numpy as np

from . import fp8 as _fp8
from .numerics import bits_to_f32, bits_to_f64


class Status(enum.Enum):
    OK = "ok"
    INVALID_ARG = "invalid_arg"
    NO_BLOCKS = "no_blocks"
    NO_SEQ = "no_seq"
    SEQ_EXISTS = "seq_exists"
    SHARED_BLOCK = "shared_block"


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


class PagedKVOracle:
    """Block pool + cache contents + float64 attention.

    Cache arrays use the pool layout [layer][block][kv_head][slot][head_dim]
    and hold raw storage bits (uint16 for bf16 / fp16, uint8 codes for FP8).
    `stored_layers` limits which layers keep contents (all by default), so
    large workloads can be checked layer by layer.
    """

    def __init__(self, *, num_layers: int, num_kv_heads: int, head_dim: int, block_size: int,
                 num_blocks: int, max_seqs: int, max_blocks_per_seq: int, kv_dtype: str,
                 free_order=None, stored_layers=None):
        self.L, self.H, self.d, self.B = num_layers, num_kv_heads, head_dim, block_size
        self.num_blocks, self.max_seqs, self.mbps = num_blocks, max_seqs, max_blocks_per_seq
        self.kv_dtype = kv_dtype
        order = range(num_blocks) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the block ids")
        self.free = collections.deque(order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.cow_log: list[tuple[int, int]] = []
        # prefix cache: whole-token-prefix tuple -> block, block -> prefix, and
        # the registered blocks nothing references, least recently used first
        self.registry: dict[tuple, int] = {}
        self.key_of: dict[int, tuple] = {}
        self.cached: collections.OrderedDict[int, None] = collections.OrderedDict()
        layers = range(num_layers) if stored_layers is None else stored_layers
        store = np.uint8 if kv_dtype == "fp8_e4m3" else np.uint16
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k = {layer: np.zeros(shape, store) for layer in layers}
        self.v = {layer: np.zeros(shape, store) for layer in layers}

    # ------------------------------------------------------------------ pool
    def reserve(self, seq: int, new_len: int) -> Status:
        """Grow (or create) `seq` to hold `new_len` tokens."""
        if not 0 <= seq < self.max_seqs or new_len < 0:
            return Status.INVALID_ARG
        table = self.tables.get(seq, [])
        cur = self.lens.get(seq, 0)
        if new_len < cur or _ceil_div(new_len, self.B) > self.mbps:
            return Status.INVALID_ARG
        cow = new_len > cur and cur % self.B != 0 and self.ref[table[-1]] > 1
        grow = _ceil_div(new_len, self.B) - len(table)
        if int(cow) + grow > len(self.free) + len(self.cached):
            return Status.NO_BLOCKS
        table = list(table)
        if cow:
            src = table[-1]
            dst = self._take()
            for layer in self.k:
                self.k[layer][dst] = self.k[layer][src]
                self.v[layer][dst] = self.v[layer][src]
            self.ref[src] -= 1
            self.ref[dst] = 1
            table[-1] = dst
            self.cow_log.append((src, dst))
        for _ in range(grow):
            b = self._take()
            self.ref[b] = 1
            table.append(b)
        self.tables[seq] = table
        self.lens[seq] = new_len
        return Status.OK

    def _take(self) -> int:
        """A block for new contents: the free list's head, else the least
        recently used cached block, which then leaves the prefix registry."""
        if self.free:
            return self.free.popleft()
        b, _ = self.cached.popitem(last=False)
        del self.registry[self.key_of.pop(b)]
        return b

    def fork(self, parent: int, child: int) -> Status:
        """`child` shares every block of `parent` (reference count + 1)."""
        if not 0 <= child < self.max_seqs or not 0 <= parent < self.max_seqs:
            return Status.INVALID_ARG
        if parent not in self.tables:
            return Status.NO_SEQ
        if child in self.tables:
            return Status.SEQ_EXISTS
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1
        return Status.OK

    def release(self, seq: int) -> Status:
        """Drop `seq`; blocks whose count reaches zero return to the free tail,
        registered ones to the recently-used end of the cached list instead."""
        if seq not in self.tables:
            return Status.NO_SEQ if 0 <= seq < self.max_seqs else Status.INVALID_ARG
        for b in self.tables[seq]:
            self.ref[b] -= 1
            if self.ref[b] == 0 and b not in self.key_of:
                self.free.append(b)
        for b in reversed(self.tables[seq]):
            if self.ref[b] == 0 and b in self.key_of:
                self.cached[b] = None
        del self.tables[seq]
        del self.lens[seq]
        return Status.OK

    def slot(self, seq: int, pos: int):
        """(physical block, slot in block) for token `pos` of `seq`, or a Status."""
        if seq not in self.tables:
            return Status.NO_SEQ
        if not 0 <= pos < self.lens[seq]:
            return Status.INVALID_ARG
        b = self.tables[seq][pos // self.B]
        if self.ref[b] > 1 or b in self.key_of:
            return Status.SHARED_BLOCK
        return b, pos % self.B

    # ---------------------------------------------------------- prefix cache
    def _prefix(self, tokens, i: int) -> tuple:
        """The token prefix that logical block i ends: tokens[0 : (i+1)*B]."""
        return tuple(int(t) for t in tokens[: (i + 1) * self.B])

    def register(self, seq: int, tokens) -> Status:
        """Register the full blocks of `seq` that `tokens` (its first n tokens,
        n <= length, KV already written) covers, each under its prefix."""
        if not 0 <= seq < self.max_seqs:
            return Status.INVALID_ARG
        if seq not in self.tables:
            return Status.NO_SEQ
        n = len(tokens)
        if n > self.lens[seq]:
            return Status.INVALID_ARG
        table = self.tables[seq]
        m = n // self.B
        for i in range(m):
            b = table[i]
            if b in self.key_of and self.key_of[b] != self._prefix(tokens, i):
                return Status.INVALID_ARG
        for i in range(m):
            b, key = table[i], self._prefix(tokens, i)
            if key not in self.registry and b not in self.key_of:
                self.registry[key] = b
                self.key_of[b] = key
        return Status.OK

    def match(self, tokens) -> int:
        """Number of leading full blocks of `tokens` whose prefix is registered."""
        m = 0
        while (m + 1) * self.B <= len(tokens) and self._prefix(tokens, m) in self.registry:
            m += 1
        return m

    def reserve_prefix(self, seq: int, tokens):
        """Create `seq` for the prompt `tokens`, reusing its cached leading
        blocks.  Returns (Status, number of prompt tokens whose KV is cached)."""
        n = len(tokens)
        if not 0 <= seq < self.max_seqs or _ceil_div(n, self.B) > self.mbps:
            return Status.INVALID_ARG, 0
        if seq in self.tables:
            return Status.SEQ_EXISTS, 0
        m = self.match(tokens)
        hit = [self.registry[self._prefix(tokens, i)] for i in range(m)]
        idle = sum(1 for b in hit if b in self.cached)
        need = _ceil_div(n, self.B) - m
        if need > len(self.free) + len(self.cached) - idle:
            return Status.NO_BLOCKS, 0
        for b in hit:
            self.cached.pop(b, None)
            self.ref[b] += 1
        table = list(hit)
        for _ in range(need):
            b = self._take()
            self.ref[b] = 1
            table.append(b)
        self.tables[seq] = table
        self.lens[seq] = n
        return Status.OK, m * self.B

    # ----------------------------------------------------------------- cache
    def append(self, layer: int, seqs, positions, k_bits, v_bits, act_dtype: str,
               k_inv=None, v_inv=None) -> Status:
        """Write one K row and one V row per (seq, pos) into its cache slot.

        `k_bits` / `v_bits`: [T, num_kv_heads, head_dim] activation bits.
        For an FP8 pool the stored code is E4M3(fp32(x * inv_scale[layer, h])).
        All targets are validated before anything is written.
        """
        slots = []
        for s, p in zip(seqs, positions):
            r = self.slot(int(s), int(p))
            if isinstance(r, Status):
                return r
            slots.append(r)
        if layer not in self.k:
            return Status.OK
        for t, (b, o) in enumerate(slots):
            if self.kv_dtype == "fp8_e4m3":
                xk = bits_to_f32(k_bits[t], act_dtype)
                xv = bits_to_f32(v_bits[t], act_dtype)
                self.k[layer][b, :, o, :] = _fp8.quantize(xk, np.asarray(k_inv[layer])[:, None])
                self.v[layer][b, :, o, :] = _fp8.quantize(xv, np.asarray(v_inv[layer])[:, None])
            else:
                self.k[layer][b, :, o, :] = k_bits[t]
                self.v[layer][b, :, o, :] = v_bits[t]
        return Status.OK

    def gather(self, layer: int, seq: int):
        """Contiguous float64 K and V of `seq`: [len, num_kv_heads, head_dim].

        FP8 values are decoded exactly; the per-head scale is applied by
        `attention`.
        """
        n = self.lens[seq]
        t = np.arange(n)
        blocks = np.asarray(self.tables[seq], dtype=np.int64)[t // self.B]
        kb = self.k[layer][blocks, :, t % self.B, :]
        vb = self.v[layer][blocks, :, t % self.B, :]
        if self.kv_dtype == "fp8_e4m3":
            return _fp8.decode(kb), _fp8.decode(vb)
        return bits_to_f64(kb, self.kv_dtype), bits_to_f64(vb, self.kv_dtype)

    def attention(self, layer: int, seqs, q_bits, act_dtype: str, scale: float,
                  k_scale=None, v_scale=None) -> np.ndarray:
        """softmax(scale * q K^T) V per (sequence, query head), float64.

        `q_bits`: [n, num_q_heads, head_dim] activation bits.  Query head i
        uses KV head i // G.  Returns float64 [n, num_q_heads, head_dim].
        """
        q = bits_to_f64(q_bits, act_dtype)
        n, hq, d = q.shape
        group = hq // self.H
        sc = float(np.float32(scale))
        out = np.zeros((n, hq, d), np.float64)
        for i, s in enumerate(seqs):
            K, V = self.gather(layer, int(s))
            for qh in range(hq):
                h = qh // group
                kh, vh = K[:, h, :], V[:, h, :]
                if self.kv_dtype == "fp8_e4m3":
                    kh = kh * float(k_scale[layer][h])
                    vh = vh * float(v_scale[layer][h])
                x = (kh @ q[i, qh]) * sc
                p = np.exp(x - x.max())
                p /= p.sum()
                out[i, qh] = p @ vh
        return out

    # ------------------------------------------------------------- swapping
    def swap_bytes(self, n_tokens: int, bytes_per_element: int) -> int:
        """Size of the host image of an n-token sequence: its allocated blocks,
        every layer, K and V."""
        return (2 * _ceil_div(n_tokens, self.B) * self.L * self.H * self.B * self.d
                * bytes_per_element)

    def swap_out(self, seq: int):
        """(Status, host image, length): copy the blocks of `seq` out, then
        release it.  The image holds the stored layers only:
        [2][blocks][stored layers][kv_head][slot][dim] raw bits."""
        if seq not in self.tables:
            return (Status.NO_SEQ if 0 <= seq < self.max_seqs else Status.INVALID_ARG), None, 0
        table, n = self.tables[seq], self.lens[seq]
        layers = sorted(self.k)
        store = np.uint8 if self.kv_dtype == "fp8_e4m3" else np.uint16
        image = np.zeros((2, len(table), len(layers), self.H, self.B, self.d), store)
        for c, cache in enumerate((self.k, self.v)):
            for j, b in enumerate(table):
                for i, layer in enumerate(layers):
                    image[c, j, i] = cache[layer][b]
        self.release(seq)
        return Status.OK, image, n

    def swap_in(self, seq: int, n_tokens: int, image) -> Status:
        """Create `seq` with `n_tokens` tokens in fresh blocks and write the
        host image (as swap_out returns it) into them."""
        if not 0 <= seq < self.max_seqs:
            return Status.INVALID_ARG
        if seq in self.tables:
            return Status.SEQ_EXISTS
        st = self.reserve(seq, n_tokens)
        if st != Status.OK:
            return st
        for j, b in enumerate(self.tables[seq]):
            for i, layer in enumerate(sorted(self.k)):
                self.k[layer][b] = image[0][j][i]
                self.v[layer][b] = image[1][j][i]
        return Status.OK

    # ------------------------------------------------------------ inspection
    def table(self, seq: int) -> list[int]:
        return list(self.tables[seq])

    def free_list(self) -> list[int]:
        return list(self.free)

    def cached_list(self) -> list[int]:
        """Registered blocks with no reference, least recently used first."""
        return list(self.cached)

    def refcounts(self) -> list[int]:
        return list(self.ref)

    def check_invariants(self) -> None:
        """Pool invariants the pages imply; raises AssertionError if broken.

        * only a sequence's final block can be partly empty, so tail waste
          is at most block_size - 1 ("Managing the KV Cache", Internal
          Fragmentation);
        * a block is on the free list iff nothing references it ("Managing
          the KV Cache", Block Tables and Sharing);
        * every block is either free or referenced, never both, never twice
          on the free list; total references = total table entries;
        * a block that nothing references is either free or cached, and a
          cached block is registered; registry and key_of are inverse maps,
          and a registered prefix is a whole number of blocks long.
        """
        counted = [0] * self.num_blocks
        for seq, table in self.tables.items():
            n = self.lens[seq]
            assert len(table) == _ceil_div(n, self.B)
            assert len(table) * self.B - n <= self.B - 1
            for b in table:
                counted[b] += 1
        assert counted == self.ref
        free = list(self.free)
        assert len(set(free)) == len(free)
        idle = set(free) | set(self.cached)
        assert not set(free) & set(self.cached)
        assert idle == {b for b in range(self.num_blocks) if self.ref[b] == 0}
        assert len(free) + len(self.cached) + sum(1 for r in self.ref if r > 0) == self.num_blocks
        assert all(b in self.key_of for b in self.cached)
        assert not set(free) & set(self.key_of)
        assert {v: k for k, v in self.registry.items()} == self.key_of
        assert all(len(k) % self.B == 0 and len(k) > 0 for k in self.registry)
