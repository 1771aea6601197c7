/*
 * pa.h -- C ABI of the paged decode-attention library (libpa.so).
 *
 * The library implements single-query decode attention over a paged KV
 * cache on one NVIDIA B200 (sm_100a), plus the pieces that keep the cache:
 * a host-side block manager (free list, per-sequence block tables,
 * reference counts, copy-on-write of a shared tail block) and the kernel
 * that writes each step's new K/V rows into their cache slots.
 *
 * What the operations compute is fixed by three public pages:
 *   [KVC] "KV cache" (AI engineering visualised): The maths, and the
 *         paragraph on paged attention (block tables, blocks handed out as
 *         a sequence grows, waste bounded by one block);
 *   [MKV] "Managing the KV Cache": Reproduce Bytes per Token, Internal
 *         Fragmentation, Block Tables and Sharing, Quantized KV, Answer Key;
 *   [PAS] "kv-cache-pagedattention-serving": PagedAttention: virtual memory
 *         for GPUs; The bonus: sharing via copy-on-write; Beyond paging:
 *         radix trees and continuous batching (block-granular prefix cache).
 *
 * Conventions for every call:
 *   - Every call returns a pa_status.  Out-parameters are written only when
 *     the call returns PA_OK.
 *   - A call that fails on the host leaves the pool exactly as it was; in
 *     particular PA_ERR_NO_BLOCKS is detected before anything changes.
 *   - Device work is enqueued on the caller's stream and never waited for,
 *     except by pa_check_device_errors.  `stream` is a cudaStream_t passed
 *     as void*; NULL means the legacy default stream.  The pool's device
 *     metadata is updated in stream order: calls on one pool that use
 *     different streams must be ordered by the caller.
 *   - Kernels are launched with programmatic stream serialization (except
 *     on the legacy default stream): a launch may start its prologue while
 *     the previous kernel on the stream finishes, and waits for that kernel
 *     before it reads or writes anything earlier work may touch.  The one
 *     exception is a decode launch's L2 prefetch hints for its first cache
 *     tiles, which cannot change any result (the data is read again after
 *     the wait; L2 is coherent with every write).
 *   - The caller owns every device buffer (caches, scales, workspace,
 *     q / out / k_new / v_new) and keeps it alive while work that uses it is
 *     in flight.  The pool owns only host memory.
 *   - A pool is not thread-safe; use one pool per host thread or lock.
 *   - Sequence ids are integers in [0, max_seqs).
 *   - pa_last_error() returns a description of the last failure on the
 *     calling thread.
 *   - Log: the environment variable PA_LOG (read once per process) set to 1
 *     writes one "[pa] <status>: <message>" line to stderr for every failing
 *     call; 2 adds one line per state-changing call (pool creation,
 *     allocation, fork, free, swap, append, and each decode with the kernel
 *     and work split it chose).  Unset, 0 or not a number: no output.
 *   - Profiling: a library built with PA_NVTX defined (the build's --nvtx
 *     option) opens an NVTX range named after the call around every entry
 *     point; otherwise the ranges compile to nothing.
 *
 * Device data layout (bytes, row-major, caller-allocated):
 *   k_cache, v_cache: [num_layers][num_blocks][num_kv_heads][block_size][head_dim]
 *       elements of kv_dtype.  One (layer, block, kv_head) tile is one
 *       contiguous block_size x head_dim slab.  A physical block id names
 *       the same tile position in every layer, so one block holds
 *       block_size token slots of the whole per-token footprint
 *       2 x layers x kv_heads x head_dim x bytes ([MKV] Reproduce Bytes per
 *       Token).  Base addresses must be 16-byte aligned.
 *   q, out:           [n][num_q_heads][head_dim] act_dtype.
 *   k_new, v_new:     [T][num_kv_heads][head_dim] act_dtype.
 *   k_scale, v_scale, k_inv_scale, v_inv_scale: [num_layers][num_kv_heads] fp32
 *       (FP8 pools only).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_pool pa_pool;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1,  /* bad argument, shape, pointer or sequence id */
  PA_ERR_NO_BLOCKS = -2,    /* the free list cannot cover the reservation */
  PA_ERR_NO_SEQ = -3,       /* the sequence does not exist */
  PA_ERR_SEQ_EXISTS = -4,   /* fork target already exists */
  PA_ERR_SHARED_BLOCK = -5, /* append into a block other sequences share */
  PA_ERR_CUDA = -6,         /* a CUDA runtime call failed */
  PA_ERR_DEVICE_CHECK = -7  /* a kernel's own bounds/timeout check fired */
} pa_status;

typedef enum {
  PA_BF16 = 0,
  PA_FP16 = 1,
  PA_FP8_E4M3 = 2 /* OCP FP8 E4M3, KV storage only */
} pa_dtype;

/* Bits of the device error word read by pa_check_device_errors. */
#define PA_DEVERR_BAD_BLOCK 0x1u   /* a table entry outside [0, num_blocks) */
#define PA_DEVERR_BAD_LEN 0x2u     /* a sequence length beyond its table */
#define PA_DEVERR_TIMEOUT 0x4u     /* a bounded wait on a copy gave up */

typedef struct {
  int32_t num_layers;
  int32_t num_kv_heads;
  int32_t head_dim;           /* must be 128 */
  int32_t block_size;         /* tokens per block: 16 or 32 (the decode kernel walks 16-token
                                 tiles: a 32-token block is read as its two halves) */
  int32_t num_blocks;         /* physical blocks in the pool */
  int32_t max_seqs;           /* sequence ids are 0 .. max_seqs-1 */
  int32_t max_blocks_per_seq; /* block-table capacity of one sequence */
  int32_t kv_dtype;           /* pa_dtype of the cache */
  int32_t act_dtype;          /* pa_dtype of q, out, k_new, v_new: PA_BF16 or PA_FP16;
                                 equal to kv_dtype unless kv_dtype is PA_FP8_E4M3 */
  int32_t min_partition_tokens; /* smallest fixed split-KV partition a decode call may ask
                                   for (sizes the workspace); 0 selects 512 */
  void *k_cache;              /* device, caller-owned; NULL together with v_cache makes a
                                 host-only pool (block manager only, no device calls) */
  void *v_cache;
  const float *k_scale;       /* device fp32 [L][H_kv]: K dequantisation scale (FP8 only) */
  const float *v_scale;       /* device fp32 [L][H_kv]: V dequantisation scale (FP8 only) */
  const float *k_inv_scale;   /* device fp32 [L][H_kv]: fp32(1/k_scale), used to quantise */
  const float *v_inv_scale;   /* device fp32 [L][H_kv]: fp32(1/v_scale) */
  void *workspace;            /* device, caller-owned, >= pa_workspace_size(desc) bytes,
                                 256-byte aligned; contents need no initialisation */
  size_t workspace_bytes;
  const int32_t *free_order;  /* host, optional: initial free-list order, a permutation
                                 of 0..num_blocks-1 (copied); NULL = ascending */
  int32_t device;             /* CUDA device ordinal holding the buffers */
} pa_pool_desc;

/* Bytes of device workspace a pool with this description needs: the
 * device mirror of the block tables and lengths, the split-KV partial
 * results and an error word.  Pure arithmetic; needs no GPU. */
size_t pa_workspace_size(const pa_pool_desc *desc);

/* Validate `desc` and create the host state of a pool.  Needs no GPU and
 * launches nothing: the device state is initialised by the first device
 * call.  Errors: PA_ERR_INVALID_ARG (shape, dtype, alignment, workspace too
 * small, free_order not a permutation). */
pa_status pa_pool_create(const pa_pool_desc *desc, pa_pool **out);

/* Release the host state.  Does not touch device buffers (caller-owned);
 * the caller must make sure no work that uses the pool is still queued. */
void pa_pool_destroy(pa_pool *pool);

/* Reserve slots so sequence `seq` holds `new_len` tokens, creating it if
 * it does not exist.  Blocks are taken from the head of the free list only
 * when the sequence crosses a block boundary ([KVC] paging paragraph; [MKV]
 * Answer Key item 2); with the free list empty, the least recently used
 * cached block is evicted and taken instead (prefix cache, below).  If the sequence's partly filled tail block is shared
 * with other sequences and the reservation grows the sequence, the tail is
 * first copied to a fresh block (copy-on-write, [MKV] Block Tables and
 * Sharing; [PAS] The bonus: sharing via copy-on-write); the copy covers the
 * whole block for every layer, K and V, and is enqueued on `stream`.
 * The number of blocks needed is checked before any change.
 * Errors: PA_ERR_INVALID_ARG (seq out of range, new_len below the current
 * length or beyond max_blocks_per_seq * block_size), PA_ERR_NO_BLOCKS,
 * PA_ERR_CUDA. */
pa_status pa_alloc_blocks(pa_pool *pool, int32_t seq, int32_t new_len, void *stream);

/* pa_alloc_blocks for n sequences in order, with all copy-on-write copies
 * of the call in one launch.  Stops at the first failure: sequences before
 * it are reserved, the failing one and those after it are untouched;
 * *n_done (always written, even on failure) counts the reserved ones. */
pa_status pa_alloc_blocks_n(pa_pool *pool, int32_t n, const int32_t *seqs,
                            const int32_t *new_lens, void *stream, int32_t *n_done);

/* Make `child` share every block of `parent` (reference count + 1 on each);
 * no data moves ([MKV] Block Tables and Sharing; [PAS] parallel sampling).
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_NO_SEQ (parent), PA_ERR_SEQ_EXISTS. */
pa_status pa_fork_cow(pa_pool *pool, int32_t parent, int32_t child);

/* Write one K row and one V row per token into its cache slot of `layer`:
 *   cache[layer][table[seq][pos / B]][h][pos % B][:] = new[t][h][:]
 * for t < T and every KV head h.  For an FP8 pool the stored code is
 * E4M3(round-to-nearest-even, saturate to +-448)(fp32(x) * inv_scale[layer][h])
 * with the product an IEEE fp32 multiply.  seqs/positions are host arrays of
 * length T; k_new/v_new are device [T][H_kv][head_dim] act_dtype.  Every
 * position must lie below the sequence's reserved length and in a block no
 * other sequence shares (copy-on-write happens in pa_alloc_blocks); (seq,
 * pos) pairs within one call must be distinct.
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_NO_SEQ, PA_ERR_SHARED_BLOCK, PA_ERR_CUDA. */
pa_status pa_append_kv(pa_pool *pool, int32_t layer, int32_t T, const int32_t *seqs,
                       const int32_t *positions, const void *k_new, const void *v_new,
                       void *stream);

/* Single-query decode attention through the block tables ([PAS]
 * PagedAttention: a fused kernel computes attention directly over the
 * non-contiguous blocks using the block table for addressing):
 *   out[i][qh][:] = sum_t softmax_t(scale * q[i][qh] . k_t) v_t
 * over the tokens t < len(seqs[i]) of layer `layer`, with k_t, v_t read from
 * KV head qh / G (G = num_q_heads / num_kv_heads, 1, 2, 4 or 8), slot t % B of
 * block table[seqs[i]][t / B].  FP8 values are dequantised as code value x
 * k_scale / v_scale of (layer, head).  Accumulation is fp32; out is rounded
 * to act_dtype (nearest even).  seqs is a host array of n sequence ids, each
 * with length >= 1; q/out are device [n][num_q_heads][head_dim].
 * partition_tokens: 0 lets the library split long sequences across thread
 * blocks to balance the GPU (results merged by a log-sum-exp reduction);
 * -1 never splits; a positive multiple of block_size, at least the pool's
 * min_partition_tokens, splits every sequence into fixed partitions of that
 * many tokens.
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_NO_SEQ, PA_ERR_CUDA. */
pa_status pa_decode_attention(pa_pool *pool, int32_t layer, int32_t n, const int32_t *seqs,
                              int32_t num_q_heads, const void *q, void *out, float scale,
                              int32_t partition_tokens, void *stream);

/* pa_append_kv of each sequence's last token followed by pa_decode_attention,
 * in one launch: the K/V rows k_new[i], v_new[i] (device [n][num_kv_heads]
 * [head_dim] act_dtype) are written to position len(seqs[i]) - 1 -- the last
 * slot reserved by pa_alloc_blocks -- and attended to in the same pass.  The
 * worker that reads that slot's block writes the row into the cache and into
 * its staged copy of the block, so the result (cache contents included) is
 * exactly that of the two separate calls, with one launch fewer per layer.
 * Each sequence may appear at most once; its last slot must lie in a block no
 * other sequence shares (copy-on-write happens in pa_alloc_blocks).  Other
 * arguments and errors as pa_decode_attention and pa_append_kv; a failure on
 * the host launches nothing. */
pa_status pa_decode_attention_append(pa_pool *pool, int32_t layer, int32_t n, const int32_t *seqs,
                                     const void *k_new, const void *v_new, int32_t num_q_heads,
                                     const void *q, void *out, float scale,
                                     int32_t partition_tokens, void *stream);

/* Decode attention for callers that cannot allocate device memory -- for
 * example a plugin or custom-operator interface of a serving engine that
 * reserves all free HBM for its own KV pool and hands a kernel only its input
 * and output buffers, or a process under a hard memory cap.  Such callers
 * cannot provide a pool's workspace.  The pages have no counterpart of this
 * entry point; it computes the same result as pa_decode_attention with the
 * library's own work split (partition_tokens = 0).
 *
 * No pool is involved: `desc` supplies the shapes, dtypes, device, k_cache /
 * v_cache and (FP8) k_scale / v_scale; its workspace, inverse scales and
 * free_order are ignored.  block_tables: device int32 [n][desc->max_blocks_per_seq],
 * row i = physical block ids of sequence i; seq_lens: host int32 [n], tokens
 * of each sequence (1 .. max_blocks_per_seq * 16); q / out: device
 * [n][num_q_heads][128] act_dtype.  Limits: block_size 16, n <= 512.
 *
 * Allocates nothing (no cudaMalloc/cudaFree).  Its scratch -- split-KV
 * partial results, arrival counters and an error word -- is one
 * static device array of 12 MiB that every GPU loading the library holds
 * until the process exits.  The first call on a device looks up that array's
 * device address (once per device, with the device current) and keeps it for
 * the life of the process; make that first call before any stream capture, and
 * do not use this entry point on a device after cudaDeviceReset (the kept
 * address then names memory of a destroyed context).  Every call shares the
 * array and clears what must start at zero, so calls whose work overlaps on
 * the GPU (other streams, other host threads) race: serialise them, e.g. on
 * one stream.  The kernel's own checks never fault: a block id outside
 * [0, num_blocks) is read as block 0 and sets PA_DEVERR_BAD_BLOCK, a length
 * beyond the table sets PA_DEVERR_BAD_LEN, a copy wait that gives up sets
 * PA_DEVERR_TIMEOUT; those bits collect in the array's error word across calls
 * until pa_noalloc_check_errors reads them.
 * Errors: PA_ERR_INVALID_ARG (shapes, pointers, lengths; n above 512),
 * PA_ERR_CUDA. */
pa_status pa_decode_attention_noalloc(const pa_pool_desc *desc, int32_t layer, int32_t n,
                                      const int32_t *block_tables, const int32_t *seq_lens,
                                      int32_t num_q_heads, const void *q, void *out, float scale,
                                      void *stream);

/* The device error bits (PA_DEVERR_*) that pa_decode_attention_noalloc calls
 * on `device` have set since the last read: synchronises `stream`, reads the
 * word from the no-allocation scratch array and clears it.  Like the calls it
 * reports on it allocates nothing, and it shares their array: a read that
 * overlaps a call on another stream may miss that call's bits, so order it
 * after the calls it checks.  *bits = 0 before the first call on `device`.
 * The pages have no counterpart of this call.
 * Returns PA_ERR_DEVICE_CHECK if any bit was set, PA_ERR_CUDA if a CUDA call
 * failed, PA_ERR_INVALID_ARG for a null `bits` or a bad ordinal. */
pa_status pa_noalloc_check_errors(int32_t device, void *stream, uint32_t *bits);

/* Drop `seq`: every block's reference count falls by one, and blocks that
 * reach zero go to the tail of the free list in logical-block order ([MKV]
 * Block Tables and Sharing) -- registered ones (prefix cache, below) to the
 * recently used end of the cached list instead, in reverse logical order.
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_NO_SEQ. */
pa_status pa_free(pa_pool *pool, int32_t seq);

/* ---- swap-out / swap-in ([MKV] Offload, Hands-On Exercise; [PAS] Beyond
 * paging: radix trees and continuous batching) ----
 *
 * A preempted sequence's KV moves to host memory and its blocks return to the
 * pool; paging it back takes fresh blocks and restores every cached token.
 * The transfer moves whole allocated blocks, every layer, K and V, as stored
 * (FP8 codes for an FP8 pool; the scales stay on the device).  Host image
 * layout, row-major: [2 (K, then V)][ceil(len / block_size)][num_layers]
 * [num_kv_heads][block_size][head_dim] kv_dtype elements.  The image is
 * caller-owned host memory: pinned (cudaHostAlloc / cudaHostRegister) for
 * asynchronous copies, or pageable (the copies then wait); device or managed
 * memory is refused.  Copies are enqueued on `stream` (copy engines, no
 * kernel) and complete in stream order; the image is complete, or the
 * sequence's blocks hold its contents, once the stream reaches that point. */

/* *bytes = size of the host image of a sequence of n_tokens tokens:
 * 2 x ceil(n_tokens / block_size) x num_layers x num_kv_heads x block_size x
 * head_dim x element bytes (the allocated-block bytes; the useful-state bytes
 * are n_tokens / (ceil(n_tokens / block_size) x block_size) of that).  Works
 * on host-only pools.  Errors: PA_ERR_INVALID_ARG. */
pa_status pa_swap_bytes(const pa_pool *pool, int32_t n_tokens, size_t *bytes);

/* Copy every block of `seq` into the host image `host` (host_bytes >=
 * pa_swap_bytes(len)), then drop `seq` as pa_free does (shared blocks stay
 * with their other sequences, registered ones go to the cached list).  Its
 * length is the caller's to keep for pa_swap_in.  Later work that reuses the
 * freed blocks must be ordered after `stream`.
 * Errors: PA_ERR_INVALID_ARG (host-only pool, image too small or not host
 * memory), PA_ERR_NO_SEQ, PA_ERR_CUDA (nothing released). */
pa_status pa_swap_out(pa_pool *pool, int32_t seq, void *host, size_t host_bytes, void *stream);

/* Create `seq` with n_tokens tokens in fresh blocks from the free list (then
 * by evicting cached blocks) and copy the host image into them; the blocks
 * are private even if the sequence shared blocks before it was swapped out.
 * The new table reaches the device with the next kernel launch on the pool.
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_SEQ_EXISTS, PA_ERR_NO_BLOCKS (checked
 * before any change; the image and the device are checked before blocks are
 * taken), PA_ERR_CUDA (a copy could not be enqueued: the sequence is dropped
 * again and its blocks go back to the free list, but cached blocks that the
 * reservation evicted stay evicted and the free list's order may differ). */
pa_status pa_swap_in(pa_pool *pool, int32_t seq, int32_t n_tokens, const void *host,
                     size_t host_bytes, void *stream);

/* ---- host state checkpoint -------------------------------------------
 * The block manager's whole host state as a byte image: the free list in
 * order, every block's reference count, every sequence's length and block
 * table, and the prefix cache (its index and the least-recently-used order
 * of idle cached blocks).  pa_state_load restores it into a pool of the same
 * geometry (num_blocks, block_size, max_seqs, max_blocks_per_seq): from then
 * on the pool hands out, shares, copies, evicts and releases blocks exactly
 * as the saved pool would have, and the device copy of the tables is
 * rewritten with the next kernel launch on the pool.  The KV cache contents
 * are the caller's buffers: a pool created over the same cache buffers and
 * restored from the image decodes as the saved pool did.  The image is plain
 * native-endian int32 words; it carries no device state and no copy-on-write
 * log (pa_get_cow_log is empty after a load). */

/* Bytes of the current state image. */
pa_status pa_state_size(const pa_pool *pool, size_t *bytes);

/* Write the state image to buf (cap bytes); *written = its size.
 * Errors: PA_ERR_INVALID_ARG (null argument, cap smaller than
 * pa_state_size). */
pa_status pa_state_save(const pa_pool *pool, void *buf, size_t cap, size_t *written);

/* Replace the pool's host state by the image in buf.  The whole image is
 * validated first: geometry, every id in range, a consistent pool (each
 * block exactly one of free, referenced by the tables it appears in, or idle
 * and cached; reference counts equal to those appearances) and a consistent
 * prefix index (parent chains reach the root, child counts and keys match,
 * no prefix twice, no node that holds no block and leads to none).
 * Errors: PA_ERR_INVALID_ARG (null argument, a truncated, corrupt or
 * inconsistent image, another geometry); on error nothing changes. */
pa_status pa_state_load(pa_pool *pool, const void *buf, size_t bytes);

/* ---- block-granular prefix cache ([PAS] Beyond paging: radix trees and
 * continuous batching; [MKV] Block Tables and Sharing, Answer Key item 4) ----
 *
 * A full block whose KV the caller has written, in every layer, may be
 * registered under the token prefix it ends: every token from the start of
 * its sequence to its last slot (a token's KV depends on all tokens before
 * it).  A new prompt then reuses, from its first block on, each block whose
 * whole prefix is registered, and stops at the first one that is not; reuse
 * is whole blocks only (a 103-token prompt reuses at most 96 tokens with
 * 16-token blocks).  Registered blocks are reference counted like any other.
 * Once nothing references one it is kept, contents intact, on a least-
 * recently-used list (pa_get_cached_blocks) instead of the free list, and it
 * is evicted -- unregistered and handed out again -- only when a block is
 * needed and the free list is empty.  A registered block is immutable:
 * pa_append_kv and pa_decode_attention_append refuse to write into it
 * (PA_ERR_SHARED_BLOCK).  The first registration of a prefix wins.  Tokens
 * are opaque int32 ids compared exactly; all of this is host work. */

/* Register the full blocks of `seq` that cover tokens[0, n_tokens), the
 * sequence's first n_tokens tokens (n_tokens <= its length; `tokens` is a
 * host array, may be NULL when n_tokens == 0).  A block whose prefix is
 * already registered under another block stays unregistered.
 * Errors: PA_ERR_INVALID_ARG (n_tokens negative or beyond the length; a block
 * already registered under a different prefix -- nothing is registered
 * then), PA_ERR_NO_SEQ. */
pa_status pa_prefix_register(pa_pool *pool, int32_t seq, int32_t n_tokens, const int32_t *tokens);

/* *n_cached = how many leading tokens of the prompt tokens[0, n_tokens) have
 * their KV in registered blocks (a multiple of block_size).  Changes nothing.
 * Errors: PA_ERR_INVALID_ARG. */
pa_status pa_prefix_match(const pa_pool *pool, int32_t n_tokens, const int32_t *tokens,
                          int32_t *n_cached);

/* Create `seq` with length n_tokens for the prompt tokens[0, n_tokens): its
 * leading blocks whose prefix is registered are shared (reference count + 1;
 * an idle one leaves the cached list), the rest are taken from the free list
 * and then by evicting cached blocks.  *n_cached = prompt tokens whose KV the
 * shared blocks already hold; the caller appends positions n_cached ..
 * n_tokens - 1 and may then register the prompt.  No device work: the new
 * table reaches the device with the next kernel launch on the pool.
 * Errors: PA_ERR_INVALID_ARG (seq out of range, n_tokens negative or beyond
 * max_blocks_per_seq * block_size), PA_ERR_SEQ_EXISTS, PA_ERR_NO_BLOCKS
 * (checked before any change). */
pa_status pa_alloc_blocks_prefix(pa_pool *pool, int32_t seq, int32_t n_tokens,
                                 const int32_t *tokens, int32_t *n_cached);

/* ---- introspection (host state; for tests and schedulers) ---- */

/* Length and block table of `seq`; `table` receives min(cap, nblocks)
 * entries (may be NULL when cap == 0). */
pa_status pa_get_seq(pa_pool *pool, int32_t seq, int32_t *len, int32_t *table, int32_t cap,
                     int32_t *nblocks);
/* Reference count of every block: `out` holds num_blocks entries. */
pa_status pa_get_refcounts(pa_pool *pool, int32_t *out, int32_t cap);
/* Free list from head to tail: `out` receives min(cap, *n) entries. */
pa_status pa_get_free_list(pa_pool *pool, int32_t *out, int32_t cap, int32_t *n);
/* Cached blocks (registered, unreferenced), least recently used first:
 * `out` receives min(cap, *n) entries. */
pa_status pa_get_cached_blocks(pa_pool *pool, int32_t *out, int32_t cap, int32_t *n);
/* Every copy-on-write made so far as (src, dst) pairs: `pairs` receives
 * min(cap, *n) pairs (2 ints each). */
pa_status pa_get_cow_log(pa_pool *pool, int32_t *pairs, int32_t cap, int32_t *n);
/* Number of kernels this pool has launched since it was created. */
uint64_t pa_launch_count(const pa_pool *pool);
/* Work plan of the last pa_decode_attention call on this pool:
 * *shared_sets = sibling sets whose common prefix was read once (0 unless
 * partition_tokens was 0), *kv_tiles = (16-token tile, KV head) pairs the call reads
 * from the cache.  Sequences forked from one prompt share the prompt's blocks
 * by reference count ([MKV] Block Tables and Sharing; [PAS] The bonus:
 * sharing via copy-on-write); with partition_tokens = 0 the library reads a
 * run of at least two full blocks that several of the call's sequences share
 * once for all of them (up to 8 / G sequences per set), so *kv_tiles can be
 * below the sum over sequences.  Either pointer may be NULL. */
pa_status pa_last_decode_plan(const pa_pool *pool, int32_t *shared_sets, int64_t *kv_tiles);
/* The sibling sets pa_decode_attention (partition_tokens = 0) would form for
 * the n sequences `seqs` with query group `group` (1, 2, 4 or 8), from the
 * host block tables alone (no device work; works on host-only pools too).
 * set_of[i] = set of item i or -1; set_cp[k] = full blocks set k reads once
 * (set_cp needs room for n entries); *n_sets = number of sets.  Sequences are
 * ordered by their block tables and consecutive ones whose tables start with
 * the same run of >= 2 full blocks are grouped, at most 8 / group per set;
 * every member keeps at least its last block to itself.
 * Errors: PA_ERR_INVALID_ARG (n above 512, bad group or sequence id),
 * PA_ERR_NO_SEQ. */
pa_status pa_plan_siblings(const pa_pool *pool, int32_t n, const int32_t *seqs, int32_t group,
                           int32_t *set_of, int32_t *set_cp, int32_t *n_sets);

/* Which decode kernel serves a query group of 8 over a 16-bit cache (every
 * other shape always runs on the warp-level kernel):
 *   PA_DECODE_WARP    warp-level tensor-core MMAs (mma.sync), 8 workers per SM;
 *   PA_DECODE_TCGEN05 5th-generation tensor cores: S^T = K Q^T and
 *                     O^T = V^T P^T accumulate in tensor memory, one worker per
 *                     SM with 128-token tiles;
 *   PA_DECODE_AUTO    the library's choice (the faster of the two on B200).
 * Both compute the same function within the stated tolerance (not bit for
 * bit).  Errors: PA_ERR_INVALID_ARG. */
#define PA_DECODE_AUTO 0
#define PA_DECODE_WARP 1
#define PA_DECODE_TCGEN05 2
pa_status pa_set_decode_path(pa_pool *pool, int32_t path);
/* *tcgen05 = 1 if the last decode call on this pool ran the tcgen05 kernel. */
pa_status pa_last_decode_kernel(const pa_pool *pool, int32_t *tcgen05);

/* Synchronise `stream`, read the device error word, clear it, and store the
 * PA_DEVERR_* bits in *bits.  Returns PA_ERR_DEVICE_CHECK if any bit was set,
 * PA_ERR_CUDA if a CUDA call failed, PA_ERR_INVALID_ARG for a host-only pool. */
pa_status pa_check_device_errors(pa_pool *pool, void *stream, uint32_t *bits);

/* Host-side fault injection for tests: after `n` more block allocations
 * succeed, further reservations that need blocks fail with PA_ERR_NO_BLOCKS
 * (state unchanged).  n < 0 switches the fault off. */
pa_status pa_debug_fail_after(pa_pool *pool, int32_t n);

/* Text of the last failure on the calling thread ("" if none). */
const char *pa_last_error(void);
/* Name of a status code. */
const char *pa_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
