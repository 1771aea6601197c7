// C ABI of the paged decode-attention library (declared in include/pa.h).
//
// Host side of every call: argument validation, the block manager, planning
// of the decode work split, and the launches.  Nothing here computes on the
// CPU what a kernel computes on the GPU; a pool without device buffers
// (host-only) supports only the block-manager calls.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <optional>
#include <cstring>
#include <memory>
#include <string>
#include <vector>

#include "block_manager.h"
#include "pa.h"
#include "pa_internal.h"
#include "trace.h"

namespace {

thread_local std::string g_last_error;

pa_status fail(pa_status st, const std::string& msg) {
  g_last_error = msg;
  pa::logf(1, "%s: %s", pa_status_string(st), msg.c_str());
  return st;
}

pa_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  pa::logf(1, "%s: %s", pa_status_string(PA_ERR_CUDA), g_last_error.c_str());
  return PA_ERR_CUDA;
}

// Workspace layout: [header: error word | 256 B] [block-table mirror + lengths]
// [stream-K arrival counters] [split-KV partial slots]
constexpr size_t kHeaderBytes = 256;
constexpr size_t kAlign = 256;
constexpr int kMinBlocksPerWorker = 4;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int64_t meta_ints(const pa_pool_desc& d) {
  return static_cast<int64_t>(d.max_seqs) * d.max_blocks_per_seq + d.max_seqs;
}

int32_t min_partition(const pa_pool_desc& d) {
  return d.min_partition_tokens > 0 ? d.min_partition_tokens : 512;
}

// Arrival counters: one per worker (indexed by the first worker of a cut unit).
size_t counter_bytes(const pa_pool_desc&) {
  return align_up(static_cast<size_t>(pa::kMaxWorkers) * sizeof(int32_t));
}

// Partial slots: two per worker (stream-K) or one per partition (fixed partitions).
int64_t partial_slots(const pa_pool_desc& d) {
  const int64_t max_tokens = static_cast<int64_t>(d.max_blocks_per_seq) * d.block_size;
  const int64_t parts = (max_tokens + min_partition(d) - 1) / min_partition(d);
  const int64_t fixed = static_cast<int64_t>(d.max_seqs) * d.num_kv_heads * parts;
  return std::max<int64_t>(2 * pa::kMaxWorkers, fixed);
}

// Switches to the pool's device for the duration of a call.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};


}  // namespace

namespace pa {
void set_last_error(const std::string& msg) {
  g_last_error = msg;
  if (!msg.empty()) logf(1, "error: %s", msg.c_str());  // the caller's status is not known here
}
}  // namespace pa

struct pa_pool {
  pa_pool_desc d{};
  std::unique_ptr<pa::BlockManager> bm;
  std::vector<pa::CowPair> cow_log;
  pa::PoolView view{};
  bool host_only = false;
  bool dev_ready = false;
  int num_sms = 0;
  pa::CacheMaps maps{};
  uint64_t launches = 0;
  // scratch reused across calls
  std::vector<pa::CowPair> cows;
  std::vector<int64_t> slots;
  std::vector<int32_t> a, b;
  std::vector<int32_t> order, set_of;  // sibling planning
  // plan of the last decode call (pa_last_decode_plan)
  int32_t last_sets = 0;
  int64_t last_tiles = 0;
  int32_t path = PA_DECODE_AUTO;  // pa_set_decode_path
  bool last_tc = false;
  // The plan of the last single-launch decode call: the calls of one step
  // (one per layer) see the same tables, so later ones reuse it.
  struct PlanCache {
    bool valid = false, sib = false, tc = false;
    uint64_t version = 0;
    int32_t group = 0, mode = 0, part_blocks = 0;
    int64_t blocks = 0;
    std::vector<int32_t> seqs;
    pa::DecodePlan plan;
    pa::SibPlan sib_plan;
  } cache;
};

namespace {

pa_status ensure_device(pa_pool* p, cudaStream_t stream) {
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  if (p->dev_ready) return PA_OK;
  cudaError_t e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->d.device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  e = cudaMemsetAsync(p->view.err, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(error word)");
  e = cudaMemsetAsync(p->view.counters, 0, counter_bytes(p->d), stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(counters)");

  const int64_t rows = static_cast<int64_t>(p->d.num_layers) * p->d.num_blocks * p->d.num_kv_heads *
                       p->d.block_size;
  if (const char* why = pa::encode_cache_maps(p->d.k_cache, p->d.v_cache, p->d.kv_dtype, rows, &p->maps))
    return fail(PA_ERR_CUDA, why);
  p->dev_ready = true;
  return PA_OK;
}

// Ship all pending mirror deltas in a launch of their own.
pa_status flush_deltas(pa_pool* p, cudaStream_t stream) {
  pa::MirrorDeltas& md = p->bm->deltas();
  if (md.size() == 0) return PA_OK;
  const int n = static_cast<int>(md.size());
  cudaError_t e = pa::launch_meta_apply(p->view, md.indices().data(), md.values().data(), n, stream);
  if (e != cudaSuccess) return cuda_fail(e, "meta apply launch");
  p->launches += (n + pa::kPayloadLarge / 2 - 1) / (pa::kPayloadLarge / 2);
  md.consume(n);
  return PA_OK;
}

pa_status launch_cows(pa_pool* p, cudaStream_t stream) {
  if (p->cows.empty()) return PA_OK;
  p->cow_log.insert(p->cow_log.end(), p->cows.begin(), p->cows.end());
  if (p->host_only) {
    p->cows.clear();
    return PA_OK;
  }
  DeviceGuard guard(p->d.device);
  if (!guard.ok) {
    p->cows.clear();
    return fail(PA_ERR_CUDA, "cannot select the pool's device");
  }
  pa_status st = ensure_device(p, stream);
  if (st != PA_OK) {
    p->cows.clear();
    return st;
  }
  pa::MirrorDeltas& md = p->bm->deltas();
  size_t at = 0;
  while (at < p->cows.size()) {
    const size_t n = std::min<size_t>(p->cows.size() - at, 1024);
    p->a.resize(n);
    p->b.resize(n);
    for (size_t k = 0; k < n; ++k) {
      p->a[k] = p->cows[at + k].src;
      p->b[k] = p->cows[at + k].dst;
    }
    const int nd = static_cast<int>(md.size());
    int launches = 0;
    cudaError_t e = pa::launch_cow_copy(p->view, p->a.data(), p->b.data(), static_cast<int>(n),
                                        md.indices().data(), md.values().data(), nd, stream,
                                        &launches);
    p->launches += launches;
    if (e != cudaSuccess) {
      p->cows.clear();
      return cuda_fail(e, "copy-on-write launch");
    }
    md.consume(nd);
    at += n;
  }
  p->cows.clear();
  return PA_OK;
}

pa_status seq_arg(const pa_pool* p, int32_t seq) {
  if (seq < 0 || seq >= p->d.max_seqs)
    return fail(PA_ERR_INVALID_ARG, "sequence id " + std::to_string(seq) + " out of range");
  return PA_OK;
}

pa_status bm_status(pa::Status s, const char* what) {
  switch (s) {
    case pa::kOk: return PA_OK;
    case pa::kInvalidArg: return fail(PA_ERR_INVALID_ARG, std::string(what) + ": invalid argument");
    case pa::kNoBlocks: return fail(PA_ERR_NO_BLOCKS, std::string(what) + ": free list too short");
    case pa::kNoSeq: return fail(PA_ERR_NO_SEQ, std::string(what) + ": no such sequence");
    case pa::kSeqExists: return fail(PA_ERR_SEQ_EXISTS, std::string(what) + ": sequence exists");
    case pa::kSharedBlock:
      return fail(PA_ERR_SHARED_BLOCK, std::string(what) + ": target block is shared");
    default: return fail(PA_ERR_INVALID_ARG, what);
  }
}

// Which kernel PA_DECODE_AUTO picks for G = 8 over 16-bit KV.
constexpr bool kAutoTcgen05 = false;

// Shortest common prefix (in full blocks) that is read once for a sibling set.
constexpr int kMinShareBlocks = 2;

// Plan that reads the common prefix of sibling sequences once.  Sequences
// share blocks by reference count after a fork ([MKV] Block Tables and
// Sharing; [PAS] The bonus: sharing via copy-on-write), so forks of one
// prompt hold the same physical ids at the start of their tables.  Items are
// ordered by their tables (lexicographically), and consecutive items form a
// set while the set's common run of full blocks stays >= kMinShareBlocks and
// members x group <= 8 (the query rows of one tensor-core tile).  Each
// member keeps at least its last block to itself, so every shared block is
// full for every member.  A set is one work unit: the shared run, then each
// member's own blocks in member order.  Returns false when no set forms;
// `sp` is then meaningless.
bool build_sib_plan(const pa_pool* p, const int32_t* seqs, int32_t cnt, int group, int cap,
                    pa::SibPlan& sp, std::vector<int32_t>& order, std::vector<int32_t>& set_of) {
  const int H = p->d.num_kv_heads;
  const int32_t alpha = pa::stream_k_alpha(p->d.kv_dtype);
  const int max_members = pa::kMaxGroup / group;
  if (max_members < 2 || cnt < 2) return false;
  const pa::BlockManager& bm = *p->bm;
  // The kernel walks 16-token tiles (two per 32-token block); sharing is a
  // property of table entries (blocks), so runs are found in blocks and
  // placed in tiles.
  const int tpb = p->d.block_size / 16;
  auto nb_of = [&](int i) { return (bm.len(seqs[i]) + p->d.block_size - 1) / p->d.block_size; };
  auto nt_of = [&](int i) { return (bm.len(seqs[i]) + 15) / 16; };
  order.clear();
  for (int i = 0; i < cnt; ++i)
    if (nb_of(i) > kMinShareBlocks) order.push_back(i);
  if (order.size() < 2) return false;
  std::sort(order.begin(), order.end(), [&](int a, int b) {
    const std::vector<int32_t>& ta = bm.table(seqs[a]);
    const std::vector<int32_t>& tb = bm.table(seqs[b]);
    const size_t m = std::min(ta.size(), tb.size());
    for (size_t k = 0; k < m; ++k)
      if (ta[k] != tb[k]) return ta[k] < tb[k];
    return ta.size() != tb.size() ? ta.size() < tb.size() : a < b;
  });
  // sets, in sorted order: members order[a .. b), shared run cp
  set_of.assign(cnt, -1);
  int nu = 0, placed = 0;
  int64_t work = 0;
  sp.pre[0] = 0;
  sp.mem0[0] = 0;
  size_t a = 0;
  while (a < order.size()) {
    const std::vector<int32_t>& ta = bm.table(seqs[order[a]]);
    int cp = nb_of(order[a]) - 1;
    size_t b = a + 1;
    while (b < order.size() && static_cast<int>(b - a) < max_members) {
      const std::vector<int32_t>& tb = bm.table(seqs[order[b]]);
      const int lim = std::min(cp, nb_of(order[b]) - 1);
      int l = 0;
      while (l < lim && ta[l] == tb[l]) ++l;
      if (l < kMinShareBlocks) break;
      cp = l;
      ++b;
    }
    if (b - a < 2) {
      ++a;
      continue;
    }
    const int cpt = cp * tpb;  // shared run in tiles
    int64_t pos = cpt;
    for (size_t j = a; j < b; ++j) {
      const int it = order[j];
      set_of[it] = nu;
      sp.mem[placed++] = static_cast<int16_t>(it);
      sp.part[it] = static_cast<int32_t>(pos);
      pos += nt_of(it) - cpt;
    }
    sp.cp[nu] = cpt;
    work += alpha + pos;
    sp.pre[nu + 1] = static_cast<int32_t>(work);
    sp.mem0[nu + 1] = static_cast<int16_t>(placed);
    ++nu;
    a = b;
  }
  if (nu == 0) return false;
  const int sets = nu;
  for (int i = 0; i < cnt; ++i) {  // every other item is a unit of its own
    sp.seq[i] = seqs[i];
    sp.len[i] = bm.len(seqs[i]);
    if (set_of[i] >= 0) continue;
    sp.mem[placed++] = static_cast<int16_t>(i);
    sp.part[i] = 0;
    sp.cp[nu] = 0;
    work += alpha + nt_of(i);
    sp.pre[nu + 1] = static_cast<int32_t>(work);
    sp.mem0[nu + 1] = static_cast<int16_t>(placed);
    ++nu;
  }
  sp.n = cnt;
  sp.nu = nu;
  sp.alpha = alpha;
  sp.pad_ = 0;
  sp.per_head = work;
  const int64_t total = work * H;
  if (total >= (int64_t{1} << 30)) return false;
  int64_t W = std::min<int64_t>(cap, total);
  W = std::min<int64_t>(W, std::max<int64_t>(1, (total + kMinBlocksPerWorker - 1) / kMinBlocksPerWorker));
  W = std::min<int64_t>(W, p->view.partial_slots / 2);
  sp.workers = static_cast<int32_t>(std::max<int64_t>(1, W));
  sp.sets = sets;
  return true;
}

}  // namespace

extern "C" {

size_t pa_workspace_size(const pa_pool_desc* d) {
  PA_RANGE();
  if (!d || d->max_seqs <= 0 || d->max_blocks_per_seq <= 0 || d->num_kv_heads <= 0 ||
      d->block_size <= 0)
    return 0;
  return kHeaderBytes + align_up(static_cast<size_t>(meta_ints(*d)) * 4) + counter_bytes(*d) +
         static_cast<size_t>(partial_slots(*d)) * pa::kPartialSlotFloats * 4;
}

pa_status pa_pool_create(const pa_pool_desc* d, pa_pool** out) {
  PA_RANGE();
  g_last_error.clear();
  if (!d || !out) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (d->head_dim != pa::kHeadDim) return fail(PA_ERR_INVALID_ARG, "head_dim must be 128");
  if (d->block_size != 16 && d->block_size != 32)
    return fail(PA_ERR_INVALID_ARG, "block_size must be 16 or 32");
  if (d->num_layers <= 0 || d->num_kv_heads <= 0 || d->num_blocks <= 0 || d->max_seqs <= 0 ||
      d->max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "sizes must be positive");
  if (d->kv_dtype < PA_BF16 || d->kv_dtype > PA_FP8_E4M3)
    return fail(PA_ERR_INVALID_ARG, "bad kv_dtype");
  if (d->act_dtype != PA_BF16 && d->act_dtype != PA_FP16)
    return fail(PA_ERR_INVALID_ARG, "act_dtype must be PA_BF16 or PA_FP16");
  if (d->kv_dtype != PA_FP8_E4M3 && d->kv_dtype != d->act_dtype)
    return fail(PA_ERR_INVALID_ARG, "16-bit caches must use the activation dtype");
  const int64_t rows = static_cast<int64_t>(d->num_layers) * d->num_blocks * d->num_kv_heads *
                       d->block_size;
  if (rows >= (int64_t{1} << 31))
    return fail(PA_ERR_INVALID_ARG, "pool too large: layers*blocks*kv_heads*block_size >= 2^31");
  if (meta_ints(*d) >= (int64_t{1} << 31)) return fail(PA_ERR_INVALID_ARG, "tables too large");
  const int32_t pmin = min_partition(*d);
  if (pmin < d->block_size || pmin % d->block_size != 0)
    return fail(PA_ERR_INVALID_ARG, "min_partition_tokens must be a multiple of block_size");
  const bool host_only = d->k_cache == nullptr && d->v_cache == nullptr;
  if (!host_only) {
    if (!d->k_cache || !d->v_cache) return fail(PA_ERR_INVALID_ARG, "k_cache and v_cache go together");
    if ((reinterpret_cast<uintptr_t>(d->k_cache) | reinterpret_cast<uintptr_t>(d->v_cache)) & 15)
      return fail(PA_ERR_INVALID_ARG, "caches must be 16-byte aligned");
    if (!d->workspace || (reinterpret_cast<uintptr_t>(d->workspace) & (kAlign - 1)))
      return fail(PA_ERR_INVALID_ARG, "workspace must be non-null and 256-byte aligned");
    if (d->workspace_bytes < pa_workspace_size(d))
      return fail(PA_ERR_INVALID_ARG, "workspace smaller than pa_workspace_size()");
    if (d->kv_dtype == PA_FP8_E4M3 &&
        (!d->k_scale || !d->v_scale || !d->k_inv_scale || !d->v_inv_scale))
      return fail(PA_ERR_INVALID_ARG, "FP8 pools need k/v scales and inverse scales");
  }
  if (d->free_order) {
    std::vector<char> seen(d->num_blocks, 0);
    for (int32_t k = 0; k < d->num_blocks; ++k) {
      const int32_t b = d->free_order[k];
      if (b < 0 || b >= d->num_blocks || seen[b])
        return fail(PA_ERR_INVALID_ARG, "free_order is not a permutation of the block ids");
      seen[b] = 1;
    }
  }
  auto p = std::make_unique<pa_pool>();
  p->d = *d;
  p->d.min_partition_tokens = pmin;
  p->d.free_order = nullptr;
  p->host_only = host_only;
  p->bm = std::make_unique<pa::BlockManager>(d->num_blocks, d->block_size, d->max_seqs,
                                             d->max_blocks_per_seq, d->free_order);
  pa::PoolView& v = p->view;
  v.k_cache = d->k_cache;
  v.v_cache = d->v_cache;
  v.k_scale = d->k_scale;
  v.v_scale = d->v_scale;
  v.k_inv = d->k_inv_scale;
  v.v_inv = d->v_inv_scale;
  if (!host_only) {
    uint8_t* ws = static_cast<uint8_t*>(d->workspace);
    v.err = reinterpret_cast<uint32_t*>(ws);
    v.meta = reinterpret_cast<int32_t*>(ws + kHeaderBytes);
    v.tables = v.meta;
    v.lens = v.meta + static_cast<int64_t>(d->max_seqs) * d->max_blocks_per_seq;
    v.counters = reinterpret_cast<int32_t*>(ws + kHeaderBytes + align_up(meta_ints(*d) * 4));
    v.partials = reinterpret_cast<float*>(ws + kHeaderBytes + align_up(meta_ints(*d) * 4) +
                                          counter_bytes(*d));
    v.partial_slots = partial_slots(*d);
  }
  v.num_layers = d->num_layers;
  v.num_kv_heads = d->num_kv_heads;
  v.block_size = d->block_size;
  v.num_blocks = d->num_blocks;
  v.max_seqs = d->max_seqs;
  v.mbps = d->max_blocks_per_seq;
  v.kv_dtype = d->kv_dtype;
  v.act_dtype = d->act_dtype;
  pa::logf(2, "pool_create: %s, %d layers, %d blocks of %d tokens, %d KV heads, %d sequences x %d blocks, "
           "kv dtype %d", host_only ? "host only" : "device buffers", d->num_layers, d->num_blocks,
           d->block_size, d->num_kv_heads, d->max_seqs, d->max_blocks_per_seq, d->kv_dtype);
  *out = p.release();
  return PA_OK;
}

void pa_pool_destroy(pa_pool* p) {
  PA_RANGE();
  delete p;
}

pa_status pa_alloc_blocks_n(pa_pool* p, int32_t n, const int32_t* seqs, const int32_t* new_lens,
                            void* stream, int32_t* n_done) {
  PA_RANGE();
  g_last_error.clear();
  if (n_done) *n_done = 0;
  if (!p || n < 0 || (n > 0 && (!seqs || !new_lens)))
    return fail(PA_ERR_INVALID_ARG, "null argument");
  p->cows.clear();
  pa_status st = PA_OK;
  int32_t k = 0;
  for (; k < n; ++k) {
    st = bm_status(p->bm->reserve(seqs[k], new_lens[k], &p->cows), "pa_alloc_blocks");
    if (st != PA_OK) break;
  }
  if (n_done) *n_done = k;
  pa::logf(2, "alloc_blocks: %d of %d sequences reserved, %zu block copies", k, n, p->cows.size());
  const pa_status launch = launch_cows(p, static_cast<cudaStream_t>(stream));
  return st != PA_OK ? st : launch;
}

pa_status pa_alloc_blocks(pa_pool* p, int32_t seq, int32_t new_len, void* stream) {
  PA_RANGE();
  int32_t done = 0;
  return pa_alloc_blocks_n(p, 1, &seq, &new_len, stream, &done);
}

pa_status pa_fork_cow(pa_pool* p, int32_t parent, int32_t child) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  pa::logf(2, "fork_cow: sequence %d -> %d", parent, child);
  return bm_status(p->bm->fork(parent, child), "pa_fork_cow");
}

pa_status pa_free(pa_pool* p, int32_t seq) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  pa::logf(2, "free: sequence %d", seq);
  return bm_status(p->bm->release(seq), "pa_free");
}

pa_status pa_prefix_register(pa_pool* p, int32_t seq, int32_t n_tokens, const int32_t* tokens) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || n_tokens < 0 || (n_tokens > 0 && !tokens)) return fail(PA_ERR_INVALID_ARG, "null argument");
  pa_status st = seq_arg(p, seq);
  if (st != PA_OK) return st;
  return bm_status(p->bm->register_prefix(seq, n_tokens, tokens), "pa_prefix_register");
}

pa_status pa_prefix_match(const pa_pool* p, int32_t n_tokens, const int32_t* tokens,
                          int32_t* n_cached) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !n_cached || n_tokens < 0 || (n_tokens > 0 && !tokens))
    return fail(PA_ERR_INVALID_ARG, "null argument");
  *n_cached = p->bm->match_prefix(n_tokens, tokens, nullptr) * p->d.block_size;
  return PA_OK;
}

pa_status pa_alloc_blocks_prefix(pa_pool* p, int32_t seq, int32_t n_tokens, const int32_t* tokens,
                                 int32_t* n_cached) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !n_cached || n_tokens < 0 || (n_tokens > 0 && !tokens))
    return fail(PA_ERR_INVALID_ARG, "null argument");
  pa_status st = seq_arg(p, seq);
  if (st != PA_OK) return st;
  int32_t c = 0;
  st = bm_status(p->bm->reserve_prefix(seq, n_tokens, tokens, &c), "pa_alloc_blocks_prefix");
  if (st == PA_OK) *n_cached = c;
  return st;
}

namespace {

// One (layer, block) tile of K or V: num_kv_heads x block_size x head_dim elements.
size_t tile_bytes(const pa_pool_desc& d) {
  return static_cast<size_t>(d.num_kv_heads) * d.block_size * pa::kHeadDim *
         (d.kv_dtype == PA_FP8_E4M3 ? 1 : 2);
}

size_t swap_image_bytes(const pa_pool_desc& d, int64_t n_tokens) {
  const int64_t blocks = (n_tokens + d.block_size - 1) / d.block_size;
  return 2 * static_cast<size_t>(blocks) * d.num_layers * tile_bytes(d);
}

// The host image must be host memory (pinned for asynchronous copies, or
// pageable); device or managed memory is refused.
pa_status check_host_image(const void* host, size_t have, size_t need) {
  if (have < need) return fail(PA_ERR_INVALID_ARG, "host image smaller than pa_swap_bytes()");
  if (need == 0) return PA_OK;
  if (host == nullptr) return fail(PA_ERR_INVALID_ARG, "null host image");
  cudaPointerAttributes a{};
  cudaError_t e = cudaPointerGetAttributes(&a, host);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "cudaPointerGetAttributes(host image)");
  }
  if (a.type != cudaMemoryTypeHost && a.type != cudaMemoryTypeUnregistered)
    return fail(PA_ERR_INVALID_ARG, "the host image must be host memory");
  return PA_OK;
}

// Copy the blocks `table` between the pool and a host image laid out
// [K, V][logical block][layer][tile]: per (K/V, block) one 2-D copy whose rows
// are the block's tiles in successive layers (one layer stride apart in the
// pool, contiguous in the image).
pa_status swap_copies(pa_pool* p, const std::vector<int32_t>& table, char* host, bool to_host,
                      cudaStream_t s) {
  const pa_pool_desc& d = p->d;
  const size_t tile = tile_bytes(d);
  const size_t layer_stride = tile * static_cast<size_t>(d.num_blocks);
  const size_t n = table.size();
  int max_pitch = 0;
  cudaError_t e = cudaDeviceGetAttribute(&max_pitch, cudaDevAttrMaxPitch, d.device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(max pitch)");
  const cudaMemcpyKind kind = to_host ? cudaMemcpyDeviceToHost : cudaMemcpyHostToDevice;
  for (int kv = 0; kv < 2; ++kv) {
    char* cache = static_cast<char*>(kv ? d.v_cache : d.k_cache);
    for (size_t j = 0; j < n; ++j) {
      char* dev = cache + static_cast<size_t>(table[j]) * tile;
      char* img = host + (static_cast<size_t>(kv) * n + j) * d.num_layers * tile;
      if (layer_stride <= static_cast<size_t>(max_pitch)) {
        e = to_host ? cudaMemcpy2DAsync(img, tile, dev, layer_stride, tile, d.num_layers, kind, s)
                    : cudaMemcpy2DAsync(dev, layer_stride, img, tile, tile, d.num_layers, kind, s);
      } else {
        for (int32_t l = 0; l < d.num_layers && e == cudaSuccess; ++l) {
          char* dl = dev + static_cast<size_t>(l) * layer_stride;
          char* hl = img + static_cast<size_t>(l) * tile;
          e = to_host ? cudaMemcpyAsync(hl, dl, tile, kind, s) : cudaMemcpyAsync(dl, hl, tile, kind, s);
        }
      }
      if (e != cudaSuccess) return cuda_fail(e, "swap copy");
    }
  }
  return PA_OK;
}

}  // namespace

pa_status pa_swap_bytes(const pa_pool* p, int32_t n_tokens, size_t* bytes) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !bytes || n_tokens < 0) return fail(PA_ERR_INVALID_ARG, "null argument or negative length");
  *bytes = swap_image_bytes(p->d, n_tokens);
  return PA_OK;
}

pa_status pa_swap_out(pa_pool* p, int32_t seq, void* host, size_t host_bytes, void* stream) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  pa_status st = seq_arg(p, seq);
  if (st != PA_OK) return st;
  if (!p->bm->active(seq)) return fail(PA_ERR_NO_SEQ, "pa_swap_out: no such sequence");
  DeviceGuard guard(p->d.device);
  if (!guard.ok) return fail(PA_ERR_CUDA, "cannot select the pool's device");
  st = check_host_image(host, host_bytes, swap_image_bytes(p->d, p->bm->len(seq)));
  if (st != PA_OK) return st;
  const std::vector<int32_t> table = p->bm->table(seq);
  pa::logf(2, "swap_out: sequence %d, %d tokens, %zu bytes", seq, p->bm->len(seq), host_bytes);
  st = swap_copies(p, table, static_cast<char*>(host), true, static_cast<cudaStream_t>(stream));
  if (st != PA_OK) return st;
  return bm_status(p->bm->release(seq), "pa_swap_out");
}

pa_status pa_swap_in(pa_pool* p, int32_t seq, int32_t n_tokens, const void* host, size_t host_bytes,
                     void* stream) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  pa_status st = seq_arg(p, seq);
  if (st != PA_OK) return st;
  if (n_tokens < 0) return fail(PA_ERR_INVALID_ARG, "negative length");
  if (p->bm->active(seq)) return fail(PA_ERR_SEQ_EXISTS, "pa_swap_in: sequence exists");
  DeviceGuard guard(p->d.device);
  if (!guard.ok) return fail(PA_ERR_CUDA, "cannot select the pool's device");
  st = check_host_image(host, host_bytes, swap_image_bytes(p->d, n_tokens));
  if (st != PA_OK) return st;
  p->cows.clear();
  pa::logf(2, "swap_in: sequence %d, %d tokens, %zu bytes", seq, n_tokens, host_bytes);
  st = bm_status(p->bm->reserve(seq, n_tokens, &p->cows), "pa_swap_in");
  if (st != PA_OK) return st;
  st = swap_copies(p, p->bm->table(seq), static_cast<char*>(const_cast<void*>(host)), false,
                   static_cast<cudaStream_t>(stream));
  if (st != PA_OK) p->bm->release(seq);
  return st;
}

pa_status pa_append_kv(pa_pool* p, int32_t layer, int32_t T, const int32_t* seqs,
                       const int32_t* positions, const void* k_new, const void* v_new,
                       void* stream) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  if (layer < 0 || layer >= p->d.num_layers) return fail(PA_ERR_INVALID_ARG, "layer out of range");
  if (T < 0 || (T > 0 && (!seqs || !positions || !k_new || !v_new)))
    return fail(PA_ERR_INVALID_ARG, "null argument");
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15)
    return fail(PA_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  if (T == 0) return PA_OK;
  p->slots.resize(T);
  for (int32_t t = 0; t < T; ++t) {
    pa_status st = seq_arg(p, seqs[t]);
    if (st != PA_OK) return st;
    st = bm_status(p->bm->slot(seqs[t], positions[t], &p->slots[t]), "pa_append_kv");
    if (st != PA_OK) return st;
  }
  DeviceGuard guard(p->d.device);
  if (!guard.ok) return fail(PA_ERR_CUDA, "cannot select the pool's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pa_status st = ensure_device(p, s);
  if (st != PA_OK) return st;
  pa::MirrorDeltas& md = p->bm->deltas();
  const int nd = static_cast<int>(md.size());
  int launches = 0;
  cudaError_t e = pa::launch_append(p->view, layer, p->slots.data(), T, k_new, v_new,
                                    md.indices().data(), md.values().data(), nd, s, &launches);
  p->launches += launches;
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  md.consume(nd);
  pa::logf(2, "append_kv: layer %d, %d rows, %d table updates", layer, T, nd);
  return PA_OK;
}

namespace {

// The plan of one decode launch over the leading items of seqs[0, n): as many
// as the parameter capacity and (fixed partitions) the workspace's partial
// slots allow.  *cnt = items taken, *blocks = their 16-token tiles; *sib tells
// whether a sibling plan (sp) replaces the plain one.
pa_status plan_launch(pa_pool* p, const int32_t* seqs, int32_t n, int32_t group, int mode,
                      int32_t part_blocks, int cap, pa::DecodePlan& plan, bool* sib, pa::SibPlan& sp,
                      int32_t* cnt_out, int64_t* blocks_out) {
  const int H = p->d.num_kv_heads;
  const int64_t slots_cap = p->view.partial_slots;
  const int32_t alpha = pa::stream_k_alpha(p->d.kv_dtype);
  int32_t cnt = 0;
  int64_t work = 0, blocks = 0;
  plan.pre[0] = 0;
  while (cnt < n && cnt < pa::kDecodeItemsCap) {
    const int32_t len = p->bm->len(seqs[cnt]);
    const int32_t nb = (len + 15) / 16;
    int64_t units = nb + alpha;
    if (mode == pa::kSplitFixed) units = (nb + part_blocks - 1) / part_blocks;
    if (mode == pa::kSplitNever) units = 1;
    if (mode == pa::kSplitFixed && cnt > 0 && (work + units) * H > slots_cap) break;
    if (cnt > 0 && (work + units) * H >= (int64_t{1} << 30)) break;  // device positions are int32
    if (mode == pa::kSplitFixed && units * H > slots_cap)
      return fail(PA_ERR_INVALID_ARG, "partition_tokens too small for the workspace");
    plan.seq[cnt] = seqs[cnt];
    plan.len[cnt] = len;
    work += units;
    blocks += nb;
    plan.pre[cnt + 1] = static_cast<int32_t>(work);
    ++cnt;
  }
  plan.n = cnt;
  plan.mode = mode;
  plan.part_blocks = part_blocks;
  plan.alpha = mode == pa::kSplitStreamK ? alpha : 0;
  plan.pad_ = 0;
  plan.per_head = work;
  const int64_t total = work * H;
  int64_t W = std::min<int64_t>(cap, total);
  if (mode != pa::kSplitStreamK) {
    // whole partitions (or sequences) per worker: the same count for every
    // worker, so no worker runs a round more than the others
    const int64_t rounds = (total + cap - 1) / cap;
    W = (total + rounds - 1) / rounds;
  } else {
    W = std::min<int64_t>(W, std::max<int64_t>(1, (total + kMinBlocksPerWorker - 1) / kMinBlocksPerWorker));
    W = std::min<int64_t>(W, slots_cap / 2);
  }
  plan.workers = static_cast<int32_t>(std::max<int64_t>(1, W));
  *sib = mode == pa::kSplitStreamK && group <= 4 &&
         build_sib_plan(p, seqs, cnt, group, cap, sp, p->order, p->set_of);
  *cnt_out = cnt;
  *blocks_out = blocks;
  return PA_OK;
}

// pa_decode_attention, and with k_new / v_new the fused append of
// pa_decode_attention_append (validated by the caller).
pa_status decode_call(pa_pool* p, int32_t layer, int32_t n, const int32_t* seqs,
                      int32_t num_q_heads, const void* q, void* out, float scale,
                      int32_t partition_tokens, void* stream, const void* k_new, const void* v_new) {
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  if (layer < 0 || layer >= p->d.num_layers) return fail(PA_ERR_INVALID_ARG, "layer out of range");
  if (n < 0 || (n > 0 && (!seqs || !q || !out))) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (num_q_heads <= 0 || num_q_heads % p->d.num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads must be a multiple of num_kv_heads");
  const int32_t group = num_q_heads / p->d.num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PA_ERR_INVALID_ARG, "query group (num_q_heads / num_kv_heads) must be 1, 2, 4 or 8");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(PA_ERR_INVALID_ARG, "q / out must be 16-byte aligned");
  int mode = pa::kSplitStreamK;
  int part_blocks = 0;
  if (partition_tokens == -1) {
    mode = pa::kSplitNever;
  } else if (partition_tokens > 0) {
    if (partition_tokens % p->d.block_size != 0 || partition_tokens < p->d.min_partition_tokens)
      return fail(PA_ERR_INVALID_ARG,
                  "partition_tokens must be a multiple of block_size and >= min_partition_tokens");
    mode = pa::kSplitFixed;
    part_blocks = partition_tokens / 16;  // in the kernel's 16-token tiles
  } else if (partition_tokens != 0) {
    return fail(PA_ERR_INVALID_ARG, "partition_tokens must be 0, -1 or positive");
  }
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite");
  for (int32_t i = 0; i < n; ++i) {
    pa_status st = seq_arg(p, seqs[i]);
    if (st != PA_OK) return st;
    if (!p->bm->active(seqs[i])) return fail(PA_ERR_NO_SEQ, "pa_decode_attention: no such sequence");
    if (p->bm->len(seqs[i]) < 1) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: empty sequence");
  }
  p->last_sets = 0;
  p->last_tiles = 0;
  if (n == 0) return PA_OK;
  DeviceGuard guard(p->d.device);
  if (!guard.ok) return fail(PA_ERR_CUDA, "cannot select the pool's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pa_status st = ensure_device(p, s);
  if (st != PA_OK) return st;
  st = flush_deltas(p, s);
  if (st != PA_OK) return st;

  const int H = p->d.num_kv_heads;
  // G = 8 over 16-bit KV is a real 8-column contraction: the tcgen05 kernel
  // (one worker per SM) unless the caller asked for the warp-level kernel
  const bool tc = (p->path == PA_DECODE_TCGEN05 || (p->path == PA_DECODE_AUTO && kAutoTcgen05)) &&
                  pa::decode_tc_applies(p->d.kv_dtype, group);
  const int cap = tc ? pa::decode_tc_worker_capacity(p->num_sms)
                     : pa::decode_worker_capacity(p->d.kv_dtype, group, p->num_sms);
  p->last_tc = false;
  pa::DecodeArgs args;
  args.use_tc = 0;
  args.k_new = k_new;
  args.v_new = v_new;
  args.q = q;
  args.out = out;
  args.layer = layer;
  args.num_q_heads = num_q_heads;
  args.group = group;
  args.scale = scale;
  args.q_item_stride = static_cast<int64_t>(num_q_heads) * pa::kHeadDim;
  pa_pool::PlanCache& pc = p->cache;
  const bool hit = pc.valid && pc.version == p->bm->version() && pc.group == group && pc.mode == mode &&
                   pc.part_blocks == part_blocks && pc.tc == tc &&
                   pc.seqs.size() == static_cast<size_t>(n) &&
                   std::equal(seqs, seqs + n, pc.seqs.begin());
  pa::DecodePlan& plan = pc.plan;
  const uint64_t launches0 = p->launches;
  int32_t at = 0;
  while (at < n) {
    // Items of this launch: up to the parameter capacity, and (fixed mode) the
    // partial slots the workspace holds.
    int32_t cnt = 0;
    int64_t blocks = 0;
    if (hit) {  // the previous call's single launch, same tables
      cnt = n;
      blocks = pc.blocks;
    } else {
      pc.valid = false;
      const pa_status st = plan_launch(p, seqs + at, n - at, group, mode, part_blocks, cap, plan,
                                       &pc.sib, pc.sib_plan, &cnt, &blocks);
      if (st != PA_OK) return st;
      if (at == 0 && cnt == n) {
        pc.valid = true;
        pc.version = p->bm->version();
        pc.group = group;
        pc.mode = mode;
        pc.part_blocks = part_blocks;
        pc.tc = tc;
        pc.blocks = blocks;
        pc.seqs.assign(seqs, seqs + n);
      }
    }
    args.item_offset = at;
    int launches = 0;
    cudaError_t e;
    const pa::SibPlan& sib = pc.sib_plan;
    if (pc.sib) {
      if (k_new != nullptr) {
        // Sibling sets put several sequences' last blocks back to back in one
        // worker's share; that worker's row patches would run in series, so the
        // rows go in with the append kernel instead (same cache contents).
        p->slots.resize(cnt);
        for (int32_t t = 0; t < cnt; ++t)
          p->bm->slot(seqs[at + t], p->bm->len(seqs[at + t]) - 1, &p->slots[t]);
        const size_t row = static_cast<size_t>(p->d.num_kv_heads) * pa::kHeadDim * 2;
        int al = 0;
        e = pa::launch_append(p->view, layer, p->slots.data(), cnt,
                              static_cast<const uint8_t*>(k_new) + at * row,
                              static_cast<const uint8_t*>(v_new) + at * row, nullptr, nullptr, 0, s, &al);
        p->launches += al;
        if (e != cudaSuccess) return cuda_fail(e, "append launch");
        args.k_new = args.v_new = nullptr;
      }
      e = pa::launch_decode_sib(p->view, p->maps, sib, args, s, &launches);
      args.k_new = k_new;
      args.v_new = v_new;
      p->last_sets += sib.sets;
      p->last_tiles += (sib.per_head - static_cast<int64_t>(sib.alpha) * sib.nu) * H;
    } else {
      args.use_tc = tc ? 1 : 0;
      e = pa::launch_decode(p->view, p->maps, plan, args, s, &launches);
      args.use_tc = 0;
      p->last_tiles += blocks * H;
      p->last_tc = p->last_tc || tc;
    }
    p->launches += launches;
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    at += cnt;
  }
  pa::logf(2, "decode: layer %d, %d sequences, G=%d, %s kernel, %s split (%d-tile partitions), "
           "%d sibling sets, %s, %llu launches, plan %s", layer, n, group,
           p->last_tc ? "tcgen05" : "warp-level",
           mode == pa::kSplitNever ? "no" : mode == pa::kSplitFixed ? "fixed" : "stream-K", part_blocks,
           p->last_sets, k_new != nullptr ? "append fused" : "no append",
           static_cast<unsigned long long>(p->launches - launches0), hit ? "reused" : "built");
  return PA_OK;
}

}  // namespace

pa_status pa_decode_attention(pa_pool* p, int32_t layer, int32_t n, const int32_t* seqs,
                              int32_t num_q_heads, const void* q, void* out, float scale,
                              int32_t partition_tokens, void* stream) {
  PA_RANGE();
  g_last_error.clear();
  return decode_call(p, layer, n, seqs, num_q_heads, q, out, scale, partition_tokens, stream,
                     nullptr, nullptr);
}

pa_status pa_decode_attention_append(pa_pool* p, int32_t layer, int32_t n, const int32_t* seqs,
                                     const void* k_new, const void* v_new, int32_t num_q_heads,
                                     const void* q, void* out, float scale,
                                     int32_t partition_tokens, void* stream) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  if (layer < 0 || layer >= p->d.num_layers) return fail(PA_ERR_INVALID_ARG, "layer out of range");
  if (n < 0 || (n > 0 && (!seqs || !k_new || !v_new))) return fail(PA_ERR_INVALID_ARG, "null argument");
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15)
    return fail(PA_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  // the target slot of every item: the last reserved position of its sequence,
  // in a block no other sequence shares; each sequence at most once
  p->a.assign(n, 0);
  std::vector<int32_t>& seen = p->b;
  seen.assign(p->d.max_seqs, 0);
  for (int32_t i = 0; i < n; ++i) {
    pa_status st = seq_arg(p, seqs[i]);
    if (st != PA_OK) return st;
    if (!p->bm->active(seqs[i])) return fail(PA_ERR_NO_SEQ, "pa_decode_attention_append: no such sequence");
    if (seen[seqs[i]]++) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention_append: a sequence named twice");
    const int32_t len = p->bm->len(seqs[i]);
    if (len < 1) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention_append: empty sequence");
    int64_t slot = 0;
    st = bm_status(p->bm->slot(seqs[i], len - 1, &slot), "pa_decode_attention_append");
    if (st != PA_OK) return st;
  }
  return decode_call(p, layer, n, seqs, num_q_heads, q, out, scale, partition_tokens, stream, k_new,
                     v_new);
}

pa_status pa_get_seq(pa_pool* p, int32_t seq, int32_t* len, int32_t* table, int32_t cap,
                     int32_t* nblocks) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  pa_status st = seq_arg(p, seq);
  if (st != PA_OK) return st;
  if (!p->bm->active(seq)) return fail(PA_ERR_NO_SEQ, "pa_get_seq: no such sequence");
  const std::vector<int32_t>& t = p->bm->table(seq);
  if (cap > 0 && !table) return fail(PA_ERR_INVALID_ARG, "null table with cap > 0");
  const int32_t m = std::min<int32_t>(cap, static_cast<int32_t>(t.size()));
  if (m > 0) std::memcpy(table, t.data(), sizeof(int32_t) * m);
  if (len) *len = p->bm->len(seq);
  if (nblocks) *nblocks = static_cast<int32_t>(t.size());
  return PA_OK;
}

pa_status pa_get_refcounts(pa_pool* p, int32_t* out, int32_t cap) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !out) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (cap < p->d.num_blocks) return fail(PA_ERR_INVALID_ARG, "cap < num_blocks");
  for (int32_t b = 0; b < p->d.num_blocks; ++b) out[b] = p->bm->refcount(b);
  return PA_OK;
}

pa_status pa_get_free_list(pa_pool* p, int32_t* out, int32_t cap, int32_t* n) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !n || (cap > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "null argument");
  std::vector<int32_t> fl;
  p->bm->free_list(&fl);
  const int32_t m = std::min<int32_t>(cap, static_cast<int32_t>(fl.size()));
  if (m > 0) std::memcpy(out, fl.data(), sizeof(int32_t) * m);
  *n = static_cast<int32_t>(fl.size());
  return PA_OK;
}

pa_status pa_get_cached_blocks(pa_pool* p, int32_t* out, int32_t cap, int32_t* n) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !n || (cap > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "null argument");
  std::vector<int32_t> cl;
  p->bm->cached_list(&cl);
  const int32_t m = std::min<int32_t>(cap, static_cast<int32_t>(cl.size()));
  if (m > 0) std::memcpy(out, cl.data(), sizeof(int32_t) * m);
  *n = static_cast<int32_t>(cl.size());
  return PA_OK;
}

pa_status pa_get_cow_log(pa_pool* p, int32_t* pairs, int32_t cap, int32_t* n) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !n || (cap > 0 && !pairs)) return fail(PA_ERR_INVALID_ARG, "null argument");
  const int32_t m = std::min<int32_t>(cap, static_cast<int32_t>(p->cow_log.size()));
  for (int32_t k = 0; k < m; ++k) {
    pairs[2 * k] = p->cow_log[k].src;
    pairs[2 * k + 1] = p->cow_log[k].dst;
  }
  *n = static_cast<int32_t>(p->cow_log.size());
  return PA_OK;
}

uint64_t pa_launch_count(const pa_pool* p) { return p ? p->launches : 0; }

pa_status pa_set_decode_path(pa_pool* p, int32_t path) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (path != PA_DECODE_AUTO && path != PA_DECODE_WARP && path != PA_DECODE_TCGEN05)
    return fail(PA_ERR_INVALID_ARG, "path must be PA_DECODE_AUTO, PA_DECODE_WARP or PA_DECODE_TCGEN05");
  p->path = path;
  return PA_OK;
}

pa_status pa_last_decode_kernel(const pa_pool* p, int32_t* tcgen05) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !tcgen05) return fail(PA_ERR_INVALID_ARG, "null argument");
  *tcgen05 = p->last_tc ? 1 : 0;
  return PA_OK;
}

pa_status pa_plan_siblings(const pa_pool* p, int32_t n, const int32_t* seqs, int32_t group,
                           int32_t* set_of, int32_t* set_cp, int32_t* n_sets) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || (n > 0 && (!seqs || !set_of || !set_cp)) || !n_sets)
    return fail(PA_ERR_INVALID_ARG, "null argument");
  if (n < 0 || n > pa::kDecodeItemsCap)
    return fail(PA_ERR_INVALID_ARG, "n must be in [0, 512] (one launch's items)");
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PA_ERR_INVALID_ARG, "group must be 1, 2, 4 or 8");
  for (int32_t i = 0; i < n; ++i) {
    pa_status st = seq_arg(p, seqs[i]);
    if (st != PA_OK) return st;
    if (!p->bm->active(seqs[i])) return fail(PA_ERR_NO_SEQ, "pa_plan_siblings: no such sequence");
    if (p->bm->len(seqs[i]) < 1) return fail(PA_ERR_INVALID_ARG, "pa_plan_siblings: empty sequence");
  }
  static thread_local pa::SibPlan sp;
  std::vector<int32_t> order, set_idx;
  int32_t sets = 0;
  if (build_sib_plan(p, seqs, n, group, pa::kMaxWorkers, sp, order, set_idx)) sets = sp.sets;
  for (int32_t i = 0; i < n; ++i) set_of[i] = sets ? set_idx[i] : -1;
  const int tpb = p->d.block_size / 16;  // the plan counts 16-token tiles
  for (int32_t k = 0; k < sets; ++k) set_cp[k] = sp.cp[k] / tpb;
  *n_sets = sets;
  return PA_OK;
}

pa_status pa_check_device_errors(pa_pool* p, void* stream, uint32_t* bits) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !bits) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (p->host_only) return fail(PA_ERR_INVALID_ARG, "host-only pool: no device buffers");
  DeviceGuard guard(p->d.device);
  if (!guard.ok) return fail(PA_ERR_CUDA, "cannot select the pool's device");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!p->dev_ready) {
    *bits = 0;
    return PA_OK;
  }
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0;
  e = cudaMemcpy(&v, p->view.err, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  e = cudaMemset(p->view.err, 0, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  if (v & PA_DEVERR_TIMEOUT) {
    // a worker that gave up may have left a stream-K arrival counter raised
    e = cudaMemset(p->view.counters, 0, counter_bytes(p->d));
    if (e != cudaSuccess) return cuda_fail(e, "clear counters");
  }
  *bits = v;
  if (v) {
    char buf[96];
    std::snprintf(buf, sizeof(buf), "device check failed: bits 0x%x", v);
    return fail(PA_ERR_DEVICE_CHECK, buf);
  }
  return PA_OK;
}

pa_status pa_last_decode_plan(const pa_pool* p, int32_t* shared_sets, int64_t* kv_tiles) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  if (shared_sets) *shared_sets = p->last_sets;
  if (kv_tiles) *kv_tiles = p->last_tiles;
  return PA_OK;
}

pa_status pa_state_size(const pa_pool* p, size_t* bytes) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !bytes) return fail(PA_ERR_INVALID_ARG, "null argument");
  std::vector<int32_t> w;
  p->bm->save_state(&w);
  *bytes = w.size() * sizeof(int32_t);
  return PA_OK;
}

pa_status pa_state_save(const pa_pool* p, void* buf, size_t cap, size_t* written) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || !buf || !written) return fail(PA_ERR_INVALID_ARG, "null argument");
  std::vector<int32_t> w;
  p->bm->save_state(&w);
  const size_t bytes = w.size() * sizeof(int32_t);
  if (cap < bytes) return fail(PA_ERR_INVALID_ARG, "pa_state_save: buffer smaller than pa_state_size");
  std::memcpy(buf, w.data(), bytes);
  *written = bytes;
  return PA_OK;
}

pa_status pa_state_load(pa_pool* p, const void* buf, size_t bytes) {
  PA_RANGE();
  g_last_error.clear();
  if (!p || (!buf && bytes > 0)) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (bytes % sizeof(int32_t) != 0) return fail(PA_ERR_INVALID_ARG, "pa_state_load: not a state image");
  std::vector<int32_t> w(bytes / sizeof(int32_t));
  if (bytes > 0) std::memcpy(w.data(), buf, bytes);
  if (p->bm->load_state(w.data(), w.size()) != pa::kOk)
    return fail(PA_ERR_INVALID_ARG,
                "pa_state_load: not a consistent state image of a pool with this geometry");
  p->cow_log.clear();
  p->cows.clear();
  p->cache.valid = false;
  pa::logf(2, "state_load: %zu bytes", bytes);
  return PA_OK;
}

pa_status pa_debug_fail_after(pa_pool* p, int32_t n) {
  PA_RANGE();
  g_last_error.clear();
  if (!p) return fail(PA_ERR_INVALID_ARG, "null pool");
  p->bm->set_fail_after(n);
  return PA_OK;
}

const char* pa_last_error(void) { return g_last_error.c_str(); }

const char* pa_status_string(int32_t s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_NO_BLOCKS: return "PA_ERR_NO_BLOCKS";
    case PA_ERR_NO_SEQ: return "PA_ERR_NO_SEQ";
    case PA_ERR_SEQ_EXISTS: return "PA_ERR_SEQ_EXISTS";
    case PA_ERR_SHARED_BLOCK: return "PA_ERR_SHARED_BLOCK";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_DEVICE_CHECK: return "PA_ERR_DEVICE_CHECK";
    default: return "PA_UNKNOWN_STATUS";
  }
}

}  // extern "C"
