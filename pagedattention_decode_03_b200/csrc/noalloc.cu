// pa_decode_attention_noalloc: decode attention for callers that cannot
// allocate device memory.
//
// Some callers own no allocator: a plugin or custom-operator interface of a
// host engine hands the kernel only its input and output buffers (the engine
// reserves all free HBM for its own KV pool up front and forbids side
// allocations), or a caller runs under a hard per-process memory cap where an
// extra cudaMalloc fails.  Such callers cannot create a pool, whose workspace
// (block-table mirror, split-KV partials) must be allocated by the caller.
//
// This entry point needs no pool and no workspace.  The caller passes the
// cache, its own device block tables and the sequence lengths (host) plus q
// and out (the lengths travel in the launch parameters); the split-KV
// scratch -- partial results, arrival counters and an error word -- lives in
// one file-scope __device__ array of
// kScratchBytes (12 MiB) that every GPU loading this library holds until the
// process exits.  The kernel's bounds checks set bits in the error word (a
// table entry outside the pool, a bounded wait that gave up); the bits stay
// set across calls until pa_noalloc_check_errors reads and clears them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_internal.h"
#include "trace.h"

namespace {

constexpr size_t kScratchBytes = size_t{12} << 20;
constexpr size_t kCountersOff = 0;                                          // int32[kMaxWorkers]
constexpr size_t kErrOff = kCountersOff + sizeof(int32_t) * pa::kMaxWorkers;  // uint32
constexpr size_t kPartialsOff = kErrOff + 256;
constexpr int64_t kScratchSlots =
    static_cast<int64_t>((kScratchBytes - kPartialsOff) / (sizeof(float) * pa::kPartialSlotFloats));
constexpr int kMaxDevices = 64;

static_assert(kPartialsOff % 256 == 0, "partials must stay 256-byte aligned");
static_assert(kScratchSlots >= 2 * 1184, "scratch must hold two partials per B200 worker");

// The scratch.  Host code must not use this name as an address: it is a host
// stand-in for the device symbol; the device address comes from
// cudaGetSymbolAddress below.
__device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
uint8_t* g_scratch_dev[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

pa_status fail(pa_status s, const std::string& m) {
  pa::set_last_error(m);  // reported by pa_last_error()
  return s;
}

// Once per device, with that device current: the scratch's device address
// and the SM count.
pa_status setup_device(int dev, uint8_t** scratch, int* sms) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_dev[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return fail(PA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
      return fail(PA_ERR_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
    g_num_sms[dev] = n;
    g_scratch_dev[dev] = static_cast<uint8_t*>(ptr);
  }
  *scratch = g_scratch_dev[dev];
  *sms = g_num_sms[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_attention_noalloc(const pa_pool_desc* d, int32_t layer, int32_t n,
                                                 const int32_t* block_tables,
                                                 const int32_t* seq_lens, int32_t num_q_heads,
                                                 const void* q, void* out, float scale,
                                                 void* stream) {
  PA_RANGE();
  pa::set_last_error("");
  if (!d || !block_tables || !seq_lens || !q || !out || !d->k_cache || !d->v_cache)
    return fail(PA_ERR_INVALID_ARG, "null argument");
  if (d->head_dim != pa::kHeadDim || d->block_size != 16)
    return fail(PA_ERR_INVALID_ARG, "head_dim must be 128 and block_size 16");
  if (d->num_layers <= 0 || d->num_kv_heads <= 0 || d->num_blocks <= 0 || d->max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "sizes must be positive");
  if (layer < 0 || layer >= d->num_layers) return fail(PA_ERR_INVALID_ARG, "layer out of range");
  if (d->kv_dtype < PA_BF16 || d->kv_dtype > PA_FP8_E4M3 ||
      (d->act_dtype != PA_BF16 && d->act_dtype != PA_FP16) ||
      (d->kv_dtype != PA_FP8_E4M3 && d->kv_dtype != d->act_dtype))
    return fail(PA_ERR_INVALID_ARG, "bad dtypes");
  if (d->kv_dtype == PA_FP8_E4M3 && (!d->k_scale || !d->v_scale))
    return fail(PA_ERR_INVALID_ARG, "FP8 caches need k_scale and v_scale");
  if (static_cast<int64_t>(d->num_layers) * d->num_blocks * d->num_kv_heads * 16 >= (int64_t{1} << 31))
    return fail(PA_ERR_INVALID_ARG, "pool too large: layers*blocks*kv_heads*16 >= 2^31");
  if (n < 1 || n > pa::kDecodeItemsCap)
    return fail(PA_ERR_INVALID_ARG, "n must be in [1, 512]: the no-allocation scratch holds at most "
                                    "512 sequences per call");
  if (num_q_heads <= 0 || num_q_heads % d->num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads must be a multiple of num_kv_heads");
  const int32_t group = num_q_heads / d->num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PA_ERR_INVALID_ARG, "query group must be 1, 2, 4 or 8");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out) |
       reinterpret_cast<uintptr_t>(d->k_cache) | reinterpret_cast<uintptr_t>(d->v_cache)) & 15)
    return fail(PA_ERR_INVALID_ARG, "q, out and the caches must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite");
  if (static_cast<int64_t>(n) * d->max_blocks_per_seq >= (int64_t{1} << 31))
    return fail(PA_ERR_INVALID_ARG, "block tables too large");
  static thread_local pa::DecodePlan plan;
  int64_t work = 0;
  const int32_t alpha = pa::stream_k_alpha(d->kv_dtype);
  plan.pre[0] = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t len = seq_lens[i];
    if (len < 1 || (len + 15) / 16 > d->max_blocks_per_seq)
      return fail(PA_ERR_INVALID_ARG, "sequence " + std::to_string(i) +
                                          ": length must be in [1, max_blocks_per_seq * 16]");
    plan.seq[i] = i;  // row i of the caller's block tables
    plan.len[i] = len;
    work += alpha + (len + 15) / 16;
    plan.pre[i + 1] = static_cast<int32_t>(work);
  }
  if (work * d->num_kv_heads >= (int64_t{1} << 30))
    return fail(PA_ERR_INVALID_ARG, "too many KV blocks for one call (blocks x kv_heads >= 2^30)");

  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
  const int dev = d->device;
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_INVALID_ARG, "device ordinal out of range");
  if (prev != dev && cudaSetDevice(dev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaSetDevice failed");
  struct Restore {
    int prev, dev;
    ~Restore() {
      if (prev != dev) cudaSetDevice(prev);
    }
  } restore{prev, dev};

  uint8_t* scratch = nullptr;
  int sms = 0;
  pa_status st = setup_device(dev, &scratch, &sms);
  if (st != PA_OK) return st;
  pa::CacheMaps maps;
  const int64_t rows = static_cast<int64_t>(d->num_layers) * d->num_blocks * d->num_kv_heads * 16;
  if (const char* why = pa::encode_cache_maps(d->k_cache, d->v_cache, d->kv_dtype, rows, &maps))
    return fail(PA_ERR_CUDA, why);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pa::PoolView v{};
  v.k_cache = d->k_cache;
  v.v_cache = d->v_cache;
  v.k_scale = d->k_scale;
  v.v_scale = d->v_scale;
  v.counters = reinterpret_cast<int32_t*>(scratch + kCountersOff);
  v.lens = nullptr;  // the lengths travel in the launch parameters
  v.meta = nullptr;
  v.err = reinterpret_cast<uint32_t*>(scratch + kErrOff);
  v.partials = reinterpret_cast<float*>(scratch + kPartialsOff);
  v.partial_slots = kScratchSlots;
  v.tables = const_cast<int32_t*>(block_tables);
  v.num_layers = d->num_layers;
  v.num_kv_heads = d->num_kv_heads;
  v.block_size = 16;
  v.num_blocks = d->num_blocks;
  v.max_seqs = n;
  v.mbps = d->max_blocks_per_seq;
  v.kv_dtype = d->kv_dtype;
  v.act_dtype = d->act_dtype;

  // The scratch keeps the previous call's contents: the arrival counters must
  // start at zero.  The error word is left alone: its bits accumulate until
  // pa_noalloc_check_errors reads them.
  cudaError_t e = cudaMemsetAsync(scratch + kCountersOff, 0, sizeof(int32_t) * pa::kMaxWorkers, s);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));

  const int64_t total = work * d->num_kv_heads;
  int64_t W = std::min<int64_t>(pa::decode_worker_capacity(d->kv_dtype, group, sms), total);
  W = std::min<int64_t>(W, std::max<int64_t>(1, (total + 3) / 4));
  W = std::min<int64_t>(W, kScratchSlots / 2);
  plan.n = n;
  plan.mode = pa::kSplitStreamK;
  plan.part_blocks = 0;
  plan.alpha = alpha;
  plan.pad_ = 0;
  plan.per_head = work;
  plan.workers = static_cast<int32_t>(std::max<int64_t>(1, W));
  pa::DecodeArgs args;
  args.k_new = args.v_new = nullptr;
  args.q = q;
  args.out = out;
  args.layer = layer;
  args.num_q_heads = num_q_heads;
  args.group = group;
  args.scale = scale;
  args.q_item_stride = static_cast<int64_t>(num_q_heads) * pa::kHeadDim;
  args.item_offset = 0;
  int launches = 0;
  e = pa::launch_decode(v, maps, plan, args, s, &launches);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
  pa::logf(2, "decode_noalloc: layer %d, %d sequences, G=%d, %d workers", layer, n, group, plan.workers);
  return PA_OK;
}

extern "C" pa_status pa_noalloc_check_errors(int32_t device, void* stream, uint32_t* bits) {
  PA_RANGE();
  pa::set_last_error("");
  if (!bits) return fail(PA_ERR_INVALID_ARG, "null argument");
  if (device < 0 || device >= kMaxDevices) return fail(PA_ERR_INVALID_ARG, "device ordinal out of range");
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_dev[device]) {  // no call on this device yet: nothing to report
      *bits = 0;
      return PA_OK;
    }
  }
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
  if (prev != device && cudaSetDevice(device) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaSetDevice failed");
  struct Restore {
    int prev, dev;
    ~Restore() {
      if (prev != dev) cudaSetDevice(prev);
    }
  } restore{prev, device};
  uint8_t* scratch = nullptr;
  int sms = 0;
  pa_status st = setup_device(device, &scratch, &sms);
  if (st != PA_OK) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("cudaStreamSynchronize: ") + cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpy(&v, scratch + kErrOff, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("read error word: ") + cudaGetErrorString(e));
  e = cudaMemset(scratch + kErrOff, 0, sizeof(v));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, std::string("clear error word: ") + cudaGetErrorString(e));
  *bits = v;
  if (v != 0)
    return fail(PA_ERR_DEVICE_CHECK, "a no-allocation decode call reported device error bits 0x" +
                                         [v] { char b[16]; std::snprintf(b, sizeof b, "%x", v); return std::string(b); }());
  return PA_OK;
}
