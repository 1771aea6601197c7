// Interfaces between the C-ABI layer (api.cpp) and the CUDA kernels.
//
// Per-launch metadata travels in the kernel parameters (up to ~30 KB), so a
// decode step needs no host-to-device copy: the block-table deltas of the
// step ride along with the append (or copy-on-write) launch that precedes the
// decode, and the decode launch carries its sequence ids and work prefix sums.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>

namespace pa {

enum DType : int32_t { kBF16 = 0, kFP16 = 1, kFP8 = 2 };

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;          // query heads per KV head handled by one warp
constexpr int kPartialRowFloats = kHeadDim;
// One split-KV partial slot: o[8][128] unnormalised fp32, then (m, l)[8].
constexpr int kPartialSlotFloats = kMaxGroup * (kHeadDim + 2);
constexpr int kMaxWorkers = 2048;     // warps of one decode launch (stream-K slots = 2x)

// Device error word bits (mirrored in pa.h).
constexpr uint32_t kErrBadBlock = 0x1u;
constexpr uint32_t kErrBadLen = 0x2u;
constexpr uint32_t kErrTimeout = 0x4u;

// ---------------------------------------------------------------- pool view
struct PoolView {
  void* k_cache;
  void* v_cache;
  const float* k_scale;
  const float* v_scale;
  const float* k_inv;
  const float* v_inv;
  int32_t* meta;        // [tables: max_seqs*mbps][lens: max_seqs]
  int32_t* tables;      // = meta
  int32_t* lens;        // = meta + max_seqs*mbps
  float* partials;      // [slots][kPartialSlotFloats]
  int32_t* counters;    // [kMaxWorkers] stream-K arrival counters, zero between launches
  uint32_t* err;
  int64_t partial_slots;
  int32_t num_layers, num_kv_heads, block_size, num_blocks, max_seqs, mbps;
  int32_t kv_dtype, act_dtype;
};

// ------------------------------------------------------ metadata payloads
// One int32 payload array shared by the small launches; each launcher
// documents its own packing.
template <int CAP>
struct Payload {
  int32_t v[CAP];
};

constexpr int kPayloadSmall = 512;
constexpr int kPayloadLarge = 7168;

// ------------------------------------------------------------ launchers
// Apply `n` deltas (idx[k], val[k]) to pool.meta.
cudaError_t launch_meta_apply(const PoolView& pool, const int32_t* idx, const int32_t* val,
                              int n, cudaStream_t stream);

// Copy-on-write: copy the whole (all layers, K and V) physical block
// src[k] -> dst[k] for k < n; also applies `nd` mirror deltas.
cudaError_t launch_cow_copy(const PoolView& pool, const int32_t* src, const int32_t* dst, int n,
                            const int32_t* didx, const int32_t* dval, int nd,
                            cudaStream_t stream, int* launches);

// Append T rows: slot[t] = block * B + offset; also applies `nd` deltas.
cudaError_t launch_append(const PoolView& pool, int layer, const int64_t* slots, int T,
                          const void* k_new, const void* v_new,
                          const int32_t* didx, const int32_t* dval, int nd,
                          cudaStream_t stream, int* launches);

// Decode work description, computed on the host from the host block tables.
enum SplitMode : int32_t { kSplitStreamK = 0, kSplitFixed = 1, kSplitNever = 2 };

constexpr int kDecodeItemsCap = 512;

struct DecodePlan {
  int32_t n;              // items in this launch (<= kDecodeItemsCap)
  int32_t mode;           // SplitMode
  int32_t part_blocks;    // fixed mode: blocks per partition
  int32_t workers;        // warps that carry work
  int32_t alpha;          // stream-K: cost positions in front of each item's blocks
  int32_t pad_;
  int64_t per_head;       // work positions per KV head (stream-K: sum of alpha + blocks)
  int32_t seq[kDecodeItemsCap];       // table row of each item
  int32_t len[kDecodeItemsCap];       // tokens of each item
  int32_t pre[kDecodeItemsCap + 1];   // prefix of per-item work units
};

// Decode work in which forks of one prompt are read together (stream-K only).
// Sequences whose block tables start with the same run of full blocks form a
// sibling set; the set is ONE work unit: the common prefix, read once with
// every member's query rows side by side on the tensor-core tile (members x
// G <= 8), followed by each member's own blocks, on which only that member's
// rows count.  Every other sequence is a unit of its own.
struct SibPlan {
  int32_t n;              // items
  int32_t nu;             // units
  int32_t workers;
  int32_t sets;           // units 0 .. sets-1 are sibling sets, the rest single items
  int32_t alpha;          // cost positions in front of each unit's blocks
  int32_t pad_;
  int64_t per_head;       // work positions per head: sum over units of alpha + blocks
  int32_t seq[kDecodeItemsCap];       // table row of each item
  int32_t len[kDecodeItemsCap];       // tokens of each item
  int32_t part[kDecodeItemsCap];      // first position of the item's own blocks in its unit
  int32_t pre[kDecodeItemsCap + 1];   // prefix of per-unit block counts
  int32_t cp[kDecodeItemsCap];        // shared full blocks at the start of the unit
  int16_t mem0[kDecodeItemsCap + 1];  // unit u holds items mem[mem0[u] .. mem0[u+1])
  int16_t mem[kDecodeItemsCap];
};

struct DecodeArgs {
  const void* q;
  void* out;
  int32_t layer;
  int32_t num_q_heads;
  int32_t group;          // G = num_q_heads / num_kv_heads
  float scale;            // softmax scale
  int64_t q_item_stride;  // elements between consecutive items of q / out (num_q_heads*128)
  int32_t item_offset;    // index of plan item 0 within the caller's arrays
  const void* k_new;      // fused append: [n][H_kv][128] rows of each item's last token,
  const void* v_new;      // or null (no append)
  int32_t use_tc = 0;     // plain plans with G = 8 over 16-bit KV: the tcgen05 kernel
};

// Stream-K cost positions per work unit, in KV blocks: they stand for the
// fixed cost of a segment (query load, finish, partial write, arrival, the
// merge) and, by shrinking the shares of workers that cross unit boundaries,
// also move boundaries off units so fewer units are cut.  Chosen by a sweep
// on B200 (0 .. 16 for 16-bit and FP8 KV; 8B-, 70B- and 7B-class layers and
// 32K-token FP8): 12 was best or within noise of best everywhere.
inline int32_t stream_k_alpha(int32_t /*kv_dtype*/) { return 12; }

// Number of decode workers (warps) that fit on the device at once.
int decode_worker_capacity(int kv_dtype, int group, int num_sms);
int decode_warps_per_cta();

// TMA tensor maps of a cache (tensor_maps.cpp): the 2-D view [rows][128] with
// boxes of 16 rows x 128 bytes, and for 16-bit caches the 3-D view
// [2 d-halves][rows][64] whose box {64, 16, 2} is a whole 16-row tile.
struct CacheMaps {
  CUtensorMap k, v;
  CUtensorMap k3, v3;  // copies of k / v for FP8 caches
};
// Returns null on success, else what failed.
const char* encode_cache_maps(void* k_cache, void* v_cache, int kv_dtype, int64_t rows, CacheMaps* maps);

cudaError_t launch_decode(const PoolView& pool, const CacheMaps& maps, const DecodePlan& plan,
                          const DecodeArgs& args, cudaStream_t stream, int* launches);
// Same for a plan with shared entries; group must be 1, 2 or 4.
cudaError_t launch_decode_sib(const PoolView& pool, const CacheMaps& maps, const SibPlan& plan,
                              const DecodeArgs& args, cudaStream_t stream, int* launches);

// The tcgen05 decode (kernels_decode_tc.cu): plain plans, G = 8, 16-bit KV;
// one worker per SM.  launch_decode calls it when args.use_tc is set.
bool decode_tc_applies(int kv_dtype, int group);
int decode_tc_worker_capacity(int num_sms);
cudaError_t launch_decode_tc(const PoolView& pool, const CacheMaps& maps, const DecodePlan& plan,
                             const DecodeArgs& args, cudaStream_t stream);

// Thread-local text returned by pa_last_error() (defined in api.cpp).
void set_last_error(const std::string& msg);

// Device properties the planner needs (cached per device by the caller).
struct DeviceInfo {
  int num_sms = 0;
  int device = -1;
};

}  // namespace pa
