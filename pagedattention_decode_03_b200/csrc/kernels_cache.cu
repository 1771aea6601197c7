// Kernels that write the cache and its device metadata:
//   * meta_apply   -- applies block-table / length deltas to the device mirror;
//   * cow_copy     -- copy-on-write of whole physical blocks (every layer, K and
//                     V), "Managing the KV Cache", Block Tables and Sharing;
//   * append       -- writes each new token's K/V rows into slot
//                     (table[seq][pos / B], pos % B) of one layer
//                     ("KV cache", paging paragraph; "Managing the KV Cache",
//                     Answer Key item 2), quantising to OCP FP8 E4M3 for an
//                     FP8 pool ("Managing the KV Cache", Quantized KV).
// All three are plain 16-byte vectorised copies bound by HBM bandwidth; the
// mirror deltas of a step ride in the parameters of whichever of them runs
// first, so a decode step needs no separate metadata transfer.
#include <algorithm>
#include <cstring>

#include "device_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

template <int CAP>
struct MetaParams {
  int32_t* meta;
  int32_t n;
  Payload<CAP> p;  // [idx (n)] [val (n)]
};

template <int CAP>
__global__ void meta_apply_kernel(const __grid_constant__ MetaParams<CAP> prm) {
  dev::grid_dep_wait();
  dev::grid_dep_launch();
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < prm.n; k += gridDim.x * blockDim.x)
    prm.meta[prm.p.v[k]] = prm.p.v[prm.n + k];
}

template <int CAP>
struct CowParams {
  uint4* k;
  uint4* v;
  int32_t* meta;
  int64_t layer_stride_v4;  // uint4 per layer (num_blocks * block_v4)
  int32_t block_v4;         // uint4 per (layer, block) slab: H * B * d * bytes / 16
  int32_t num_layers;
  int32_t n;                // copy pairs
  int32_t nd;               // mirror deltas
  Payload<CAP> p;           // [src (n)] [dst (n)] [idx (nd)] [val (nd)]
};

// grid.x = pairs * num_layers * 2 (K|V); each CTA copies one (layer, block) slab.
template <int CAP>
__global__ void __launch_bounds__(256) cow_copy_kernel(const __grid_constant__ CowParams<CAP> prm) {
  dev::grid_dep_wait();
  dev::grid_dep_launch();
  if (blockIdx.x == 0) {
    for (int k = threadIdx.x; k < prm.nd; k += blockDim.x)
      prm.meta[prm.p.v[2 * prm.n + k]] = prm.p.v[2 * prm.n + prm.nd + k];
  }
  const int job = blockIdx.x;
  const int kv = job & 1;
  const int layer = (job >> 1) % prm.num_layers;
  const int pair = (job >> 1) / prm.num_layers;
  const int64_t src = prm.p.v[pair];
  const int64_t dst = prm.p.v[prm.n + pair];
  uint4* base = kv ? prm.v : prm.k;
  const uint4* s = base + layer * prm.layer_stride_v4 + src * prm.block_v4;
  uint4* d = base + layer * prm.layer_stride_v4 + dst * prm.block_v4;
  for (int e = threadIdx.x; e < prm.block_v4; e += blockDim.x) d[e] = s[e];
}

template <int CAP>
struct AppendParams {
  const uint8_t* k_new;  // [T][H][128] act dtype
  const uint8_t* v_new;
  uint8_t* k_cache;
  uint8_t* v_cache;
  const float* k_inv;    // [L][H] fp32 (FP8 pools)
  const float* v_inv;
  int32_t* meta;
  int64_t layer_off;     // elements before this layer: layer * num_blocks * H * B * 128
  int32_t H, B;
  int32_t T, nd;
  int32_t layer;
  Payload<CAP> p;        // [slot (T)] [idx (nd)] [val (nd)]; slot = block * B + offset
};

// One warp per (token, head, K|V) row of 128 elements.
template <int KV, int ACT, int CAP>
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams<CAP> prm) {
  dev::grid_dep_wait();
  dev::grid_dep_launch();
  if (blockIdx.x == 0) {
    const int off = prm.T;
    for (int k = threadIdx.x; k < prm.nd; k += blockDim.x)
      prm.meta[prm.p.v[off + k]] = prm.p.v[off + prm.nd + k];
  }
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= prm.T * prm.H * 2) return;
  const int kv = row & 1;
  const int h = (row >> 1) % prm.H;
  const int t = (row >> 1) / prm.H;
  const int64_t slot = prm.p.v[t];
  const int64_t blk = slot / prm.B;
  const int64_t off = slot - blk * prm.B;
  const int64_t dst_el = prm.layer_off + ((blk * prm.H + h) * prm.B + off) * kHeadDim;
  const int64_t src_el = (static_cast<int64_t>(t) * prm.H + h) * kHeadDim;
  const uint8_t* src = (kv ? prm.v_new : prm.k_new) + src_el * 2;
  uint8_t* cache = kv ? prm.v_cache : prm.k_cache;
  if constexpr (KV == kFP8) {
    const float inv = (kv ? prm.v_inv : prm.k_inv)[prm.layer * prm.H + h];
    const uint2 raw = reinterpret_cast<const uint2*>(src)[lane];  // 4 act values
    float x0, x1, x2, x3;
    if constexpr (ACT == kBF16) {
      x0 = dev::bf16lo_to_f32(raw.x);
      x1 = dev::bf16hi_to_f32(raw.x);
      x2 = dev::bf16lo_to_f32(raw.y);
      x3 = dev::bf16hi_to_f32(raw.y);
    } else {
      x0 = dev::f16lo_to_f32(raw.x);
      x1 = dev::f16hi_to_f32(raw.x);
      x2 = dev::f16lo_to_f32(raw.y);
      x3 = dev::f16hi_to_f32(raw.y);
    }
    const uint16_t lo = dev::f32x2_to_e4m3x2(__fmul_rn(x0, inv), __fmul_rn(x1, inv));
    const uint16_t hi = dev::f32x2_to_e4m3x2(__fmul_rn(x2, inv), __fmul_rn(x3, inv));
    reinterpret_cast<uint32_t*>(cache + dst_el)[lane] =
        static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  } else {
    if (lane < 16) {  // 128 x 2 bytes = 16 lanes x 16 bytes
      const uint4 val = reinterpret_cast<const uint4*>(src)[lane];
      reinterpret_cast<uint4*>(cache + dst_el * 2)[lane] = val;
    }
  }
}

int kv_bytes(int dtype) { return dtype == kFP8 ? 1 : 2; }

template <int CAP>
cudaError_t do_meta_apply(const PoolView& pool, const int32_t* idx, const int32_t* val, int n,
                          cudaStream_t stream) {
  MetaParams<CAP> prm;
  prm.meta = pool.meta;
  prm.n = n;
  std::memcpy(prm.p.v, idx, sizeof(int32_t) * n);
  std::memcpy(prm.p.v + n, val, sizeof(int32_t) * n);
  const int threads = 256;
  const int blocks = std::max(1, std::min(64, (n + threads - 1) / threads));
  return launch_pdl(meta_apply_kernel<CAP>, dim3(blocks), dim3(threads), 0, stream, prm);
}

template <int CAP>
cudaError_t do_cow(const PoolView& pool, const int32_t* src, const int32_t* dst, int n,
                   const int32_t* didx, const int32_t* dval, int nd, cudaStream_t stream) {
  CowParams<CAP> prm;
  prm.k = static_cast<uint4*>(pool.k_cache);
  prm.v = static_cast<uint4*>(pool.v_cache);
  prm.meta = pool.meta;
  prm.block_v4 = pool.num_kv_heads * pool.block_size * kHeadDim * kv_bytes(pool.kv_dtype) / 16;
  prm.layer_stride_v4 = static_cast<int64_t>(pool.num_blocks) * prm.block_v4;
  prm.num_layers = pool.num_layers;
  prm.n = n;
  prm.nd = nd;
  std::memcpy(prm.p.v, src, sizeof(int32_t) * n);
  std::memcpy(prm.p.v + n, dst, sizeof(int32_t) * n);
  if (nd) {
    std::memcpy(prm.p.v + 2 * n, didx, sizeof(int32_t) * nd);
    std::memcpy(prm.p.v + 2 * n + nd, dval, sizeof(int32_t) * nd);
  }
  return launch_pdl(cow_copy_kernel<CAP>, dim3(n * pool.num_layers * 2), dim3(256), 0, stream, prm);
}

template <int KV, int ACT, int CAP>
cudaError_t do_append(const PoolView& pool, int layer, const int64_t* slots, int T,
                      const void* k_new, const void* v_new, const int32_t* didx,
                      const int32_t* dval, int nd, cudaStream_t stream) {
  AppendParams<CAP> prm;
  prm.k_new = static_cast<const uint8_t*>(k_new);
  prm.v_new = static_cast<const uint8_t*>(v_new);
  prm.k_cache = static_cast<uint8_t*>(pool.k_cache);
  prm.v_cache = static_cast<uint8_t*>(pool.v_cache);
  prm.k_inv = pool.k_inv;
  prm.v_inv = pool.v_inv;
  prm.meta = pool.meta;
  prm.layer_off = static_cast<int64_t>(layer) * pool.num_blocks * pool.num_kv_heads *
                  pool.block_size * kHeadDim;
  prm.H = pool.num_kv_heads;
  prm.B = pool.block_size;
  prm.T = T;
  prm.nd = nd;
  prm.layer = layer;
  for (int t = 0; t < T; ++t) prm.p.v[t] = static_cast<int32_t>(slots[t]);
  if (nd) {
    std::memcpy(prm.p.v + T, didx, sizeof(int32_t) * nd);
    std::memcpy(prm.p.v + T + nd, dval, sizeof(int32_t) * nd);
  }
  const int rows = T * pool.num_kv_heads * 2;
  const int warps = 8;
  const int blocks = std::max(1, (rows + warps - 1) / warps);
  return launch_pdl(append_kernel<KV, ACT, CAP>, dim3(blocks), dim3(warps * 32), 0, stream, prm);
}

template <int CAP>
cudaError_t dispatch_append(const PoolView& pool, int layer, const int64_t* slots, int T,
                            const void* k_new, const void* v_new, const int32_t* didx,
                            const int32_t* dval, int nd, cudaStream_t stream) {
  if (pool.kv_dtype == kFP8) {
    if (pool.act_dtype == kBF16)
      return do_append<kFP8, kBF16, CAP>(pool, layer, slots, T, k_new, v_new, didx, dval, nd, stream);
    return do_append<kFP8, kFP16, CAP>(pool, layer, slots, T, k_new, v_new, didx, dval, nd, stream);
  }
  return do_append<kBF16, kBF16, CAP>(pool, layer, slots, T, k_new, v_new, didx, dval, nd, stream);
}

}  // namespace

cudaError_t launch_meta_apply(const PoolView& pool, const int32_t* idx, const int32_t* val, int n,
                              cudaStream_t stream) {
  while (n > 0) {
    const int chunk = std::min(n, kPayloadLarge / 2);
    cudaError_t e = (2 * chunk <= kPayloadSmall)
                        ? do_meta_apply<kPayloadSmall>(pool, idx, val, chunk, stream)
                        : do_meta_apply<kPayloadLarge>(pool, idx, val, chunk, stream);
    if (e != cudaSuccess) return e;
    idx += chunk;
    val += chunk;
    n -= chunk;
  }
  return cudaSuccess;
}

cudaError_t launch_cow_copy(const PoolView& pool, const int32_t* src, const int32_t* dst, int n,
                            const int32_t* didx, const int32_t* dval, int nd,
                            cudaStream_t stream, int* launches) {
  // Deltas beyond what fits beside the copy list go in launches of their own first.
  const int room = kPayloadLarge - 2 * n;
  if (room < 0) return cudaErrorInvalidValue;  // caller splits copy lists
  if (2 * nd > room) {
    cudaError_t e = launch_meta_apply(pool, didx, dval, nd, stream);
    if (e != cudaSuccess) return e;
    *launches += (nd + kPayloadLarge / 2 - 1) / (kPayloadLarge / 2);
    nd = 0;
  }
  cudaError_t e = (2 * n + 2 * nd <= kPayloadSmall)
                      ? do_cow<kPayloadSmall>(pool, src, dst, n, didx, dval, nd, stream)
                      : do_cow<kPayloadLarge>(pool, src, dst, n, didx, dval, nd, stream);
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_append(const PoolView& pool, int layer, const int64_t* slots, int T,
                          const void* k_new, const void* v_new, const int32_t* didx,
                          const int32_t* dval, int nd, cudaStream_t stream, int* launches) {
  if (T + 2 * nd > kPayloadLarge) {
    cudaError_t e = launch_meta_apply(pool, didx, dval, nd, stream);
    if (e != cudaSuccess) return e;
    *launches += (nd + kPayloadLarge / 2 - 1) / (kPayloadLarge / 2);
    nd = 0;
  }
  const size_t row_bytes = static_cast<size_t>(pool.num_kv_heads) * kHeadDim * 2;
  const uint8_t* k = static_cast<const uint8_t*>(k_new);
  const uint8_t* v = static_cast<const uint8_t*>(v_new);
  while (T > 0) {
    const int chunk = std::min(T, kPayloadLarge - 2 * nd);
    cudaError_t e = (chunk + 2 * nd <= kPayloadSmall)
                        ? dispatch_append<kPayloadSmall>(pool, layer, slots, chunk, k, v, didx, dval, nd, stream)
                        : dispatch_append<kPayloadLarge>(pool, layer, slots, chunk, k, v, didx, dval, nd, stream);
    if (e != cudaSuccess) return e;
    ++*launches;
    nd = 0;
    slots += chunk;
    k += row_bytes * chunk;
    v += row_bytes * chunk;
    T -= chunk;
  }
  return cudaSuccess;
}

}  // namespace pa
