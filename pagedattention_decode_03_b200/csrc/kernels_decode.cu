// Paged single-query decode attention for sm_100a.
//
// Computes, for every (sequence, query head),
//     out = sum_t softmax_t(scale * q . k_t) v_t      over t < len(seq),
// reading k_t, v_t from slot t % B of physical block table[seq][t / B] of the
// query head's KV head -- attention taken directly over the non-contiguous
// blocks, addressed through the block table (kv-cache-pagedattention-serving,
// PagedAttention: virtual memory for GPUs; "Managing the KV Cache", Block
// Tables and Sharing: the kernel gathers K/V through the block table).
//
// Design (B200-first; the pages give no kernel design):
//   * Work unit = (sequence, KV head); the G = H_q / H_kv query heads of the
//     group are processed together, so every K/V byte is read once.
//   * Each warp is an independent worker with its own ring of shared-memory
//     stages.  One (layer, block, head) K tile and its V tile are one stage,
//     fetched by TMA tensor loads (cp.async.bulk.tensor, 128-byte swizzle)
//     that complete on a per-stage mbarrier; the warp keeps STAGES tiles in
//     flight while it computes on the oldest.  Block ids come from the device
//     mirror of the block tables, cached 32 at a time in registers.
//   * G >= 4: QK^T and P.V are warp-level tensor-core MMAs (m16n8k16) with the
//     16 tokens of a block on M and the (padded) query group on N; S^T stays in
//     registers, the online softmax runs on the accumulator fragments, and P^T
//     reaches the PV MMA through movmatrix.  G <= 2: fp32 FMAs on CUDA cores.
//   * Work is spread over all warps of the GPU in equal shares of a work axis
//     that lists each unit's KV blocks after a few "cost positions" standing
//     for the unit's fixed segment cost (stream-K style): a worker's share can
//     start and end inside a sequence; partial results (running max m, sum l,
//     unnormalised o) of a cut sequence are merged by log-sum-exp inside the
//     kernel, by the last of its workers to finish.  Fixed-size partitions
//     (merged by a separate reduction kernel) and "never split" are the two
//     other modes.
//   * Forks of one prompt share its blocks by reference count ("Managing the
//     KV Cache", Block Tables and Sharing); a sibling set is one unit whose
//     common blocks are read once for all members' query rows, followed by
//     each member's own blocks with the other members' rows masked.
//   * The step's append may ride along: the worker that reads a sequence's
//     last block writes the new K/V row into the cache and into its staged
//     tile before computing on it.
//   * FP8 E4M3 KV: tiles are half the bytes; codes are converted to f16 with
//     the hardware cvt (exact), K's scale is folded into the logit scale and
//     V's into the output.
//   * Launched with programmatic stream serialization: the parameter-only
//     prologue overlaps the previous kernel, which is waited for before any
//     memory access.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <type_traits>

#include "device_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kWarps = 4;              // warps (independent workers) per CTA

#include "decode_common.cuh"

template <int KV>
struct Tile {
  static constexpr int kBytes = KV == kFP8 ? kBlock * kHeadDim : kBlock * kHeadDim * 2;  // one K or V tile
  static constexpr int kStageBytes = 2 * kBytes;
  static constexpr int kStages = KV == kFP8 ? 6 : 3;
  static constexpr int kRingBytes = kStages * kStageBytes;
};


// ------------------------------------------------------------------ producer
template <int KV>
struct Producer {
  Cursor cur;
  Seg seg;
  int32_t b;          // next block of seg to fetch
  int32_t tc_val, tc_base, tc_unit;
  Members mem;        // members of seg's unit, for the table refreshes
  uint32_t issued;
  int32_t* phys_s;    // shared memory: first cache row (token slot) of each staged tile

  // Starts from a copy of the consumer's cursor (same segments, same order).
  template <class Prm>
  __device__ __forceinline__ void init(const Prm& prm, const Cursor& c) {
    cur = c;
    seg = cur.next(prm);
    b = seg.b0;
    mem = load_members(prm, seg, threadIdx.x & 31);
    tc_unit = -1;
    tc_base = 0;
    tc_val = 0;
    issued = 0;
  }

  // Before the dependency wait: prefetch the first n tiles of the first
  // segment into L2, while the previous kernel's tail leaves HBM mostly idle.
  // The table entries may be stale here (a kernel still running may rewrite
  // them): a stale id only wastes a prefetch, since the copies after the wait
  // read the tables again and L2 holds the current data; ids are clamped into
  // the pool, so every address lies inside the cache.
  template <class Prm>
  __device__ __forceinline__ void prefetch_l2(const Prm& prm, int n, int lane) {
    if (!seg.valid) return;  // warp-uniform
    const int nb = min(n, seg.b1 - seg.b0);
    if (nb <= 0) return;     // warp-uniform
    // locate_in is collective (shuffles over a unit's members): all lanes
    const BlockRef r = locate_in<1>(prm, mem, seg, seg.b0 + min(lane, nb - 1));
    if (lane >= nb) return;
    const int32_t e = r.b >> prm.bshift;
    int32_t phys = r.b >= 0 && e < prm.mbps ? prm.tables[static_cast<int64_t>(r.seq) * prm.mbps + e] : 0;
    if (static_cast<uint32_t>(phys) >= static_cast<uint32_t>(prm.num_blocks)) phys = 0;
    const int64_t row =
        ((static_cast<int64_t>(prm.layer) * prm.num_blocks + phys) * prm.num_kv_heads + seg.h) *
            (kBlock << prm.bshift) +
        (r.b & ((1 << prm.bshift) - 1)) * kBlock;
    const int64_t off = row * kHeadDim * (KV == kFP8 ? 1 : 2);
    dev::bulk_prefetch_l2(prm.k_cache + off, Tile<KV>::kBytes);
    dev::bulk_prefetch_l2(prm.v_cache + off, Tile<KV>::kBytes);
  }

  // Fetch the next block of this worker into stage issued % kStages.
  template <class Prm>
  __device__ __forceinline__ void issue(const Prm& prm, const CUtensorMap* tmk,
                                        const CUtensorMap* tmv, uint32_t ring, uint32_t bars,
                                        int w, int lane) {
    if (!seg.valid) return;
    if (b == seg.b1) {
      seg = cur.next(prm);
      if (!seg.valid) {
        // every copy of this worker is out: let the next kernel in the stream
        // start placing its blocks.  (Signalled at kernel start instead, the
        // queued successor's launch slowed this kernel's first copies from
        // ~1.6 to ~4.5 us in traces of back-to-back layers.)
        dev::grid_dep_launch();
        return;
      }
      b = seg.b0;
      mem = load_members(prm, seg, lane);
    }
    // physical ids of the unit's tiles b .. b+31, one per lane (a sibling
    // set's positions run through several table rows); the low bit of a
    // 32-token block's tile index picks its half
    if (seg.k != tc_unit || b < tc_base || b >= tc_base + 32) {
      tc_unit = seg.k;
      tc_base = b;
      const BlockRef r = locate_in<1>(prm, mem, seg, b + lane);
      const int32_t e = r.b >> prm.bshift;
      tc_val = r.b >= 0 && e < prm.mbps ? prm.tables[static_cast<int64_t>(r.seq) * prm.mbps + e] : 0;
      // physical id in the upper bits, half in bit 0 (ids < 2^30)
      tc_val = static_cast<int32_t>((static_cast<uint32_t>(tc_val) << 1) |
                                    static_cast<uint32_t>(r.b & ((1 << prm.bshift) - 1)));
    }
    const int32_t tv = __shfl_sync(0xffffffffu, tc_val, b - tc_base);
    int32_t phys = static_cast<int32_t>(static_cast<uint32_t>(tv) >> 1);
    if (static_cast<uint32_t>(phys) >= static_cast<uint32_t>(prm.num_blocks)) {
      if (lane == 0) atomicOr(prm.err, kErrBadBlock);
      phys = 0;
    }
    const uint32_t stage = issued % Tile<KV>::kStages;
    const uint32_t bar = bars + stage * 8;
    const uint32_t dst = ring + stage * Tile<KV>::kStageBytes;
    const int32_t row =
        (((prm.layer * prm.num_blocks + phys) * prm.num_kv_heads + seg.h) << (4 + prm.bshift)) +
        (tv & 1) * kBlock;
    if (lane == 0) phys_s[stage] = row;
    if (lane == 0) {
      dev::mbar_arrive_expect_tx(bar, Tile<KV>::kStageBytes);
      if constexpr (KV == kFP8) {
        dev::tma_load_2d(dst, tmk, 0, row, bar);
        dev::tma_load_2d(dst + Tile<KV>::kBytes, tmv, 0, row, bar);
      } else {  // 3-D boxes: both d-halves of the 16 rows in one copy
        dev::tma_load_3d(dst, tmk, 0, row, 0, bar);
        dev::tma_load_3d(dst + Tile<KV>::kBytes, tmv, 0, row, 0, bar);
      }
    }
    ++issued;
    ++b;
  }
};

// Zero V rows [nvalid, 16) of a staged tile so masked tokens contribute exact
// zeros whatever stale bits the slots hold.
template <int KV>
__device__ __forceinline__ void zero_tail_rows(uint8_t* vtile, int nvalid, int lane) {
  constexpr int kRowChunks = KV == kFP8 ? 8 : 16;  // 16-byte chunks per token row
  const int n = (kBlock - nvalid) * kRowChunks;
  for (int c = lane; c < n; c += 32) {
    const int t = nvalid + c / kRowChunks;
    const int k = c % kRowChunks;
    uint8_t* p;
    if constexpr (KV == kFP8) {
      p = vtile + t * 128 + k * 16;
    } else {
      p = vtile + (k >> 3) * 2048 + t * 128 + (k & 7) * 16;
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(0, 0, 0, 0);
  }
  dev::fence_proxy_async_smem();
  __syncwarp();
}

// Query row `g` (MMA column) of a segment, or null past the unit's rows.
template <int G, class Prm>
__device__ __forceinline__ const uint16_t* q_row(const Prm& prm, const Seg& s, int g, int rows) {
  if (g >= rows) return nullptr;
  return reinterpret_cast<const uint16_t*>(prm.q) + row_offset<G>(prm, s, g);
}

// ============================================================ tensor-core path
// Up to 8 query rows on the MMA N dimension: a query group of G in {4, 8}
// heads, or the side-by-side groups of a shared prefix's sibling set.
template <int KV, int ACT, int G>
struct MmaPath {
  static constexpr bool kF16 = (KV == kFP16) || (KV == kFP8);
  uint32_t qf[8][2];   // Q^T B-fragments for the 8 k-steps
  float o[8][4];       // O^T accumulators: 8 m-tiles (d) x (2 heads per lane)
  float m0, m1, l0, l1;
  float sl2;           // logit scale in log2 units
  float vmul;          // V dequantisation scale (1 for 16-bit KV)
  int rows;            // query rows of the segment (<= 8)

  template <class Prm>
  __device__ __forceinline__ void begin(const Prm& prm, const Seg& s, int lane) {
    const int g = lane >> 2, tig = lane & 3;
    rows = unit_rows<G>(prm, s);
    const uint16_t* qrow = q_row<G>(prm, s, g, rows);
    float qscale = 1.f;
    sl2 = prm.scale * kLog2e;
    vmul = 1.f;
    if constexpr (KV == kFP8) {
      // Q is pre-multiplied by the softmax scale before rounding to f16; K's
      // dequantisation scale is folded into the logit scale.
      qscale = prm.scale;
      sl2 = prm.k_scale[prm.layer * prm.num_kv_heads + s.h] * kLog2e;
      vmul = prm.v_scale[prm.layer * prm.num_kv_heads + s.h];
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      if (qrow != nullptr) {
        if constexpr (KV == kFP8) {
          const uint2 raw = *reinterpret_cast<const uint2*>(qrow + 16 * ks + 4 * tig);
          const float a = act_to_f32<ACT>(raw.x & 0xffff) * qscale;
          const float b = act_to_f32<ACT>(raw.x >> 16) * qscale;
          const float c = act_to_f32<ACT>(raw.y & 0xffff) * qscale;
          const float d = act_to_f32<ACT>(raw.y >> 16) * qscale;
          qf[ks][0] = dev::pack_f16(a, b);
          qf[ks][1] = dev::pack_f16(c, d);
        } else {
          qf[ks][0] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tig);
          qf[ks][1] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * tig);
        }
      } else {
        qf[ks][0] = 0u;
        qf[ks][1] = 0u;
      }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  }

  __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (kF16) dev::mma_f16(d, a, b0, b1);
    else dev::mma_bf16(d, a, b0, b1);
  }

  __device__ __forceinline__ void block(uint32_t ks_addr, uint32_t vs_addr, int nvalid, uint32_t cols,
                                       int lane) {
    const int g = lane >> 2, tig = lane & 3;
    const int r8 = lane & 7, j = lane >> 3;
    // ---- S^T = K Q^T : 16 tokens x 8 heads
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int tok = r8 + ((j & 1) << 3);
      const int add = j >> 1;
      if constexpr (KV == kFP8) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t R[4];
          dev::ldsm_x4(ks_addr + tok * 128 + (((2 * kk + add) ^ r8) << 4), R);
          uint32_t a0[4] = {dev::e4m3x2_to_f16x2(R[0] & 0xffff), dev::e4m3x2_to_f16x2(R[1] & 0xffff),
                            dev::e4m3x2_to_f16x2(R[0] >> 16), dev::e4m3x2_to_f16x2(R[1] >> 16)};
          uint32_t a1[4] = {dev::e4m3x2_to_f16x2(R[2] & 0xffff), dev::e4m3x2_to_f16x2(R[3] & 0xffff),
                            dev::e4m3x2_to_f16x2(R[2] >> 16), dev::e4m3x2_to_f16x2(R[3] >> 16)};
          mma(sa, a0, qf[2 * kk][0], qf[2 * kk][1]);
          mma(sb, a1, qf[2 * kk + 1][0], qf[2 * kk + 1][1]);
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int chunk = 2 * ks + add;
          uint32_t a[4];
          dev::ldsm_x4(ks_addr + (ks >> 2) * 2048 + tok * 128 + (((chunk & 7) ^ r8) << 4), a);
          if (ks & 1) mma(sb, a, qf[ks][0], qf[ks][1]);
          else mma(sa, a, qf[ks][0], qf[ks][1]);
        }
      }
    }
    float s0 = (sa[0] + sb[0]) * sl2, s1 = (sa[1] + sb[1]) * sl2;  // token g, heads 2tig, 2tig+1
    float s2 = (sa[2] + sb[2]) * sl2, s3 = (sa[3] + sb[3]) * sl2;  // token g+8
    if (nvalid < kBlock) {
      if (g >= nvalid) s0 = s1 = -INFINITY;
      if (g + 8 >= nvalid) s2 = s3 = -INFINITY;
    }
    if (cols != 0xffu) {  // a sibling's own block: the other members' rows sit it out
      if (!(cols >> (2 * tig) & 1u)) s0 = s2 = -INFINITY;
      if (!(cols >> (2 * tig + 1) & 1u)) s1 = s3 = -INFINITY;
    }
    // ---- online softmax over the 16 tokens (rows) per head (column); a
    // column that no token has reached yet keeps m = -inf and uses 0 as the
    // reference, so its weights stay exact zeros
    const float mx0 = warp_max_rows(fmaxf(s0, s2));
    const float mx1 = warp_max_rows(fmaxf(s1, s3));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float r0 = mn0 == -INFINITY ? 0.f : mn0, r1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = dev::exp2_approx(m0 - r0), c1 = dev::exp2_approx(m1 - r1);
    m0 = mn0;
    m1 = mn1;
    const float p0 = dev::exp2_approx(s0 - r0), p1 = dev::exp2_approx(s1 - r1);
    const float p2 = dev::exp2_approx(s2 - r0), p3 = dev::exp2_approx(s3 - r1);
    l0 = l0 * c0 + p0 + p2;
    l1 = l1 * c1 + p1 + p3;
    if (__any_sync(0xffffffffu, c0 != 1.f || c1 != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= c0;
        o[mt][1] *= c1;
        o[mt][2] *= c0;
        o[mt][3] *= c1;
      }
    }
    // ---- P^T as the B operand of O^T += V^T P^T.  f16 keeps 11 significant
    // bits of P; bf16 keeps 8, so with bf16 V the weights go in as two parts,
    // P = hi + lo (each bf16), and the product is taken twice: P's rounding
    // error drops from 2^-9 to 2^-17 relative, below the fp32 accumulation.
    const uint32_t x0 = kF16 ? dev::pack_f16(p0, p1) : dev::pack_bf16(p0, p1);
    const uint32_t x1 = kF16 ? dev::pack_f16(p2, p3) : dev::pack_bf16(p2, p3);
    const uint32_t pb0 = dev::movm_t(x0);
    const uint32_t pb1 = dev::movm_t(x1);
    uint32_t pl0 = 0, pl1 = 0;
    if constexpr (!kF16) {
      pl0 = dev::movm_t(dev::pack_bf16(p0 - dev::bf16lo_to_f32(x0), p1 - dev::bf16hi_to_f32(x0)));
      pl1 = dev::movm_t(dev::pack_bf16(p2 - dev::bf16lo_to_f32(x1), p3 - dev::bf16hi_to_f32(x1)));
    }
    if constexpr (KV == kFP8) {
      const int tok = r8 + ((j & 1) << 3);
      const int add = j >> 1;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t R[4];
        dev::ldsm_x4_t(vs_addr + tok * 128 + (((2 * cc + add) ^ r8) << 4), R);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t X0 = dev::prmt(R[2 * half], 0, 0x3120);
          const uint32_t X1 = dev::prmt(R[2 * half + 1], 0, 0x3120);
          uint32_t a[4] = {dev::e4m3x2_to_f16x2(X0 & 0xffff), dev::e4m3x2_to_f16x2(X0 >> 16),
                           dev::e4m3x2_to_f16x2(X1 & 0xffff), dev::e4m3x2_to_f16x2(X1 >> 16)};
          mma(o[2 * cc + half], a, pb0, pb1);
        }
      }
    } else {
      const int tok = r8 + ((j >> 1) << 3);
      const int add = j & 1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int chunk = 2 * mt + add;
        uint32_t a[4];
        dev::ldsm_x4_t(vs_addr + (mt >> 2) * 2048 + tok * 128 + (((chunk & 7) ^ r8) << 4), a);
        mma(o[mt], a, pb0, pb1);
        if constexpr (!kF16) mma(o[mt], a, pl0, pl1);
      }
    }
  }

  // d index of accumulator o[mt][k] (k = 0,1: first row; 2,3: second row).
  __device__ __forceinline__ static int d_of(int mt, int second, int g) {
    if constexpr (KV == kFP8) return 16 * mt + 2 * g + second;
    else return 16 * mt + 8 * second + g;
  }

  template <class Prm>
  __device__ __forceinline__ void finish(const Prm& prm, const Seg& s, int lane, const MergeStage& stage) {
    const int g = lane >> 2, tig = lane & 3;
    const float lt0 = warp_sum_rows(l0), lt1 = warp_sum_rows(l1);
    const int h0 = 2 * tig, h1 = 2 * tig + 1;
    if (s.dest < 0) {
      uint16_t* out = reinterpret_cast<uint16_t*>(prm.out);
      uint16_t* orow0 = h0 < rows ? out + row_offset<G>(prm, s, h0) : nullptr;
      uint16_t* orow1 = h1 < rows ? out + row_offset<G>(prm, s, h1) : nullptr;
      const float f0 = vmul / lt0, f1 = vmul / lt1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int sec = 0; sec < 2; ++sec) {
          const int d = d_of(mt, sec, g);
          if (orow0) orow0[d] = f32_to_act<ACT>(o[mt][2 * sec] * f0);
          if (orow1) orow1[d] = f32_to_act<ACT>(o[mt][2 * sec + 1] * f1);
        }
      }
    } else {
      float* slot = prm.partials + static_cast<int64_t>(s.dest) * kPartialSlotFloats;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int sec = 0; sec < 2; ++sec) {
          const int d = d_of(mt, sec, g);
          if (h0 < rows) slot[h0 * kHeadDim + d] = o[mt][2 * sec] * vmul;
          if (h1 < rows) slot[h1 * kHeadDim + d] = o[mt][2 * sec + 1] * vmul;
        }
      }
      if (g == 0) {
        float* ml = slot + kMaxGroup * kHeadDim;
        if (h0 < rows) { ml[2 * h0] = m0; ml[2 * h0 + 1] = lt0; }
        if (h1 < rows) { ml[2 * h1] = m1; ml[2 * h1 + 1] = lt1; }
      }
      if constexpr (kSibParams<Prm>) {
        if (s.shared) {
          settle_partial<ACT, G, kMaxGroup>(prm, s, rows, lane, stage);
          return;
        }
      }
      settle_partial<ACT, G, G>(prm, s, G, lane, stage);
    }
  }
};

// =============================================================== CUDA-core path
// G in {1, 2}: lane = (token row r = lane / 4, d-quarter qd = lane % 4); a
// block is processed as two halves (tokens r and r + 8).
template <int KV, int ACT, int G>
struct FmaPath {
  // 16-bit KV: each lane covers 32 d as 4 chunks of 8; FP8: 2 chunks of 16.
  static constexpr int kChunks = KV == kFP8 ? 2 : 4;
  static constexpr int kPer = KV == kFP8 ? 16 : 8;
  float qv[G][kChunks][kPer];
  float acc[G][kChunks][kPer];
  float m[G], l[G];
  float sl2, vmul;

  // chunk position (16-byte unit within the 128-byte row of its box) and box
  __device__ __forceinline__ static int cib(int qd, int i) {
    if constexpr (KV == kFP8) return 2 * qd + i;
    else return 4 * (qd & 1) + ((i + 2 * (qd >> 1)) & 3);
  }
  __device__ __forceinline__ static int d0_of(int qd, int i) {
    if constexpr (KV == kFP8) return 16 * (2 * qd + i);
    else return 64 * (qd >> 1) + 8 * cib(qd, i);
  }
  __device__ __forceinline__ static uint32_t row_addr(uint32_t base, int t, int qd, int i) {
    if constexpr (KV == kFP8) return base + t * 128 + ((cib(qd, i) ^ (t & 7)) << 4);
    else return base + (qd >> 1) * 2048 + t * 128 + ((cib(qd, i) ^ (t & 7)) << 4);
  }

  __device__ __forceinline__ void to_f32(const uint4& raw, float (&f)[kPer]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    if constexpr (KV == kFP8) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t lo = dev::e4m3x2_to_f16x2(w[k] & 0xffff);
        const uint32_t hi = dev::e4m3x2_to_f16x2(w[k] >> 16);
        f[4 * k + 0] = dev::f16lo_to_f32(lo);
        f[4 * k + 1] = dev::f16hi_to_f32(lo);
        f[4 * k + 2] = dev::f16lo_to_f32(hi);
        f[4 * k + 3] = dev::f16hi_to_f32(hi);
      }
    } else if constexpr (KV == kBF16) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[2 * k] = dev::bf16lo_to_f32(w[k]);
        f[2 * k + 1] = dev::bf16hi_to_f32(w[k]);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[2 * k] = dev::f16lo_to_f32(w[k]);
        f[2 * k + 1] = dev::f16hi_to_f32(w[k]);
      }
    }
  }

  template <class Prm>
  __device__ __forceinline__ void begin(const Prm& prm, const Seg& s, int lane) {
    const int qd = lane & 3;
    sl2 = prm.scale * kLog2e;
    vmul = 1.f;
    if constexpr (KV == kFP8) {
      sl2 *= prm.k_scale[prm.layer * prm.num_kv_heads + s.h];
      vmul = prm.v_scale[prm.layer * prm.num_kv_heads + s.h];
    }
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const uint16_t* qrow = reinterpret_cast<const uint16_t*>(prm.q) + s.i * prm.q_item_stride +
                             (s.h * G + gg) * kHeadDim;
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const uint16_t* src = qrow + d0_of(qd, i);
#pragma unroll
        for (int e = 0; e < kPer; ++e) qv[gg][i][e] = act_to_f32<ACT>(src[e]);
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[gg][i][e] = 0.f;
      }
      m[gg] = -INFINITY;
      l[gg] = 0.f;
    }
  }

  __device__ __forceinline__ void block(uint32_t ks_addr, uint32_t vs_addr, int nvalid,
                                       uint32_t /*cols: every row takes part in a plain unit*/,
                                       int lane) {
    const int r = lane >> 2, qd = lane & 3;
    float s[2][G];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int t = r + 8 * half;
#pragma unroll
      for (int gg = 0; gg < G; ++gg) s[half][gg] = 0.f;
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        uint4 raw;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(raw.x), "=r"(raw.y), "=r"(raw.z), "=r"(raw.w)
                     : "r"(row_addr(ks_addr, t, qd, i)));
        float kf[kPer];
        to_f32(raw, kf);
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
#pragma unroll
          for (int e = 0; e < kPer; ++e) s[half][gg] = fmaf(qv[gg][i][e], kf[e], s[half][gg]);
      }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half)
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        float x = s[half][gg];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x *= sl2;
        if (r + 8 * half >= nvalid) x = -INFINITY;
        s[half][gg] = x;
      }
    float p[2][G];
    bool rescale = false;
    float corr[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const float mx = warp_max_rows(fmaxf(s[0][gg], s[1][gg]));
      const float mn = fmaxf(m[gg], mx);
      corr[gg] = dev::exp2_approx(m[gg] - mn);
      m[gg] = mn;
      p[0][gg] = dev::exp2_approx(s[0][gg] - mn);
      p[1][gg] = dev::exp2_approx(s[1][gg] - mn);
      l[gg] = l[gg] * corr[gg] + p[0][gg] + p[1][gg];
      rescale |= corr[gg] != 1.f;
    }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
      for (int gg = 0; gg < G; ++gg)
#pragma unroll
        for (int i = 0; i < kChunks; ++i)
#pragma unroll
          for (int e = 0; e < kPer; ++e) acc[gg][i][e] *= corr[gg];
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int t = r + 8 * half;
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        uint4 raw;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(raw.x), "=r"(raw.y), "=r"(raw.z), "=r"(raw.w)
                     : "r"(row_addr(vs_addr, t, qd, i)));
        float vf[kPer];
        to_f32(raw, vf);
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
#pragma unroll
          for (int e = 0; e < kPer; ++e) acc[gg][i][e] = fmaf(p[half][gg], vf[e], acc[gg][i][e]);
      }
    }
  }

  template <class Prm>
  __device__ __forceinline__ void finish(const Prm& prm, const Seg& s, int lane, const MergeStage& stage) {
    const int r = lane >> 2, qd = lane & 3;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      l[gg] = warp_sum_rows(l[gg]);
#pragma unroll
      for (int i = 0; i < kChunks; ++i)
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[gg][i][e] = warp_sum_rows(acc[gg][i][e]);
    }
    // lanes with r < kChunks write chunk i = r of their d-quarter
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        if (r != i) continue;
        const int d0 = d0_of(qd, i);
        if (s.dest < 0) {
          uint16_t* orow = reinterpret_cast<uint16_t*>(prm.out) + s.i * prm.q_item_stride +
                           (s.h * G + gg) * kHeadDim + d0;
          const float f = vmul / l[gg];
#pragma unroll
          for (int e = 0; e < kPer; e += 2) {
            const uint32_t two = static_cast<uint32_t>(f32_to_act<ACT>(acc[gg][i][e] * f)) |
                                 (static_cast<uint32_t>(f32_to_act<ACT>(acc[gg][i][e + 1] * f)) << 16);
            *reinterpret_cast<uint32_t*>(orow + e) = two;
          }
        } else {
          float* slot = prm.partials + static_cast<int64_t>(s.dest) * kPartialSlotFloats +
                        gg * kHeadDim + d0;
#pragma unroll
          for (int e = 0; e < kPer; e += 4)
            *reinterpret_cast<float4*>(slot + e) =
                make_float4(acc[gg][i][e] * vmul, acc[gg][i][e + 1] * vmul,
                            acc[gg][i][e + 2] * vmul, acc[gg][i][e + 3] * vmul);
        }
      }
    }
    if (s.dest >= 0) {
      if (lane == 0) {
        float* ml = prm.partials + static_cast<int64_t>(s.dest) * kPartialSlotFloats +
                    kMaxGroup * kHeadDim;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          ml[2 * gg] = m[gg];
          ml[2 * gg + 1] = l[gg];
        }
      }
      settle_partial<ACT, G, G>(prm, s, G, lane, stage);
    }
  }
};

template <int KV, int ACT, int G>
using PathFor = typename std::conditional<(G >= 4), MmaPath<KV, ACT, G>, FmaPath<KV, ACT, G>>::type;

// ===================================================================== kernel
// Fused append: the K/V rows of `item`'s last token (position len-1) for KV
// head h.  Lane l < 16 carries elements 8l .. 8l+7 of the K row, lane 16 + l
// those of the V row (act dtype, 16 bytes).
// Write those rows into their cache slot (tile_row + (len-1) % 16) and into row
// (len-1) % 16 of the staged K and V tiles (the copy brought the block in
// before the row was written).  Same values as the append kernel: 16-bit rows
// are copied; FP8 codes are E4M3(rn, satfinite)(fp32(x) * inv_scale).
template <int KV, int ACT, class Prm>
__device__ __forceinline__ void append_last_token(const Prm& prm, int h, int len, int32_t tile_row,
                                                  uint8_t* st, uint4 val, int lane) {
  using T = Tile<KV>;
  const int r = (len - 1) % kBlock;
  const int kv = lane >> 4, c = lane & 15;
  uint8_t* tile = st + kv * T::kBytes;
  uint8_t* cache = kv ? prm.v_cache : prm.k_cache;
  // tile_row = cache row of the staged tile's first token slot
  const int64_t dst_el = (static_cast<int64_t>(tile_row) + r) * kHeadDim;
  if constexpr (KV == kFP8) {
    const float inv = (kv ? prm.v_inv : prm.k_inv)[prm.layer * prm.num_kv_heads + h];
    const uint32_t w[4] = {val.x, val.y, val.z, val.w};
    uint32_t code[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float x0 = act_to_f32<ACT>(w[2 * k] & 0xffff), x1 = act_to_f32<ACT>(w[2 * k] >> 16);
      const float x2 = act_to_f32<ACT>(w[2 * k + 1] & 0xffff), x3 = act_to_f32<ACT>(w[2 * k + 1] >> 16);
      code[k] = static_cast<uint32_t>(dev::f32x2_to_e4m3x2(__fmul_rn(x0, inv), __fmul_rn(x1, inv))) |
                (static_cast<uint32_t>(dev::f32x2_to_e4m3x2(__fmul_rn(x2, inv), __fmul_rn(x3, inv))) << 16);
    }
    const uint2 codes = make_uint2(code[0], code[1]);  // elements 8c .. 8c+7, one byte each
    *reinterpret_cast<uint2*>(tile + r * 128 + (((c >> 1) ^ (r & 7)) << 4) + (c & 1) * 8) = codes;
    dev::fence_proxy_async_smem();  // the stage's next copy overwrites these bytes
    *reinterpret_cast<uint2*>(cache + dst_el + c * 8) = codes;
  } else {
    *reinterpret_cast<uint4*>(tile + (c >> 3) * 2048 + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = val;
    dev::fence_proxy_async_smem();  // the stage's next copy overwrites these bytes
    *reinterpret_cast<uint4*>(cache + (dst_el + c * 8) * 2) = val;
  }
  __syncwarp();  // the staged row is complete before any lane reads the tile
}

// One segment: wait for each staged block in turn, compute on it, and refill
// the freed stage with the worker's next block.  False if a wait gave up.
template <int KV, int ACT, int G, class Path, class Prm>
__device__ __forceinline__ bool consume_segment(Path& path, const Prm& prm, const Seg& s,
                                                Producer<KV>& prod, const CUtensorMap* tmk,
                                                const CUtensorMap* tmv, uint8_t* ring_ptr,
                                                uint32_t ring, uint32_t bars, uint32_t& consumed,
                                                int w, int lane, uint32_t merge_bar, uint32_t& merge_phase) {
  using T = Tile<KV>;
  path.begin(prm, s, lane);
  const Members mem = load_members(prm, s, lane);
#pragma unroll 1
  for (int b = s.b0; b < s.b1; ++b) {
    const uint32_t stage = consumed % T::kStages;
    const uint32_t parity = (consumed / T::kStages) & 1u;
    if (!dev::mbar_wait_bounded(bars + stage * 8, parity, kWaitLimit)) {
      if (lane == 0) atomicOr(prm.err, kErrTimeout);
      return false;
    }
    const BlockRef br = locate_in<G>(prm, mem, s, b);
    const int nvalid = max(0, min(kBlock, br.len - br.b * kBlock));
    uint8_t* st = ring_ptr + stage * T::kStageBytes;
    if (nvalid < kBlock) zero_tail_rows<KV>(st + T::kBytes, nvalid, lane);
    if constexpr (!kSibParams<Prm>) {  // sibling plans never carry a fused append
      if (prm.k_new != nullptr && is_last_block(br))
        append_last_token<KV, ACT>(prm, s.h, br.len, prod.phys_s[stage], st,
                                   __ldcg(new_row_ptr(prm, s.h, br.item, lane)), lane);
    }
    path.block(ring + stage * T::kStageBytes, ring + stage * T::kStageBytes + T::kBytes, nvalid,
               br.cols, lane);
    __syncwarp();
    ++consumed;
    prod.issue(prm, tmk, tmv, ring, bars, w, lane);
  }
  // With no copy of its own in flight (its last segment), the worker's ring
  // can stage the partial slots of a merge.
  MergeStage stage{nullptr, 0, 0, 0, nullptr};
  if (prod.issued == consumed) stage = MergeStage{ring_ptr, ring, T::kRingBytes / static_cast<int>(kSlotBytes),
                                                  merge_bar, &merge_phase};
  path.finish(prm, s, lane, stage);
  return true;
}

template <int KV, int ACT, int G, class PlanT>
__global__ void __launch_bounds__(kWarps * 32)
    decode_kernel(const __grid_constant__ DecodeKParams<PlanT> prm,
                  const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * kWarps + warp;
  const int W = prm.plan.workers;
  if (w >= W) return;

  using T = Tile<KV>;
  uint8_t* ring_ptr = smem + warp * T::kRingBytes;
  const uint32_t ring = dev::smem_u32(ring_ptr);
  const uint32_t bars = dev::smem_u32(smem + kWarps * T::kRingBytes) + warp * T::kStages * 8;
  int32_t* phys_s = reinterpret_cast<int32_t*>(smem + kWarps * T::kRingBytes + kWarps * T::kStages * 8) +
                    warp * T::kStages;
  const uint32_t merge_bar =
      dev::smem_u32(smem + kWarps * T::kRingBytes + kWarps * T::kStages * 12) + warp * 8;
  uint32_t merge_phase = 0;
  if (lane == 0) {
    dev::tma_prefetch_desc(&tmk);
    dev::tma_prefetch_desc(&tmv);
    for (int s = 0; s < T::kStages; ++s) dev::mbar_init(bars + s * 8, 1);
    dev::mbar_init(merge_bar, 1);
    dev::fence_mbar_init();
  }
  __syncwarp();

  const int64_t g0 = worker_start(prm.total, w, W);
  const int64_t g1 = worker_start(prm.total, w + 1, W);
  Producer<KV> prod;
  prod.phys_s = phys_s;
  Cursor cur;
  cur.init(prm, g0, g1, w);  // kernel parameters only: may overlap the previous kernel
  prod.init(prm, cur);
  // Twice the ring's depth of 16-bit tiles (measured best on the 80-layer
  // GQA layers: 33.1 us per layer against 34.9 without, worse at 16 tiles).
  // Not for FP8 pools, whose deeper ring covers as many tiles, nor for
  // sibling plans, whose prologue overlaps the append launch (both measured
  // slightly slower with it).
  if constexpr (!kIsSib<PlanT> && KV != kFP8) prod.prefetch_l2(prm, 2 * T::kStages, lane);
  dev::grid_dep_wait();
#pragma unroll 1
  for (int k = 0; k < T::kStages; ++k) prod.issue(prm, &tmk, &tmv, ring, bars, w, lane);

  // Sibling plans put every unit on the tensor cores: a set's rows fill the
  // tile, and one path keeps the kernel within the register budget.
  typename std::conditional<kIsSib<PlanT>, MmaPath<KV, ACT, G>, PathFor<KV, ACT, G>>::type path;
  uint32_t consumed = 0;
  bool failed = false;
#pragma unroll 1
  while (true) {
    const Seg s = cur.next(prm);
    if (!s.valid) break;
    const bool ok =
        consume_segment<KV, ACT, G>(path, prm, s, prod, &tmk, &tmv, ring_ptr, ring, bars, consumed, w, lane,
                                    merge_bar, merge_phase);
    if (!ok) {
      failed = true;
      break;
    }
  }
  if (failed) {
    // Let copies already in flight land before the CTA's shared memory goes away.
    for (uint32_t c = consumed; c < prod.issued; ++c)
      dev::mbar_wait_bounded(bars + (c % T::kStages) * 8, (c / T::kStages) & 1u, kWaitLimit);
  }
}

// ===================================================================== reduce
struct ReduceKParams {
  uint8_t* out;
  const float* partials;
  int64_t q_item_stride;
  int32_t group;
  int64_t total;
  DecodePlan plan;
};

// Fixed partitions: CTA = (head, item, query row); its 4 warps merge a quarter
// of the item's partitions each, then warp 0 combines the four partial merges
// (shared memory) and writes the output row.  Items with a single partition
// wrote their output directly.
template <int ACT>
__global__ void __launch_bounds__(128) reduce_fixed_kernel(const __grid_constant__ ReduceKParams prm) {
  dev::grid_dep_wait();
  dev::grid_dep_launch();
  const DecodePlan& P = prm.plan;
  const int row = blockIdx.x % prm.group;
  const int hi = blockIdx.x / prm.group;
  const int h = hi / P.n;
  const int i = hi - h * P.n;
  const int np = P.pre[i + 1] - P.pre[i];
  if (np <= 1) return;  // uniform over the CTA
  const int64_t base = static_cast<int64_t>(h) * P.per_head + P.pre[i];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (np + 3) / 4;
  const int kb = min(np, warp * per), ke = min(np, kb + per);
  float M, L;
  float4 acc;
  merge_row_part(prm.partials, row, kb, ke, [&](int q) { return base + q; }, lane, M, L, acc);
  __shared__ float s_m[4], s_l[4];
  __shared__ float4 s_acc[4][32];
  if (lane == 0) {
    s_m[warp] = M;
    s_l[warp] = L;
  }
  s_acc[warp][lane] = acc;
  __syncthreads();
  if (warp != 0) return;
  float Mt = fmaxf(fmaxf(s_m[0], s_m[1]), fmaxf(s_m[2], s_m[3]));
  const float ref = Mt == -INFINITY ? 0.f : Mt;
  float Lt = 0.f;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float wq = dev::exp2_approx(s_m[q] - ref);  // 0 for an empty quarter
    const float4 x = s_acc[q][lane];
    Lt += wq * s_l[q];
    a.x += wq * x.x;
    a.y += wq * x.y;
    a.z += wq * x.z;
    a.w += wq * x.w;
  }
  const float inv = 1.f / Lt;
  uint16_t* orow = reinterpret_cast<uint16_t*>(prm.out) + i * prm.q_item_stride +
                   (h * prm.group + row) * kHeadDim;
  const uint32_t lo = static_cast<uint32_t>(f32_to_act<ACT>(a.x * inv)) |
                      (static_cast<uint32_t>(f32_to_act<ACT>(a.y * inv)) << 16);
  const uint32_t hi2 = static_cast<uint32_t>(f32_to_act<ACT>(a.z * inv)) |
                       (static_cast<uint32_t>(f32_to_act<ACT>(a.w * inv)) << 16);
  *reinterpret_cast<uint2*>(orow + 4 * lane) = make_uint2(lo, hi2);
}

// ================================================================== launchers
template <int KV>
constexpr size_t smem_bytes() {
  // rings, one mbarrier per stage, the cache row of each staged block, one
  // mbarrier per warp for merge staging
  return 1024 + kWarps * Tile<KV>::kRingBytes + kWarps * Tile<KV>::kStages * (8 + 4) + kWarps * 8;
}

template <int KV, int ACT, int G, class PlanT>
cudaError_t run_decode(const DecodeKParams<PlanT>& prm, const CUtensorMap* tmk,
                       const CUtensorMap* tmv, cudaStream_t stream) {
  constexpr size_t smem = smem_bytes<KV>();
  static uint64_t configured = 0;  // bit per device: dynamic shared memory attribute set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured >> dev & 1u)) {
    e = cudaFuncSetAttribute(decode_kernel<KV, ACT, G, PlanT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= uint64_t{1} << dev;
  }
  const int grid = (prm.plan.workers + kWarps - 1) / kWarps;
  return launch_pdl(decode_kernel<KV, ACT, G, PlanT>, dim3(grid), dim3(kWarps * 32), smem, stream,
                    prm, *tmk, *tmv);
}

template <int KV, int ACT>
cudaError_t dispatch_group(const DecodeKParams<DecodePlan>& prm, const CUtensorMap* tmk,
                           const CUtensorMap* tmv, cudaStream_t stream) {
  switch (prm.group) {
    case 1: return run_decode<KV, ACT, 1>(prm, tmk, tmv, stream);
    case 2: return run_decode<KV, ACT, 2>(prm, tmk, tmv, stream);
    case 4: return run_decode<KV, ACT, 4>(prm, tmk, tmv, stream);
    case 8: return run_decode<KV, ACT, 8>(prm, tmk, tmv, stream);
    default: return cudaErrorInvalidValue;
  }
}

// A sibling set needs members x G <= 8 rows with at least two members.
template <int KV, int ACT>
cudaError_t dispatch_group(const DecodeKParams<SibPlan>& prm, const CUtensorMap* tmk,
                           const CUtensorMap* tmv, cudaStream_t stream) {
  switch (prm.group) {
    case 1: return run_decode<KV, ACT, 1>(prm, tmk, tmv, stream);
    case 2: return run_decode<KV, ACT, 2>(prm, tmk, tmv, stream);
    case 4: return run_decode<KV, ACT, 4>(prm, tmk, tmv, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <class PlanT>
cudaError_t dispatch_dtypes(const PoolView& pool, const DecodeKParams<PlanT>& prm,
                            const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t stream) {
  if (pool.kv_dtype == kFP8) {
    return pool.act_dtype == kBF16 ? dispatch_group<kFP8, kBF16>(prm, tmk, tmv, stream)
                                   : dispatch_group<kFP8, kFP16>(prm, tmk, tmv, stream);
  }
  if (pool.kv_dtype == kBF16) return dispatch_group<kBF16, kBF16>(prm, tmk, tmv, stream);
  return dispatch_group<kFP16, kFP16>(prm, tmk, tmv, stream);
}

}  // namespace

int decode_warps_per_cta() { return kWarps; }

int decode_worker_capacity(int kv_dtype, int /*group*/, int num_sms) {
  const size_t smem = kv_dtype == kFP8 ? smem_bytes<kFP8>() : smem_bytes<kBF16>();
  const size_t per_sm = 227 * 1024;
  const int ctas = std::max<int>(1, static_cast<int>(per_sm / smem));
  return std::min(kMaxWorkers, num_sms * ctas * kWarps);
}

cudaError_t launch_decode(const PoolView& pool, const CacheMaps& maps, const DecodePlan& plan,
                          const DecodeArgs& args, cudaStream_t stream, int* launches) {
  static thread_local DecodeKParams<DecodePlan> prm;
  fill_decode_params(prm, pool, plan, args);
  // 16-bit tiles come in whole (3-D boxes), FP8 tiles are one 2-D box each
  cudaError_t e = args.use_tc ? launch_decode_tc(pool, maps, plan, args, stream)
                              : dispatch_dtypes(pool, prm, &maps.k3, &maps.v3, stream);
  if (e != cudaSuccess) return e;
  ++*launches;

  // Stream-K splits are merged inside the decode kernel by the last worker of
  // each cut unit; fixed partitions get the separate reduction kernel.
  if (plan.mode != kSplitFixed) return cudaSuccess;
  ReduceKParams rp;
  rp.out = prm.out;
  rp.partials = pool.partials;
  rp.q_item_stride = args.q_item_stride;
  rp.group = args.group;
  rp.total = prm.total;
  std::memcpy(&rp.plan, &plan, sizeof(DecodePlan));
  const int grid = plan.n * pool.num_kv_heads * args.group;
  e = pool.act_dtype == kBF16
          ? launch_pdl(reduce_fixed_kernel<kBF16>, dim3(grid), dim3(128), 0, stream, rp)
          : launch_pdl(reduce_fixed_kernel<kFP16>, dim3(grid), dim3(128), 0, stream, rp);
  if (e == cudaSuccess) ++*launches;
  return e;
}

cudaError_t launch_decode_sib(const PoolView& pool, const CacheMaps& maps, const SibPlan& plan,
                              const DecodeArgs& args, cudaStream_t stream, int* launches) {
  static thread_local DecodeKParams<SibPlan> prm;
  fill_decode_params(prm, pool, plan, args);
  const cudaError_t e = dispatch_dtypes(pool, prm, &maps.k3, &maps.v3, stream);
  if (e == cudaSuccess) ++*launches;
  return e;
}

}  // namespace pa
