// Paged decode attention on the 5th-generation tensor cores (tcgen05) for a
// query group of G = 8 over a 16-bit KV cache.
//
// Same result as decode_kernel (kernels_decode.cu): for every (sequence,
// query head) out = sum_t softmax_t(scale * q . k_t) v_t over the sequence's
// tokens, read through its block table (kv-cache-pagedattention-serving,
// PagedAttention: virtual memory for GPUs).  The 8 query heads that share a
// KV head ("Managing the KV Cache": the 80-layer model's 64 query heads over 8
// KV heads) are a real 8-column contraction, so both products run on tcgen05
// with fp32 accumulators in tensor memory:
//
//   S^T[128 tokens][16] = K[128 tokens][128 d] . Q^T      (A, B K-major, 128B swizzle)
//   O^T[128 d][16]     += V^T[128 d][128 tokens] . P^T    (A = the V tile read MN-major,
//                                                          B = P^T MN-major, no swizzle)
//
// The query group sits on N.  N = 16: Q's rows 8..15 are zero for S, and for
// O the 16 columns carry P = hi + lo (each rounded to the KV dtype, columns
// 0..7 and 8..15), so P's rounding error is 2^-17 relative for bf16 instead
// of 2^-9; the two halves of O^T are added in the epilogue.
//
// CTA = one worker (one per SM, 192 threads):
//   warp 0     TMA producer: per 128-token tile, 8 blocks x (K, V) x 2 d-halves
//              of 64 elements into a 3-stage ring (64 KB a stage), and the
//              segment's 8 query rows (a tensor map over q) into one of two
//              Q buffers;
//   warp 1     allocates 64 TMEM columns; one lane issues the MMAs and commits
//              them to mbarriers; the warp patches the fused append's rows
//              into a staged tile and zeroes V rows past a sequence's length;
//   warps 2-5  one TMEM lane (token for S^T, d for O^T) per thread: online
//              softmax with a lazily moved reference max (O is rescaled only
//              when a tile's max exceeds the reference by more than 2^8),
//              P^T into shared memory, and the epilogue (output rows, or a
//              split-KV partial merged by log-sum-exp as in decode_kernel).
// Work is split over the CTAs exactly as decode_kernel splits it over warps
// (stream-K shares, fixed partitions or whole sequences); segments are cut
// into tiles of up to 8 blocks.  Every wait is bounded; a wait that gives up
// sets PA_DEVERR_TIMEOUT and the CTA drains its copies, frees its tensor
// memory and returns.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "device_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

#include "decode_common.cuh"

constexpr int kTcTiles = 8;                    // 16-token tiles per stage: 128 tokens on M
constexpr int kTcStages = 3;
constexpr int kTcHalf = kTcTiles * 2048;       // one 64-element d-half of 8 tiles (16 KB)
constexpr int kTcKV = 2 * kTcHalf;             // K or V of a stage (32 KB)
constexpr int kTcStage = 2 * kTcKV;            // K and V (64 KB)
constexpr int kTcQ = 4096;                     // [2 d-halves][16 rows][128 B]
constexpr int kTcP = 4096;                     // P^T: [16 token groups][2 column blocks][8][8]
constexpr int kTcCols = 64;                    // TMEM: S^T x 2 buffers (16 each), O^T (16)
constexpr int kTcThreads = 224;
constexpr int kTcSoftmax = 128;                // threads of warps 2..5

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr int kOffQ = kTcStages * kTcStage;                  // 2 Q buffers
constexpr int kOffP = kOffQ + 2 * kTcQ;                      // 2 P buffers (by tile parity)
constexpr int kOffBar = kOffP + 2 * kTcP;
// barriers: full[3] empty[3] qfull[2] qempty[2] sfull[2] sempty[2] pfull[2] obar[2] done
// part[2]; pfull[b] / obar[b] complete with the softmax / P.V of each tile of
// parity b (the softmax may run one tile ahead of the MMA warp's wait, so one
// barrier would let two phases complete under one parity); part[k] completes
// once, when the partial result of slot 2w + k is written
constexpr int kBarFull = 0, kBarEmpty = 3, kBarQFull = 6, kBarQEmpty = 8, kBarSFull = 10,
              kBarSEmpty = 12, kBarPFull = 14, kBarO = 16, kBarDone = 18, kBarPart = 19,
              kNumBars = 21;
constexpr int kOffTmem = kOffBar + kNumBars * 8;              // TMEM base address
constexpr int kOffRows = kOffTmem + 8;                        // cache row of each staged tile [3][8]
constexpr int kOffRed = kOffRows + kTcStages * kTcTiles * 4;  // reductions [2][4][8] x 2
constexpr int kTcSmem = kOffRed + 2 * 2 * 4 * 8 * 4;
constexpr size_t kTcSmemAlloc = 1024 + kTcSmem;
static_assert(kTcSmemAlloc <= 227 * 1024, "tcgen05 decode exceeds the shared memory of an SM");

// Operand layouts (UMMA shared-memory descriptors, sm_100 format: start
// address, leading and stride byte offsets in 16-byte units, version 1,
// layout type in bits 61..63).
constexpr uint32_t kLayoutSW128 = 2, kLayoutNone = 0;
constexpr uint32_t kPvALbo = 16384, kPvASbo = 1024;  // V^T: d-halves 16 KB apart, 8-token groups 1 KB
constexpr uint32_t kPvBLbo = 256, kPvBSbo = 128;     // P^T: 8-token groups 256 B, column blocks 128 B

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t{1} << 46) |
         (static_cast<uint64_t>(layout & 7u) << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulate, A/B bf16 or f16,
// major-ness of A and B, N >> 3, M >> 4.
__host__ __device__ constexpr uint32_t instr_desc(bool bf16, bool a_mn, bool b_mn, int M, int N) {
  return (1u << 4) | (uint32_t(bf16) << 7) | (uint32_t(bf16) << 10) | (uint32_t(a_mn) << 15) |
         (uint32_t(b_mn) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(static_cast<uint32_t>(acc)));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Named barrier of the softmax warps that also ORs a predicate over them, so
// every softmax warp takes the same branch after a wait that may give up.
__device__ __forceinline__ bool softmax_bar_or(bool x) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(x)), "n"(kTcSoftmax)
      : "memory");
  return r != 0;
}

// Bounded wait taken by a whole warp with one outcome for all its lanes (a
// phase that any lane saw complete has completed).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  return __any_sync(0xffffffffu, dev::mbar_wait_bounded(bar, parity, kWaitLimit));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

struct TcParams {
  DecodeKParams<DecodePlan> k;   // plan, split and fused-append arguments
  int32_t num_q_heads;
};

// Blocks [b, b + n) of a segment as a tile: tokens of the tile are
// (b + j) * 16 + r for block j < n, row r; valid while below the length.
struct TcTile {
  int32_t b, n, valid;  // first block, blocks, valid tokens from the tile start
};
__device__ __forceinline__ TcTile tile_of(const Seg& s, int32_t b) {
  TcTile t;
  t.b = b;
  t.n = min(kTcTiles, s.b1 - b);
  t.valid = min(t.n * kBlock, s.len - b * kBlock);
  return t;
}

template <int ACT>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const __grid_constant__ TcParams tp, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmq) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const DecodeKParams<DecodePlan>& prm = tp.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w = blockIdx.x;
  const int W = prm.plan.workers;
  if (w >= W) return;  // uniform over the CTA
  const uint32_t base = dev::smem_u32(sm);
  const uint32_t bars = base + kOffBar;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  int32_t* rows_s = reinterpret_cast<int32_t*>(sm + kOffRows);
  float* red = reinterpret_cast<float*>(sm + kOffRed);  // [max|sum][2][4 warps][8]

  // ---- set-up: barriers, zero rows 8..15 of both Q buffers, TMEM
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      dev::mbar_init(bar(kBarFull + s), 1);
      dev::mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(bar(kBarQFull + b), 1);
      dev::mbar_init(bar(kBarQEmpty + b), 1);
      dev::mbar_init(bar(kBarSFull + b), 1);
      dev::mbar_init(bar(kBarSEmpty + b), 4);
    }
    dev::mbar_init(bar(kBarPFull), 4);
    dev::mbar_init(bar(kBarPFull + 1), 4);
    dev::mbar_init(bar(kBarO), 1);
    dev::mbar_init(bar(kBarO + 1), 1);
    dev::mbar_init(bar(kBarDone), 1);
    dev::mbar_init(bar(kBarPart), 4);
    dev::mbar_init(bar(kBarPart + 1), 4);
    dev::fence_mbar_init();
    dev::tma_prefetch_desc(&tmk);
    dev::tma_prefetch_desc(&tmv);
    dev::tma_prefetch_desc(&tmq);
  }
  for (int i = threadIdx.x; i < 2 * 2 * 1024 / 16; i += kTcThreads) {
    const int buf = i / 128, half = (i / 64) & 1, c = i & 63;
    *reinterpret_cast<uint4*>(sm + kOffQ + buf * kTcQ + half * 2048 + 1024 + c * 16) = make_uint4(0, 0, 0, 0);
  }
  dev::fence_proxy_async_smem();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + kOffTmem),
                 "n"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + kOffTmem);

  const int64_t g0 = worker_start(prm.total, w, W);
  const int64_t g1 = worker_start(prm.total, w + 1, W);
  Cursor cur;
  cur.init(prm, g0, g1, w);  // kernel parameters only: may overlap the previous kernel
  dev::grid_dep_wait();
  bool failed = false;

  if (warp == 0) {
    // ================================================================ producer
    uint32_t tile_i = 0, seg_i = 0, q_issued = 0;
    int32_t tc_val = 0, tc_base = 0, tc_unit = -1;
    for (;;) {
      const Seg s = cur.next(prm);
      if (!s.valid) break;
      const uint32_t qb = seg_i & 1;
      if (!warp_wait(bar(kBarQEmpty + qb), ((seg_i >> 1) & 1) ^ 1)) {
        failed = true;
        break;
      }
      if (lane == 0) {
        const int32_t qrow = s.i * tp.num_q_heads + s.h * 8;
        const uint32_t qdst = base + kOffQ + qb * kTcQ;
        dev::mbar_arrive_expect_tx(bar(kBarQFull + qb), 2048);
        dev::tma_load_2d(qdst, &tmq, 0, qrow, bar(kBarQFull + qb));
        dev::tma_load_2d(qdst + 2048, &tmq, 64, qrow, bar(kBarQFull + qb));
      }
      ++q_issued;
      for (int32_t b = s.b0; b < s.b1; b += kTcTiles) {
        const TcTile t = tile_of(s, b);
        const uint32_t st = tile_i % kTcStages;
        if (!warp_wait(bar(kBarEmpty + st), ((tile_i / kTcStages) & 1) ^ 1)) {
          failed = true;
          break;
        }
        if (lane == 0) dev::mbar_arrive_expect_tx(bar(kBarFull + st), t.n * 8192);
        __syncwarp();  // the expected bytes are counted before any copy is issued
        // physical ids of blocks b .. b + n - 1 (the lane cache holds 32 of the unit's)
        if (s.k != tc_unit || b < tc_base || b + t.n > tc_base + 32) {
          tc_unit = s.k;
          tc_base = b;
          const BlockRef r = locate<8>(prm, s, b + lane);
          const int32_t e = r.b >> prm.bshift;
          int32_t v = r.b >= 0 && e < prm.mbps ? prm.tables[static_cast<int64_t>(r.seq) * prm.mbps + e] : 0;
          tc_val = static_cast<int32_t>((static_cast<uint32_t>(v) << 1) |
                                        static_cast<uint32_t>(r.b & ((1 << prm.bshift) - 1)));
        }
        // lane j issues block j's four copies: the copies of a tile go out in
        // parallel rather than one after another from a single lane
        const int32_t tv = __shfl_sync(0xffffffffu, tc_val, (b - tc_base + lane) & 31);
        if (lane < t.n) {
          int32_t phys = static_cast<int32_t>(static_cast<uint32_t>(tv) >> 1);
          if (static_cast<uint32_t>(phys) >= static_cast<uint32_t>(prm.num_blocks)) {
            atomicOr(prm.err, kErrBadBlock);
            phys = 0;
          }
          const int32_t row =
              (((prm.layer * prm.num_blocks + phys) * prm.num_kv_heads + s.h) << (4 + prm.bshift)) +
              (tv & 1) * kBlock;
          rows_s[st * kTcTiles + lane] = row;
          const uint32_t dst = base + st * kTcStage + lane * 2048;
          dev::tma_load_2d(dst, &tmk, 0, row, bar(kBarFull + st));
          dev::tma_load_2d(dst + kTcHalf, &tmk, 64, row, bar(kBarFull + st));
          dev::tma_load_2d(dst + kTcKV, &tmv, 0, row, bar(kBarFull + st));
          dev::tma_load_2d(dst + kTcKV + kTcHalf, &tmv, 64, row, bar(kBarFull + st));
        }
        ++tile_i;
      }
      if (failed) break;
      ++seg_i;
    }
    // every copy is out: the next kernel in the stream may start placing its
    // blocks (not at kernel start: a queued successor's launch slows the
    // first copies)
    dev::grid_dep_launch();
    // let every copy already issued land before the CTA can exit: the last
    // tile of each stage and the last load of each Q buffer
    for (uint32_t k = tile_i > kTcStages ? tile_i - kTcStages : 0; k < tile_i; ++k)
      warp_wait(bar(kBarFull + k % kTcStages), (k / kTcStages) & 1);
    for (uint32_t k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
      warp_wait(bar(kBarQFull + (k & 1)), (k >> 1) & 1);
  } else if (warp == 1) {
    // ================================================================== MMA
    constexpr bool kBf = ACT == kBF16;
    constexpr uint32_t kIdS = instr_desc(kBf, false, false, 128, 16);
    constexpr uint32_t kIdO = instr_desc(kBf, true, true, 128, 16);
    // An event loop: the P.V of the oldest tile whose softmax is done, and the
    // S of the next tile whose data, S buffer and query rows are in, each
    // issued as soon as it can go (a P.V never waits for a later tile's copy,
    // so a stage is released as early as possible).
    struct PvTile {
      uint32_t st;
      int32_t n;
      bool first;
    };
    PvTile ring[4];
    uint32_t ns = 0, np = 0, seg_i = 0;   // tiles whose S / P.V went out; segments started
    bool s_done = false, q_ready = false;
    Seg s;
    int32_t b = 0;
    auto next_segment = [&]() {
      s = cur.next(prm);
      s_done = !s.valid;
      b = s.b0;
      q_ready = false;
    };
    auto ready = [&](int idx, uint32_t parity) {
      return __any_sync(0xffffffffu, dev::mbar_test_wait(bar(idx), parity));
    };
    next_segment();
    uint32_t idle = 0;
    while (!s_done || np < ns) {
      bool progress = false;
      if (np < ns && ready(kBarPFull + (np & 1), (np >> 1) & 1)) {
        tc_fence_after();
        const PvTile& pt = ring[np & 3];
        if (lane == 0) {
          const uint32_t vbase = base + pt.st * kTcStage + kTcKV;
          const uint32_t pbase = base + kOffP + (np & 1) * kTcP;
          for (int j = 0; j < pt.n; ++j)
            umma(tmem + 32, smem_desc(vbase + j * 2048, kPvALbo, kPvASbo, kLayoutSW128),
                 smem_desc(pbase + j * 512, kPvBLbo, kPvBSbo, kLayoutNone), kIdO, !(pt.first && j == 0));
          umma_commit(bar(kBarO + (np & 1)));
          umma_commit(bar(kBarEmpty + pt.st));
        }
        __syncwarp();
        ++np;
        progress = true;
      }
      if (!s_done && ns - np < 3) {
        const uint32_t qb = seg_i & 1;
        const uint32_t st = ns % kTcStages;
        if (!q_ready) q_ready = ready(kBarQFull + qb, (seg_i >> 1) & 1);
        if (q_ready && ready(kBarFull + st, (ns / kTcStages) & 1) &&
            ready(kBarSEmpty + (ns & 1), ((ns >> 1) & 1) ^ 1)) {
          const TcTile t = tile_of(s, b);
          const uint32_t kst = base + st * kTcStage;
          uint8_t* kst_p = sm + st * kTcStage;
          // the item's last block in this tile: fused append row, V rows past the length
          const int32_t last = (s.len - 1) / kBlock - b;
          if (last >= 0 && last < t.n) {
            const int r = (s.len - 1) % kBlock;
            if (prm.k_new != nullptr) {
              const int kv = lane >> 4, c = lane & 15;
              const uint4 val = __ldcg(new_row_ptr(prm, s.h, s.i, lane));
              uint8_t* tile = kst_p + kv * kTcKV + (c >> 3) * kTcHalf + last * 2048;
              *reinterpret_cast<uint4*>(tile + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = val;
              uint8_t* cache = kv ? prm.v_cache : prm.k_cache;
              const int64_t dst_el =
                  (static_cast<int64_t>(rows_s[st * kTcTiles + last]) + r) * kHeadDim + c * 8;
              *reinterpret_cast<uint4*>(cache + dst_el * 2) = val;
            }
            const int nvalid = r + 1;
            for (int c = lane; c < (kBlock - nvalid) * 16; c += 32) {
              const int tr = nvalid + c / 16, k = c % 16;
              *reinterpret_cast<uint4*>(kst_p + kTcKV + (k >> 3) * kTcHalf + last * 2048 + tr * 128 +
                                        ((k & 7) << 4)) = make_uint4(0, 0, 0, 0);
            }
            dev::fence_proxy_async_smem();
          }
          __syncwarp();
          tc_fence_after();
          const uint32_t sb = ns & 1;
          const bool seg_last = b + kTcTiles >= s.b1;
          if (lane == 0) {
            const uint32_t qbase = base + kOffQ + qb * kTcQ;
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ka = kst + (kk >> 2) * kTcHalf + (kk & 3) * 32;
              const uint32_t qa = qbase + (kk >> 2) * 2048 + (kk & 3) * 32;
              umma(tmem + sb * 16, smem_desc(ka, 16, 1024, kLayoutSW128),
                   smem_desc(qa, 16, 1024, kLayoutSW128), kIdS, kk > 0);
            }
            umma_commit(bar(kBarSFull + sb));
            if (seg_last) umma_commit(bar(kBarQEmpty + qb));  // last S of the segment
          }
          __syncwarp();
          ring[ns & 3] = PvTile{st, t.n, b == s.b0};
          ++ns;
          b += kTcTiles;
          if (seg_last) {
            ++seg_i;
            next_segment();
          }
          progress = true;
        }
      }
      if (progress) {
        idle = 0;
      } else if (++idle > kWaitLimit) {
        failed = true;
        break;
      }
    }
    // every MMA issued has finished before the tensor memory is released
    if (lane == 0) umma_commit(bar(kBarDone));
    __syncwarp();
    warp_wait(bar(kBarDone), 0);
  } else if (warp == 6) {
    // ================================================================ merge
    // A worker writes at most one partial to slot 2w (its share starts inside
    // a unit) and one to slot 2w + 1 (its share ends inside one).
    if (prm.plan.mode == kSplitStreamK) {
      for (;;) {
        const Seg s = cur.next(prm);
        if (!s.valid) break;
        if (s.dest < 0) continue;
        if (!warp_wait(bar(kBarPart + (s.dest & 1)), 0)) {
          failed = true;
          break;
        }
        settle_partial<ACT, 8, 8>(prm, s, 8, lane);
      }
    }
  } else {
    // ======================================================= softmax, epilogue
    const int sw = warp - 2;                    // softmax warp 0..3
    const int quad = warp & 3;                  // TMEM lanes 32*quad .. 32*quad+31
    const int t = quad * 32 + lane;             // token row of S^T, d row of O^T
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float sl2 = prm.scale * kLog2e;
    uint32_t tile_i = 0, seg_i = 0;
    // the P.V of tile i completes phase (i >> 1) of obar[i & 1]
    auto pv_done = [&](uint32_t i) {
      return dev::mbar_wait_bounded(bar(kBarO + (i & 1)), (i >> 1) & 1, kWaitLimit);
    };
    // `failed` may differ between the softmax warps until the next barrier ORs
    // it over them; `abort` is that agreed value, the same in every warp
    bool abort = false;
    for (;;) {
      const Seg s = cur.next(prm);
      if (!s.valid) break;
      float mref[8], lpart[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        mref[g] = -INFINITY;
        lpart[g] = 0.f;
      }
      for (int32_t b = s.b0; b < s.b1; b += kTcTiles) {
        const TcTile tt = tile_of(s, b);
        const uint32_t sb = tile_i & 1;
        bool ok = dev::mbar_wait_bounded(bar(kBarSFull + sb), (tile_i >> 1) & 1, kWaitLimit);
        tc_fence_after();
        float x[8];
        tmem_ld8(tl + sb * 16, x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarSEmpty + sb));
        const bool valid = t < tt.valid;
        float mx[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          x[g] = valid ? x[g] * sl2 : -INFINITY;
          mx[g] = x[g];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int g = 0; g < 8; ++g) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
        float* rm = red + (tile_i & 1) * 32;
        if (lane == 0) {  // after the butterfly every lane holds all 8 maxima
          *reinterpret_cast<float4*>(rm + sw * 8) = make_float4(mx[0], mx[1], mx[2], mx[3]);
          *reinterpret_cast<float4*>(rm + sw * 8 + 4) = make_float4(mx[4], mx[5], mx[6], mx[7]);
        }
        if (softmax_bar_or(!ok || failed)) {
          failed = abort = true;
          break;
        }
        bool rescale = false;
        float tmax[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          tmax[g] = fmaxf(fmaxf(rm[g], rm[8 + g]), fmaxf(rm[16 + g], rm[24 + g]));
          rescale |= tmax[g] > mref[g] + 8.f;
        }
        float corr[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          corr[g] = 1.f;
          if (rescale) {
            const float mn = fmaxf(mref[g], tmax[g]);
            corr[g] = mref[g] == -INFINITY ? 0.f : dev::exp2_approx(mref[g] - mn);
            mref[g] = mn;
          }
        }
        float p[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          p[g] = dev::exp2_approx(x[g] - mref[g]);
          lpart[g] = lpart[g] * corr[g] + p[g];
        }
        // O is rescaled between the P.V of the previous tile and this one's;
        // otherwise only this tile's P buffer must be free (the P.V of two
        // tiles back), so this softmax overlaps the previous tile's P.V
        const bool rescale_o = rescale && b != s.b0;
        if (rescale_o) {
          ok = pv_done(tile_i - 1);
        } else if (tile_i > 1) {
          ok = pv_done(tile_i - 2);
        }
        tc_fence_after();
        if (rescale_o) {
          float o[16];
          tmem_ld16(tl + 32, o);
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] *= corr[c & 7];
          tmem_st16(tl + 32, o);
        }
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if constexpr (ACT == kBF16) {
            hi[k] = dev::pack_bf16(p[2 * k], p[2 * k + 1]);
            lo[k] = dev::pack_bf16(p[2 * k] - dev::bf16lo_to_f32(hi[k]), p[2 * k + 1] - dev::bf16hi_to_f32(hi[k]));
          } else {
            hi[k] = dev::pack_f16(p[2 * k], p[2 * k + 1]);
            lo[k] = dev::pack_f16(p[2 * k] - dev::f16lo_to_f32(hi[k]), p[2 * k + 1] - dev::f16hi_to_f32(hi[k]));
          }
        }
        uint8_t* pt = sm + kOffP + (tile_i & 1) * kTcP + (t >> 3) * 256 + (t & 7) * 16;
        *reinterpret_cast<uint4*>(pt) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(pt + 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        dev::fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarPFull + (tile_i & 1)));
        failed |= !ok;   // agreed on at the next barrier
        ++tile_i;
      }
      if (abort) break;
      // ---- epilogue: the segment's last P.V, the row sums, the output
      bool ok = !failed && pv_done(tile_i - 1);
      tc_fence_after();
      float oc[16];
      tmem_ld16(tl + 32, oc);
      tc_fence_before();
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < 8; ++g) lpart[g] += __shfl_xor_sync(0xffffffffu, lpart[g], o);
      float* rs = red + 64 + (seg_i & 1) * 32;
      if (lane == 0) {
        *reinterpret_cast<float4*>(rs + sw * 8) = make_float4(lpart[0], lpart[1], lpart[2], lpart[3]);
        *reinterpret_cast<float4*>(rs + sw * 8 + 4) = make_float4(lpart[4], lpart[5], lpart[6], lpart[7]);
      }
      if (softmax_bar_or(!ok)) {
        failed = abort = true;
        break;
      }
      float lt[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) lt[g] = (rs[g] + rs[8 + g]) + (rs[16 + g] + rs[24 + g]);
      if (s.dest < 0) {
        uint16_t* out = reinterpret_cast<uint16_t*>(prm.out);
#pragma unroll
        for (int g = 0; g < 8; ++g)
          out[row_offset<8>(prm, s, g) + t] = f32_to_act<ACT>((oc[g] + oc[8 + g]) / lt[g]);
      } else {
        float* slot = prm.partials + static_cast<int64_t>(s.dest) * kPartialSlotFloats;
#pragma unroll
        for (int g = 0; g < 8; ++g) slot[g * kHeadDim + t] = oc[g] + oc[8 + g];
        if (t == 0) {
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<float2*>(slot + kMaxGroup * kHeadDim + 2 * g) = make_float2(mref[g], lt[g]);
        }
        if (prm.plan.mode == kSplitStreamK) {
          // the merge warp counts this partial in (and merges, if last) while
          // the softmax goes on with the next segment
          __threadfence();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarPart + (s.dest & 1)));
        }
      }
      ++seg_i;
    }
  }
  if (failed && lane == 0) atomicOr(prm.err, kErrTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTcCols)
                              : "memory");
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tc_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <int ACT>
cudaError_t run_tc(const TcParams& tp, const CUtensorMap* tmk, const CUtensorMap* tmv,
                   const CUtensorMap& tmq, cudaStream_t stream) {
  static uint64_t configured = 0;  // bit per device: dynamic shared memory attribute set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured >> dev & 1u)) {
    e = cudaFuncSetAttribute(decode_tc_kernel<ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kTcSmemAlloc));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured |= uint64_t{1} << dev;
  }
  return launch_pdl(decode_tc_kernel<ACT>, dim3(tp.k.plan.workers), dim3(kTcThreads), kTcSmemAlloc, stream,
                    tp, *tmk, *tmv, tmq);
}

}  // namespace

bool decode_tc_applies(int kv_dtype, int group) { return group == 8 && kv_dtype != kFP8; }

cudaError_t launch_decode_tc(const PoolView& pool, const CacheMaps& maps, const DecodePlan& plan,
                             const DecodeArgs& args, cudaStream_t stream) {
  if (!decode_tc_applies(pool.kv_dtype, args.group)) return cudaErrorInvalidValue;
  EncodeTiledFn encode = tc_encoder();
  if (!encode) return cudaErrorNotSupported;
  static thread_local TcParams tp;
  fill_decode_params(tp.k, pool, plan, args);
  tp.num_q_heads = args.num_q_heads;
  // q of this launch as a 2-D tensor [items * H_q][128], boxes of 8 rows x 64
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim),
                              static_cast<cuuint64_t>(plan.n) * static_cast<cuuint64_t>(args.num_q_heads)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
  const cuuint32_t box[2] = {64u, 8u};
  const cuuint32_t estr[2] = {1, 1};
  CUtensorMap tmq;
  if (encode(&tmq, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint8_t*>(tp.k.q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return pool.act_dtype == kBF16 ? run_tc<kBF16>(tp, &maps.k, &maps.v, tmq, stream)
                                 : run_tc<kFP16>(tp, &maps.k, &maps.v, tmq, stream);
}

int decode_tc_worker_capacity(int num_sms) { return std::min(kMaxWorkers, num_sms); }

}  // namespace pa
