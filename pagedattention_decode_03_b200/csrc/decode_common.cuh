// Work split and merge shared by the decode kernels (included inside
// namespace pa { namespace { ... } } of each kernel file): launch parameters,
// the stream-K / fixed / whole-sequence segments of a worker's share, where a
// segment's KV tiles live, and the log-sum-exp merge of split results.
#pragma once
// (no includes: the including file provides device_common.cuh, pa_internal.h
// and <type_traits>)
constexpr int kBlock = 16;             // tokens per staged tile: a 16-token block, or half of a
                                       // 32-token block (the kernel walks 16-token tiles)
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

template <class PlanT>
struct DecodeKParams {
  const uint8_t* q;
  uint8_t* out;
  const int32_t* tables;
  float* partials;
  int32_t* counters;       // stream-K arrival counters (zero between launches)
  uint32_t* err;
  const float* k_scale;
  const float* v_scale;
  int64_t q_item_stride;   // elements between items of q / out
  float scale;
  int32_t layer, num_kv_heads, num_blocks, mbps, group;
  int32_t bshift;          // log2(block_size / 16): 0 for 16-token blocks, 1 for 32
  int64_t total;           // work units over all heads
  // Fused append (null k_new: none): the K/V rows of each item's last token,
  // [n][H][128] act dtype, written into the cache by the worker that reads the
  // item's last block, which also patches them into its staged tile.
  const uint8_t* k_new;
  const uint8_t* v_new;
  uint8_t* k_cache;
  uint8_t* v_cache;
  const float* k_inv;
  const float* v_inv;
  PlanT plan;
};

template <class PlanT>
constexpr bool kIsSib = std::is_same<PlanT, SibPlan>::value;
template <class Prm>
constexpr bool kSibParams = std::is_same<Prm, DecodeKParams<SibPlan>>::value;

// A worker's contiguous piece of one work unit.  Positions b0 .. b1-1 are the
// unit's KV blocks in order (for a plain unit: table blocks of item i).
struct Seg {
  int32_t h, i, b0, b1, dest, len, seq;
  int32_t k;      // work unit (== i for plain plans)
  bool valid;
  bool shared;    // a sibling set (two or more items) of a sibling plan
};

// Table position, valid length and active query rows of one KV block.
struct BlockRef {
  int32_t seq, b, len;
  uint32_t cols;  // bit r set: query row r takes part (all 8 for plain units)
  int32_t item;   // the item whose table row this is
};

__device__ __forceinline__ int n_entries(const DecodePlan& P) { return P.n; }
__device__ __forceinline__ int n_entries(const SibPlan& P) { return P.nu; }
__device__ __forceinline__ int plan_mode(const DecodePlan& P) { return P.mode; }
__device__ __forceinline__ int plan_mode(const SibPlan&) { return kSplitStreamK; }

// Index of the entry whose prefix range holds r: pre[i] <= r < pre[i+1].
template <class PlanT>
__device__ __forceinline__ int find_item(const PlanT& P, int64_t r) {
  int lo = 0, hi = n_entries(P) - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.pre[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// find_item, first trying `hint` and the entry after it (a worker's next
// segment almost always starts in one of those).
template <class PlanT>
__device__ __forceinline__ int find_item_hint(const PlanT& P, int64_t r, int hint) {
  const int n = n_entries(P);
  if (hint >= 0 && hint < n && P.pre[hint] <= r) {
    if (r < P.pre[hint + 1]) return hint;
    if (hint + 1 < n && r < P.pre[hint + 2]) return hint + 1;
  }
  return find_item(P, r);
}

__device__ __forceinline__ int64_t worker_start(int64_t total, int w, int W) {
  return (total * w) / W;
}

// Worker whose share [worker_start(w), worker_start(w+1)) holds position x:
// the largest w with total*w < (x+1)*W.
__device__ __forceinline__ int find_worker(int64_t total, int W, int64_t x) {
  return min(W - 1, static_cast<int>(((x + 1) * W - 1) / total));
}

// Stream-K piece of one unit.  A unit occupies alpha + nb positions of the
// work axis: alpha positions that stand for the fixed cost of a segment
// (begin, finish, partial write and arrival) and carry no block, then its nb
// KV blocks.  Shares are equal in positions, so a worker whose share crosses
// unit boundaries gets fewer blocks.  From position r (offset o = r - v0 in
// the unit [v0, v1)) the worker takes `take` positions; the piece reads blocks
// [b0, b1).  Returns false when those positions hold no block.  A piece that
// covers the unit's blocks only in part writes partial slot 2w if it starts
// inside the blocks (it holds the share's start; one per worker), else 2w+1
// (it holds the share's end).
__device__ __forceinline__ bool stream_piece(int64_t r, int32_t v0, int32_t v1, int32_t alpha,
                                             int64_t avail, int w, int64_t& take, Seg& s) {
  const int32_t unit_nb = v1 - v0 - alpha;
  take = min(static_cast<int64_t>(v1) - r, avail);
  const int64_t o = r - v0;
  s.b0 = static_cast<int32_t>(max(o - alpha, int64_t{0}));
  s.b1 = static_cast<int32_t>(max(o + take - alpha, int64_t{0}));
  if (s.b1 <= s.b0) return false;
  const bool whole = s.b0 == 0 && s.b1 == unit_nb;
  s.dest = whole ? -1 : (s.b0 > 0 ? 2 * w : 2 * w + 1);
  return true;
}

// Next segment of worker `w` within the remaining range [g, g_end) of its
// share; `hint` carries the entry of the previous segment.
__device__ __forceinline__ Seg next_seg(const DecodeKParams<DecodePlan>& prm, int64_t& g,
                                        int64_t g_end, int w, int64_t /*g0*/, int& hint) {
  Seg s;
  s.shared = false;
  const DecodePlan& P = prm.plan;
  const int64_t per_head = P.per_head;
  for (;;) {
    s.valid = g < g_end;
    if (!s.valid) return s;
    s.h = static_cast<int32_t>(g / per_head);
    const int64_t r = g - static_cast<int64_t>(s.h) * per_head;
    if (P.mode == kSplitNever) {
      s.i = static_cast<int32_t>(r);
    } else {
      s.i = find_item_hint(P, r, hint);
      hint = s.i;
    }
    s.k = s.i;
    s.seq = P.seq[s.i];
    s.len = P.len[s.i];
    int32_t nb = (s.len + kBlock - 1) / kBlock;
    if (s.len <= 0 || nb > (prm.mbps << prm.bshift)) {
      atomicOr(prm.err, kErrBadLen);
      nb = min(max(nb, 1), prm.mbps << prm.bshift);
      s.len = max(s.len, 1);
    }
    if (P.mode == kSplitStreamK) {
      const int32_t v0 = P.pre[s.i], v1 = P.pre[s.i + 1];
      if (v1 - v0 - P.alpha != nb) atomicOr(prm.err, kErrBadLen);
      int64_t take;
      const bool any = stream_piece(r, v0, v1, P.alpha, g_end - g, w, take, s);
      g += take;
      if (!any) continue;
    } else if (P.mode == kSplitFixed) {
      const int32_t p = static_cast<int32_t>(r - P.pre[s.i]);
      const int32_t np = P.pre[s.i + 1] - P.pre[s.i];
      s.b0 = p * P.part_blocks;
      s.b1 = min(nb, s.b0 + P.part_blocks);
      if (s.b0 >= s.b1) {  // inconsistent lengths: clamp to an empty-free range
        atomicOr(prm.err, kErrBadLen);
        s.b0 = max(0, s.b1 - 1);
      }
      s.dest = np == 1 ? -1 : static_cast<int32_t>(g);
      g += 1;
    } else {
      s.b0 = 0;
      s.b1 = nb;
      s.dest = -1;
      g += 1;
    }
    return s;
  }
}

// Sibling plan (always stream-K): same cutting and partial slots as a plain
// stream-K plan, over units that may hold several items.
__device__ __forceinline__ Seg next_seg(const DecodeKParams<SibPlan>& prm, int64_t& g,
                                        int64_t g_end, int w, int64_t /*g0*/, int& hint) {
  Seg s;
  const SibPlan& P = prm.plan;
  for (;;) {
    s.valid = g < g_end;
    if (!s.valid) return s;
    s.h = static_cast<int32_t>(g / P.per_head);
    const int64_t r = g - static_cast<int64_t>(s.h) * P.per_head;
    s.k = find_item_hint(P, r, hint);
    hint = s.k;
    const int m0 = P.mem0[s.k];
    s.shared = P.mem0[s.k + 1] - m0 > 1;
    s.i = P.mem[m0];
    s.seq = P.seq[s.i];
    s.len = P.len[s.i];
    const int32_t v0 = P.pre[s.k], v1 = P.pre[s.k + 1];
    const int32_t unit_nb = v1 - v0 - P.alpha;
    if (!s.shared && (s.len <= 0 || (s.len + kBlock - 1) / kBlock != unit_nb || unit_nb > (prm.mbps << prm.bshift)))
      atomicOr(prm.err, kErrBadLen);
    int64_t take;
    const bool any = stream_piece(r, v0, v1, P.alpha, g_end - g, w, take, s);
    g += take;
    if (any) return s;
  }
}

// Where position o of segment s lives.  Plain plans: block o of the item.
// Sibling plans: positions below the unit's shared run cp are the common
// blocks (every row takes part); after it come the members' own blocks in
// member order, each taken only by that member's G rows.
template <int G>
__device__ __forceinline__ BlockRef locate(const DecodeKParams<DecodePlan>&, const Seg& s, int o) {
  return BlockRef{s.seq, o, s.len, 0xffu, s.i};
}
template <int G>
__device__ __forceinline__ BlockRef locate(const DecodeKParams<SibPlan>& prm, const Seg& s, int o) {
  const SibPlan& P = prm.plan;
  const int cp = P.cp[s.k];
  if (o < cp) return BlockRef{s.seq, o, s.len, 0xffu, s.i};
  const int m0 = P.mem0[s.k], m = P.mem0[s.k + 1] - m0;
  int j = 0, item = s.i;
  for (int jj = 1; jj < m; ++jj) {
    const int it = P.mem[m0 + jj];
    if (P.part[it] > o) break;
    j = jj;
    item = it;
  }
  return BlockRef{P.seq[item], cp + (o - P.part[item]), P.len[item],
                  ((1u << G) - 1u) << (j * G), item};
}

// The members of a segment's unit held in registers, lane j < m holding
// member j's item, own-block start in the unit (part), table row and length,
// so a warp locates positions with shuffles instead of walking the plan in
// parameter memory: a walk whose lanes look at different positions makes
// divergent parameter loads, which the hardware serialises.  (Plain units
// have one member and need none of this.)
struct Members {
  int32_t m, cp;                    // members, shared blocks at the unit's start
  int32_t item, part, seq, len;     // member `lane` (lanes < m)
};
__device__ __forceinline__ Members load_members(const DecodeKParams<DecodePlan>&, const Seg& s, int) {
  return Members{1, 0, s.i, 0, s.seq, s.len};
}
__device__ __forceinline__ Members load_members(const DecodeKParams<SibPlan>& prm, const Seg& s, int lane) {
  const SibPlan& P = prm.plan;
  const int m0 = P.mem0[s.k];
  Members u{P.mem0[s.k + 1] - m0, P.cp[s.k], s.i, 0, s.seq, s.len};
  if (lane < u.m) {
    u.item = P.mem[m0 + lane];
    u.part = P.part[u.item];
    u.seq = P.seq[u.item];
    u.len = P.len[u.item];
  }
  return u;
}
// locate() from registers: every lane may ask for its own position o; all 32
// lanes must call it together.
template <int G>
__device__ __forceinline__ BlockRef locate_in(const DecodeKParams<DecodePlan>&, const Members&, const Seg& s,
                                              int o) {
  return BlockRef{s.seq, o, s.len, 0xffu, s.i};
}
template <int G>
__device__ __forceinline__ BlockRef locate_in(const DecodeKParams<SibPlan>&, const Members& u, const Seg& s,
                                              int o) {
  int j = 0;
#pragma unroll
  for (int jj = 1; jj < kMaxGroup; ++jj) {
    const int pj = __shfl_sync(0xffffffffu, u.part, jj);
    if (jj < u.m && pj <= o) j = jj;
  }
  const int item = __shfl_sync(0xffffffffu, u.item, j);
  const int part = __shfl_sync(0xffffffffu, u.part, j);
  const int seq = __shfl_sync(0xffffffffu, u.seq, j);
  const int len = __shfl_sync(0xffffffffu, u.len, j);
  if (o < u.cp) return BlockRef{s.seq, o, s.len, 0xffu, s.i};
  return BlockRef{seq, u.cp + (o - part), len, ((1u << G) - 1u) << (j * G), item};
}

// The segments of one worker, in processing order.  Stream-K: a worker's last
// segment, when it starts inside the worker's share (the head of a sequence
// cut at the share's end), is processed first, then the share from its start
// (whose first segment is the tail of a sequence cut at the share's start).
// Both halves of every cut sequence thus finish early and the merge of their
// partial results happens off the kernel's critical path.
struct Cursor {
  int64_t g, end, g0, glast;
  int w;
  int hint, hint_g0;  // entry of the next segment, and of the share's start
  bool second;

  template <class Prm>
  __device__ __forceinline__ void init(const Prm& prm, int64_t s0, int64_t s1, int wk) {
    g0 = s0;
    w = wk;
    glast = s0;
    hint = hint_g0 = -1;
    const auto& P = prm.plan;
    if (plan_mode(P) == kSplitStreamK && s1 > s0) {
      // entries of the share's last and first positions, two searches
      // interleaved so their dependent loads overlap
      const int64_t x = s1 - 1;
      const int64_t h = x / P.per_head;
      const int64_t r1 = x - h * P.per_head;
      const int64_t r0 = s0 - (s0 / P.per_head) * P.per_head;
      int lo1 = 0, hi1 = n_entries(P) - 1, lo0 = 0, hi0 = hi1;
      while (lo1 < hi1 || lo0 < hi0) {
        if (lo1 < hi1) {
          const int mid = (lo1 + hi1 + 1) >> 1;
          if (P.pre[mid] <= r1) lo1 = mid; else hi1 = mid - 1;
        }
        if (lo0 < hi0) {
          const int mid = (lo0 + hi0 + 1) >> 1;
          if (P.pre[mid] <= r0) lo0 = mid; else hi0 = mid - 1;
        }
      }
      glast = max(s0, h * P.per_head + P.pre[lo1]);
      hint = lo1;
      hint_g0 = lo0;
    }
    g = glast;
    end = s1;
    second = false;
  }

  template <class Prm>
  __device__ __forceinline__ Seg next(const Prm& prm) {
    for (;;) {
      if (g >= end && !second && glast > g0) {
        second = true;
        g = g0;
        end = glast;
        hint = hint_g0;
      }
      const Seg s = next_seg(prm, g, end, w, g0, hint);
      // the first phase may hold only cost positions: go on with the second
      if (s.valid || second || glast <= g0) return s;
    }
  }
};

// ------------------------------------------------------ fused append rows
__device__ __forceinline__ bool is_last_block(const BlockRef& br) { return br.b == (br.len - 1) / kBlock; }

// Address of this lane's 16 bytes of the rows.  (Calls whose plan has sibling
// sets append with the append kernel instead: a set puts several sequences'
// last blocks into one worker's share, and their row loads would run in
// series.)
template <class Prm>
__device__ __forceinline__ const uint4* new_row_ptr(const Prm& prm, int h, int item, int lane) {
  const int64_t src_el = (static_cast<int64_t>(item) * prm.num_kv_heads + h) * kHeadDim + (lane & 15) * 8;
  return reinterpret_cast<const uint4*>((lane < 16 ? prm.k_new : prm.v_new) + src_el * 2);
}


__device__ __forceinline__ float warp_max_rows(float x) {  // over lanes sharing lane & 3
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
  return x;
}
__device__ __forceinline__ float warp_sum_rows(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  x += __shfl_xor_sync(0xffffffffu, x, 16);
  return x;
}

template <int ACT>
__device__ __forceinline__ float act_to_f32(uint16_t x) {
  if constexpr (ACT == kBF16) return __uint_as_float(static_cast<uint32_t>(x) << 16);
  else return __half2float(__ushort_as_half(x));
}

template <int ACT>
__device__ __forceinline__ uint16_t f32_to_act(float x) {
  if constexpr (ACT == kBF16) return __bfloat16_as_ushort(__float2bfloat16_rn(x));
  else return __half_as_ushort(__float2half_rn(x));
}

// ================================================================ LSE merge
// One warp's share of a log-sum-exp merge: query row `gg` over partial slots
// kb .. ke-1, each (m, l, o~).  Leaves M = max m_k, L = sum 2^(m_k - M) l_k and
// acc = sum 2^(m_k - M) o~_k (d = 4*lane .. 4*lane+3), unnormalised; M = -inf
// for an empty range.  Partials written by other SMs are read through L2
// (ld.global.cg): the (m, l) pairs 32 slots at a time across the lanes, the o~
// rows 32 slots at a time with every load issued before any use.
template <class SlotFn>
__device__ __forceinline__ void merge_row_part(const float* partials, int gg, int kb, int ke,
                                               SlotFn slot_of, int lane, float& M, float& L,
                                               float4& acc) {
  auto ml_of = [&](int k) {
    return partials + static_cast<int64_t>(slot_of(k)) * kPartialSlotFloats + kMaxGroup * kHeadDim +
           2 * gg;
  };
  M = -INFINITY;
  for (int k = kb + lane; k < ke; k += 32) M = fmaxf(M, __ldcg(ml_of(k)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float ref = M == -INFINITY ? 0.f : M;
  constexpr int kInFlight = 32;
  L = 0.f;
  acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = kb; k0 < ke; k0 += kInFlight) {
    const int k = k0 + lane;
    float wk = 0.f;
    if (k < ke) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(ml_of(k)));
      wk = dev::exp2_approx(ml.x - ref);
      L += wk * ml.y;
    }
    const int cnt = min(kInFlight, ke - k0);
    float4 x[kInFlight];
#pragma unroll
    for (int t = 0; t < kInFlight; ++t) {
      if (t < cnt)
        x[t] = __ldcg(reinterpret_cast<const float4*>(
                          partials + static_cast<int64_t>(slot_of(k0 + t)) * kPartialSlotFloats +
                          gg * kHeadDim) + lane);
    }
#pragma unroll
    for (int t = 0; t < kInFlight; ++t) {
      const float wj = __shfl_sync(0xffffffffu, wk, t);
      if (t < cnt) {
        acc.x += wj * x[t].x;
        acc.y += wj * x[t].y;
        acc.z += wj * x[t].z;
        acc.w += wj * x[t].w;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
}

// Query rows of a segment: a plain unit has its item's G query heads of KV
// head h (rows 0 .. G-1); a sibling set has member j's G heads at rows
// j*G .. j*G+G-1.  item_of_row(r) is the item whose output row r is.
template <int G>
__device__ __forceinline__ int unit_rows(const DecodeKParams<DecodePlan>&, const Seg&) { return G; }
template <int G>
__device__ __forceinline__ int unit_rows(const DecodeKParams<SibPlan>& prm, const Seg& s) {
  return (prm.plan.mem0[s.k + 1] - prm.plan.mem0[s.k]) * G;
}
template <int G>
__device__ __forceinline__ int item_of_row(const DecodeKParams<DecodePlan>&, const Seg& s, int) {
  return s.i;
}
template <int G>
__device__ __forceinline__ int item_of_row(const DecodeKParams<SibPlan>& prm, const Seg& s, int r) {
  return prm.plan.mem[prm.plan.mem0[s.k] + r / G];
}
// Element offset of (row r, d = 0) in q / out.
template <int G, class Prm>
__device__ __forceinline__ int64_t row_offset(const Prm& prm, const Seg& s, int r) {
  return item_of_row<G>(prm, s, r) * prm.q_item_stride + (s.h * G + r % G) * kHeadDim;
}

// One warp merges query rows 0 .. rows-1 (rows <= R) of one unit over
// `nslots` partial slots (m_k, l_k, o~_k) in two passes:
//   M = max_k m_k (lanes split the slots, butterfly max), then in slot order
//   w_k = 2^(m_k - M'), L = sum w_k l_k, acc = sum w_k o~_k  (M' = M, or 0 for
//   a row that no token of any slot reached),
// and writes acc / L.  With a fixed reference the slots' terms are
// independent, and every row is computed (rows past `rows` hold no data and
// are not written), so the rows' chains interleave.  The arithmetic depends
// only on the slot order, never on how many slots are in flight, so this and
// merge_unit_warp_staged agree bit for bit.
// Each lane owns d = 4*lane .. 4*lane+3 of every row and reads the (m, l)
// pairs itself (same address in all lanes: one broadcast transaction).
// out_of(r) = element offset of output row r.
template <int R, class SlotFn>
__device__ __forceinline__ void merge_max_pass(const float* partials, int nslots, SlotFn slot_of, int lane,
                                               float (&M)[R]) {
#pragma unroll
  for (int gg = 0; gg < R; ++gg) M[gg] = -INFINITY;
  for (int k = lane; k < nslots; k += 32) {
    const float* ml = partials + static_cast<int64_t>(slot_of(k)) * kPartialSlotFloats + kMaxGroup * kHeadDim;
#pragma unroll
    for (int gg = 0; gg < R; ++gg) M[gg] = fmaxf(M[gg], __ldcg(ml + 2 * gg));
  }
#pragma unroll
  for (int gg = 0; gg < R; ++gg) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M[gg] = fmaxf(M[gg], __shfl_xor_sync(0xffffffffu, M[gg], o));
    if (M[gg] == -INFINITY) M[gg] = 0.f;  // the reference of an empty row
  }
}

// One slot's terms into every row's sums (reference M).
template <int R>
__device__ __forceinline__ void merge_add_slot(const float2 (&ml)[R], const float4 (&x)[R], const float (&M)[R],
                                               float (&L)[R], float4 (&acc)[R]) {
#pragma unroll
  for (int gg = 0; gg < R; ++gg) {
    const float w = dev::exp2_approx(ml[gg].x - M[gg]);
    L[gg] = fmaf(ml[gg].y, w, L[gg]);
    acc[gg].x = fmaf(x[gg].x, w, acc[gg].x);
    acc[gg].y = fmaf(x[gg].y, w, acc[gg].y);
    acc[gg].z = fmaf(x[gg].z, w, acc[gg].z);
    acc[gg].w = fmaf(x[gg].w, w, acc[gg].w);
  }
}

// acc / L of rows < rows to the output; lane r < rows holds row r's offset.
template <int ACT, int R>
__device__ __forceinline__ void merge_write(uint16_t* out, int rows, int64_t out_lane, const float (&L)[R],
                                            const float4 (&acc)[R], int lane) {
#pragma unroll
  for (int gg = 0; gg < R; ++gg) {
    const int64_t off = __shfl_sync(0xffffffffu, out_lane, gg);
    if (gg < rows) {
      const float inv = 1.f / L[gg];
      const uint32_t a = static_cast<uint32_t>(f32_to_act<ACT>(acc[gg].x * inv)) |
                         (static_cast<uint32_t>(f32_to_act<ACT>(acc[gg].y * inv)) << 16);
      const uint32_t b = static_cast<uint32_t>(f32_to_act<ACT>(acc[gg].z * inv)) |
                         (static_cast<uint32_t>(f32_to_act<ACT>(acc[gg].w * inv)) << 16);
      *reinterpret_cast<uint2*>(out + off + 4 * lane) = make_uint2(a, b);
    }
  }
}

// Slots are read a few at a time, every load of a batch issued before any use.
template <int ACT, int R, class SlotFn, class OutFn>
__device__ __forceinline__ void merge_unit_warp(const float* partials, uint16_t* out, int nslots,
                                                int rows, SlotFn slot_of, OutFn out_of, int lane) {
  constexpr int kBatch = R >= 8 ? 2 : (R >= 4 ? 3 : 4);  // loads in flight within the register budget
  const int64_t out_lane = lane < rows ? out_of(lane) : 0;
  float M[R], L[R];
  float4 acc[R];
  merge_max_pass<R>(partials, nslots, slot_of, lane, M);
#pragma unroll
  for (int gg = 0; gg < R; ++gg) {
    L[gg] = 0.f;
    acc[gg] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int k0 = 0; k0 < nslots; k0 += kBatch) {
    float2 ml[kBatch][R];
    float4 x[kBatch][R];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (k0 + j < nslots) {
        const float* slot = partials + static_cast<int64_t>(slot_of(k0 + j)) * kPartialSlotFloats;
#pragma unroll
        for (int gg = 0; gg < R; ++gg) {
          ml[j][gg] = __ldcg(reinterpret_cast<const float2*>(slot + kMaxGroup * kHeadDim) + gg);
          x[j][gg] = __ldcg(reinterpret_cast<const float4*>(slot + gg * kHeadDim) + lane);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (k0 + j < nslots) merge_add_slot<R>(ml[j], x[j], M, L, acc);
  }
  merge_write<ACT, R>(out, rows, out_lane, L, acc, lane);
}

__device__ __forceinline__ int atom_add_acq_rel(int32_t* p, int32_t v) {
  int32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Shared memory a merging warp may stage partial slots in: a worker's copy
// ring once no copy of its own is in flight.  slots = 0: merge from registers.
struct MergeStage {
  uint8_t* ptr;
  uint32_t addr;      // shared-state address of ptr
  int slots;          // whole partial slots that fit
  uint32_t bar;       // an mbarrier of this warp for the staging copies
  uint32_t* phase;    // its phase count
};

constexpr uint32_t kSlotBytes = sizeof(float) * kPartialSlotFloats;

// merge_unit_warp with the slots brought into shared memory by bulk copies,
// stage.slots at a time (one copy per slot, all in flight together, the first
// round's copies overlapping the maximum pass), so a merge of n slots takes
// ceil(n / stage.slots) round trips to L2 instead of one per two slots.  Same
// arithmetic, same slot order, so the same result bit for bit.  False if a
// copy wait gave up (nothing was written).
template <int ACT, int R, class SlotFn, class OutFn>
__device__ __forceinline__ bool merge_unit_warp_staged(const float* partials, uint16_t* out, int nslots,
                                                       int rows, SlotFn slot_of, OutFn out_of, int lane,
                                                       const MergeStage& st) {
  const int64_t out_lane = lane < rows ? out_of(lane) : 0;
  // the arrivals' acquire comes before the copies' reads; the ring's last
  // reads come before the copies' writes
  dev::fence_proxy_async_global();
  dev::fence_proxy_async_smem();
  auto issue = [&](int k0) {
    const int cnt = min(st.slots, nslots - k0);
    if (lane == 0) dev::mbar_arrive_expect_tx(st.bar, cnt * kSlotBytes);
    __syncwarp();
    if (lane < cnt)
      dev::bulk_load(st.addr + lane * kSlotBytes,
                     partials + static_cast<int64_t>(slot_of(k0 + lane)) * kPartialSlotFloats, kSlotBytes, st.bar);
  };
  issue(0);
  float M[R], L[R];
  float4 acc[R];
  merge_max_pass<R>(partials, nslots, slot_of, lane, M);
#pragma unroll
  for (int gg = 0; gg < R; ++gg) {
    L[gg] = 0.f;
    acc[gg] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int k0 = 0; k0 < nslots; k0 += st.slots) {
    if (k0 > 0) issue(k0);
    const int cnt = min(st.slots, nslots - k0);
    const bool ok = dev::mbar_wait_bounded(st.bar, *st.phase & 1u, kWaitLimit);
    if (!__all_sync(0xffffffffu, ok)) {
      // let the copies land before the ring can be reused or released
      dev::mbar_wait_bounded(st.bar, *st.phase & 1u, kWaitLimit);
      ++*st.phase;
      return false;
    }
    ++*st.phase;
    for (int j = 0; j < cnt; ++j) {
      const float* slot = reinterpret_cast<const float*>(st.ptr + j * kSlotBytes);
      float2 ml[R];
      float4 x[R];
#pragma unroll
      for (int gg = 0; gg < R; ++gg) {
        ml[gg] = *reinterpret_cast<const float2*>(slot + kMaxGroup * kHeadDim + 2 * gg);
        x[gg] = *reinterpret_cast<const float4*>(slot + gg * kHeadDim + 4 * lane);
      }
      merge_add_slot<R>(ml, x, M, L, acc);
    }
    __syncwarp();  // every lane is done with the stage before it is refilled
    dev::fence_proxy_async_smem();
  }
  merge_write<ACT, R>(out, rows, out_lane, L, acc, lane);
  return true;
}

// Stream-K: after a worker wrote the partial of a cut unit, it counts itself
// in; the last of the unit's workers merges all of them into the output and
// re-arms the counter.  (Counter = the unit's first worker, unique per cut
// unit.)  R = row capacity of the merge (rows <= R).  With stage.slots > 0
// the merge stages the slots in shared memory (merge_unit_warp_staged).
template <int ACT, int G, int R, class Prm>
__device__ __forceinline__ void settle_partial(const Prm& prm, const Seg& s, int rows, int lane,
                                               const MergeStage& stage = MergeStage{nullptr, 0, 0, 0, nullptr}) {
  const auto& P = prm.plan;
  if (plan_mode(P) != kSplitStreamK) return;  // fixed partitions: a separate reduce kernel merges
  const int W = P.workers;
  // the unit's blocks: positions [u0, u1) (after its alpha cost positions)
  const int64_t u0 = static_cast<int64_t>(s.h) * P.per_head + P.pre[s.k] + P.alpha;
  const int64_t u1 = static_cast<int64_t>(s.h) * P.per_head + P.pre[s.k + 1];
  const int wa = find_worker(prm.total, W, u0);
  const int wb = find_worker(prm.total, W, u1 - 1);
  const int nslots = wb - wa + 1;
  // __syncwarp orders the other lanes' partial writes before lane 0's
  // release; the acquire half orders the merge's reads after the arrivals.
  __syncwarp();
  int old = 0;
  if (lane == 0) old = atom_add_acq_rel(prm.counters + wa, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old != nslots - 1) return;
  __syncwarp();
  // wa's piece starts inside the blocks (slot 2wa) only if its share does
  const bool a_inside = worker_start(prm.total, wa, W) > u0;
  auto slot_of = [&](int q) {
    const int wk = wa + q;
    return (q == 0 && !a_inside) ? 2 * wk + 1 : 2 * wk;
  };
  auto out_of = [&](int r) { return row_offset<G>(prm, s, r); };
  uint16_t* out = reinterpret_cast<uint16_t*>(prm.out);
  if (stage.slots > 0) {
    if (!merge_unit_warp_staged<ACT, R>(prm.partials, out, nslots, rows, slot_of, out_of, lane, stage) &&
        lane == 0)
      atomicOr(prm.err, kErrTimeout);
  } else {
    merge_unit_warp<ACT, R>(prm.partials, out, nslots, rows, slot_of, out_of, lane);
  }
  // every arrival is in: re-arm the counter for the next launch (no reply needed)
  if (lane == 0) asm volatile("st.relaxed.gpu.global.s32 [%0], 0;" ::"l"(prm.counters + wa) : "memory");
}


// Launch parameters of one decode launch from the pool, its plan and the call.
template <class PlanT>
void fill_decode_params(DecodeKParams<PlanT>& prm, const PoolView& pool, const PlanT& plan,
                 const DecodeArgs& args) {
  prm.q = static_cast<const uint8_t*>(args.q);
  prm.out = static_cast<uint8_t*>(args.out);
  prm.tables = pool.tables;
  prm.partials = pool.partials;
  prm.counters = pool.counters;
  prm.err = pool.err;
  prm.k_scale = pool.k_scale;
  prm.v_scale = pool.v_scale;
  prm.q_item_stride = args.q_item_stride;
  prm.scale = args.scale;
  prm.layer = args.layer;
  prm.num_kv_heads = pool.num_kv_heads;
  prm.num_blocks = pool.num_blocks;
  prm.mbps = pool.mbps;
  prm.bshift = pool.block_size == 32 ? 1 : 0;
  prm.group = args.group;
  prm.total = plan.per_head * pool.num_kv_heads;
  std::memcpy(&prm.plan, &plan, sizeof(PlanT));
  // q / out of this launch start at item_offset
  prm.q += static_cast<int64_t>(args.item_offset) * args.q_item_stride * 2;
  prm.out += static_cast<int64_t>(args.item_offset) * args.q_item_stride * 2;
  // fused append: new rows [n][H][128] act dtype, from item_offset on
  const int64_t kv_off = static_cast<int64_t>(args.item_offset) * pool.num_kv_heads * kHeadDim * 2;
  prm.k_new = args.k_new ? static_cast<const uint8_t*>(args.k_new) + kv_off : nullptr;
  prm.v_new = args.v_new ? static_cast<const uint8_t*>(args.v_new) + kv_off : nullptr;
  prm.k_cache = static_cast<uint8_t*>(pool.k_cache);
  prm.v_cache = static_cast<uint8_t*>(pool.v_cache);
  prm.k_inv = pool.k_inv;
  prm.v_inv = pool.v_inv;
}

