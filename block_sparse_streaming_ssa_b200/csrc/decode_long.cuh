// decode_long.cuh -- paged decode over long windows (full-attention layers of
// a ZigZag stack, where a query reads every page of its sequence).
//
// The two-page split kernel (decode.cuh) keeps a split's whole O in tensor
// memory and writes one partial per two pages; over a window of hundreds of
// pages that is hundreds of partial outputs per head group, spilled to DRAM
// and read back by the merge, and the V columns it reloads after S no longer
// hit L2.  This kernel instead streams many pages through one CTA with an
// online softmax and writes one partial per run of pages:
//
//   * CTA pairs.  O over 128 heads x 512 columns in fp32 fills all 512 TMEM
//     columns, leaving none for S.  So two CTAs share a run of pages: CTA h
//     keeps O[:, 256h .. 256h+256) in TMEM columns [256, 512) and both compute
//     the same S = Q K^T (double-buffered in columns [0, 256)) and the same
//     softmax, so their running max and row sum agree without any exchange.
//     The pair reads each page once from DRAM; the second CTA's reads are L2
//     hits.
//   * Stream-K split.  A plan kernel lists the pages of every (row, head
//     group) unit -- its SSA window, or every page up to the query's for a
//     full-attention layer -- as prefix offsets.  Pair k takes pages
//     [k T / P, (k+1) T / P) of the flattened list (T pages, P = min(pairs
//     launched, T) pairs, so that no pair's range is empty), so every pair
//     gets the same number of pages; a pair's range may cross unit
//     boundaries, and each (unit, pair) run is one segment with its own
//     partial, in slot unit + pair of the workspace (the slots of one unit
//     are consecutive and all written).
//   * Per CTA: Q (128 heads x 576, nine 64-column boxes, 147 KB) resident in
//     shared memory for a segment; a ring of five 16 KB slots carries each
//     page's nine K boxes and then, after the next page's K boxes, this half's
//     four V boxes of the previous page again (L2 hits).  MMA order per segment:
//     S(first), then S(f), P(f-1) V(f-1) for every later page, then P(last)
//     V(last); the producer issues its loads in the same order.
//   * Softmax: one warpgroup, one head row per thread, 128 keys per page; the
//     reference max is raised only when a page's max exceeds it by more than
//     2^8 (then O and the row sum are rescaled), so P stays <= 2^8.
//   * Output: at a segment's end the warpgroup writes O / l as fp16 into the
//     same partial layout as the split kernel ([slot][64 column groups][128
//     heads][8]; this CTA's 32 groups) and, in CTA 0 of the pair, the LSE; the
//     split kernel's merge kernel combines a unit's slots.
//
// Warps: 0 TMA producer, 1 MMA issuer (and TMEM allocation), 2-3 idle,
// 4-7 softmax and output.
#pragma once

#include "decode.cuh"

namespace loza {

constexpr int kLongPlanThreads = 1024;
// Pairs are capped so that the workspace bound holds on any device.
constexpr int kLongMaxPairs = 128;
// Windows of more than this many listed pages take the long-window kernel.
constexpr int kLongMinPages = 16;
constexpr float kLongRescaleLog2 = 8.f;
// Pages of a segment the producer pulls into L2 ahead of its ring loads.
constexpr int kLongPrefetch = 3;

struct LongDecodeLayout {
  static constexpr int CHUNK = 128 * 128;      // one box: 128 rows x 64 bf16, 128B swizzle
  static constexpr int KV_CH = kDecodeDqk / 64;  // 9 K boxes per page
  static constexpr int V_CH = 4;                 // V boxes of one half (256 columns)
  // Q boxes 0..NQ-1 stay in shared memory for a segment; boxes NQ..8 would
  // come through the ring again for every page (L2 hits), each right before
  // the K box it multiplies.  All nine resident is fastest: the TMA moves one
  // 16 KB box of 128 rows per SM in about the same time however deep the
  // ring, so every extra load a page costs time (5 resident Q boxes with 9
  // ring slots, 17 loads a page, measured 15-20 % slower than 9 with 5
  // slots, 13 loads a page).
  static constexpr int NQ = 9;
  static constexpr int NSLOT = 5;                // ring slots
  static constexpr int LOADS_PER_PAGE = KV_CH + (KV_CH - NQ) + V_CH;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = NQ * CHUNK;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * CHUNK;
  static constexpr int B_FULL = 0;                  // NSLOT
  static constexpr int B_EMPTY = B_FULL + NSLOT;    // NSLOT
  static constexpr int B_Q_FULL = B_EMPTY + NSLOT;  // a segment's Q landed
  static constexpr int B_Q_EMPTY = B_Q_FULL + 1;    // a segment's S products are done
  static constexpr int B_S_FULL = B_Q_EMPTY + 1;    // 2: S buffer ready
  static constexpr int B_S_FREE = B_S_FULL + 2;     // 2: P V of the buffer's page done
  static constexpr int B_P_READY = B_S_FREE + 2;    // 2: 128 arrivals
  static constexpr int B_O_DONE = B_P_READY + 2;    // one phase per P V product
  static constexpr int B_O_FULL = B_O_DONE + 1;     // one phase per segment: its O is final
  static constexpr int B_O_FREE = B_O_FULL + 1;     // 128 arrivals: a segment's O read
  static constexpr int B_DRAIN = B_O_FREE + 1;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // [0] TMEM base, [1] abort, [2] unit
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_O = 256;
  static constexpr int THREADS = 256;
};
static_assert(LongDecodeLayout::SMEM_BYTES <= 227 * 1024, "long decode layout exceeds smem");

// Pages unit u (row u / HG) lists: its window's, then the chosen pages that
// count (decode_extra_page); 0 for a row whose seq_len is out of range.
__device__ __forceinline__ int long_unit_pages(const DecodeParams& p, int u) {
  DecodeWindow w;
  const int b = u / p.HG;
  return decode_window(p, b, w) ? w.tr.count + decode_extra_count(p, b, w) : 0;
}

// Logical page of listed entry i of row b.
__device__ __forceinline__ int long_listed_page(const DecodeParams& p, int b,
                                                const DecodeWindow& w, int i) {
  return i < w.tr.count ? tile_block(w.tr, i) : decode_extra_page(p, b, w, i - w.tr.count);
}

// The plan: plan[u] = pages listed by units 0..u-1, plan[U] = T, then per
// unit its first partial slot and slot count (for the merge).  One CTA;
// thread t sums a contiguous run of units, a block scan gives the offsets.
__global__ void __launch_bounds__(kLongPlanThreads, 1)
    ssa_decode_plan_kernel(const DecodeParams p, int* plan) {
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ int warp_sum[kLongPlanThreads / 32];
  const int U = p.B * p.HG;
  const int per = (U + kLongPlanThreads - 1) / kLongPlanThreads;
  const int u0 = threadIdx.x * per, u1 = min(U, u0 + per);
  int local = 0;
  for (int u = u0; u < u1; ++u) {
    const int n = long_unit_pages(p, u);
    if (n == 0 && u % p.HG == 0) atomicOr(&g_loza_status, 4);  // seq_len out of range
    local += n;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sum[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, d);
      if (lane >= d) s += y;
    }
    warp_sum[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - local + (warp > 0 ? warp_sum[warp - 1] : 0);
  const long long T = warp_sum[31];
  const int P = long_pairs(p.n_pairs, T);
  int* slots = plan + U + 1;
  for (int u = u0; u < u1; ++u) {
    plan[u] = run;
    const int n = long_unit_pages(p, u);
    long_unit_slot_range(u, run, n, T, P, slots + 2 * u, slots + 2 * u + 1);
    run += n;
  }
  if (threadIdx.x == kLongPlanThreads - 1) plan[U] = run;
}

// One segment of this CTA: unit u (row b, head group hg), listed pages
// [lo, hi) of its window, partial slot `slot`.
struct LongSeg {
  int u, b, hg, lo, hi;
  size_t slot;
  DecodeWindow w;
};

// Walks the segments of pair k's page range [x, x1) in order, starting at
// unit u (the unit holding page x, found once per CTA); every role of the CTA
// walks them the same way.
struct LongWalk {
  const DecodeParams* p;
  long long x, x1;
  int u, k;
  __device__ bool next(LongSeg& s) {
    const int U = p->B * p->HG;
    while (x < x1 && u < U) {
      const long long ou = p->plan[u], ou1 = p->plan[u + 1];
      if (ou1 <= x) {
        ++u;
        continue;
      }
      s.u = u;
      s.b = u / p->HG;
      s.hg = u % p->HG;
      s.lo = (int)(x - ou);
      s.hi = (int)(min(x1, ou1) - ou);
      s.slot = (size_t)u + k;
      decode_window(*p, s.b, s.w);  // true: the unit lists pages
      x = min(x1, ou1);
      ++u;
      return true;
    }
    return false;
  }
};

__global__ void __launch_bounds__(LongDecodeLayout::THREADS, 1)
    ssa_decode_long_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_kv,
                           const __grid_constant__ DecodeParams p) {
  using Lay = LongDecodeLayout;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x >> 1, half = blockIdx.x & 1;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t qreg = sb + Lay::OFF_Q, ring = sb + Lay::OFF_RING;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::OFF_BAR + 8 * i; };
  int* status = &g_loza_status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Lay::NSLOT; ++s) {
      mbar_init(bar(Lay::B_FULL + s), 1);
      mbar_init(bar(Lay::B_EMPTY + s), 1);
    }
    mbar_init(bar(Lay::B_Q_FULL), 1);
    mbar_init(bar(Lay::B_Q_EMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Lay::B_S_FULL + i), 1);
      mbar_init(bar(Lay::B_S_FREE + i), 1);
      mbar_init(bar(Lay::B_P_READY + i), 128);
    }
    mbar_init(bar(Lay::B_O_DONE), 1);
    mbar_init(bar(Lay::B_O_FULL), 1);
    mbar_init(bar(Lay::B_O_FREE), 128);
    mbar_init(bar(Lay::B_DRAIN), 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_kv);
  }
  if (warp == 1) {
    tmem_alloc(sb + Lay::OFF_MISC, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  // The plan is the previous kernel's output.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int U = p.B * p.HG;
  const long long T = p.plan[U];
  const int P = long_pairs(p.n_pairs, T);  // pairs k >= P have no pages
  const long long x0 = k < P ? long_pair_start(k, T, P) : T;
  const long long x1 = k < P ? long_pair_start(k + 1, T, P) : T;
  if (threadIdx.x == 0) {
    // the unit holding page x0: the last u in [0, U) with plan[u] <= x0
    int lo = 0, hi = U - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.plan[mid] <= x0) lo = mid;
      else hi = mid - 1;
    }
    misc[2] = (uint32_t)lo;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const LongWalk walk0{&p, x0, x1, (int)misc[2], k};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      LongWalk wk = walk0;
      LongSeg sg;
      int n_ld = 0, g = 0;
      bool ok = true;
      // With one head group and one token per sequence a page is read by this
      // pair alone (unless the page table maps two sequences to one page); a
      // value box, reloaded after both CTAs' S products read it, is then read
      // for the last time and is marked first to leave L2.  The policy only
      // orders evictions, never what a load returns.
      const bool once = p.HG == 1 && p.q_len == 1;
      const uint64_t pol = l2_policy_evict_first();
      // c >= 0: K box c of physical page phys; c < 0: Q box -c-1 of the segment's row
      auto ring_load = [&](int c, int phys, const LongSeg& s, bool last_read = false) -> bool {
        const int slot = n_ld % Lay::NSLOT, r = n_ld / Lay::NSLOT;
        if (r > 0 && !mbar_wait(bar(Lay::B_EMPTY + slot), (r - 1) & 1, abort_flag, status, 1))
          return false;
        mbar_arrive_expect_tx(bar(Lay::B_FULL + slot), Lay::CHUNK);
        if (c >= 0 && once && last_read)
          tma_load_2d_hint(ring + slot * Lay::CHUNK, &tm_kv, bar(Lay::B_FULL + slot), c * 64,
                           phys * 128, pol);
        else if (c >= 0)
          tma_load_2d(ring + slot * Lay::CHUNK, &tm_kv, bar(Lay::B_FULL + slot), c * 64, phys * 128);
        else
          tma_load_3d(ring + slot * Lay::CHUNK, &tm_q, bar(Lay::B_FULL + slot), (-c - 1) * 64,
                      s.hg * 128, s.b);
        ++n_ld;
        return true;
      };
      auto prefetch_page = [&](int phys) {
        for (int c = 0; c < Lay::KV_CH; ++c) tma_prefetch_2d(&tm_kv, c * 64, phys * 128);
      };
      auto phys_of = [&](const LongSeg& s, int i) -> int {
        const int ph = decode_page(p, s.b, long_listed_page(p, s.b, s.w, i));
        if (ph < 0) atomicOr(status, 2);
        return ph < 0 ? 0 : ph;  // a bad entry reads page 0, fully masked by the softmax
      };
      while (ok && wk.next(sg)) {
        if (g > 0 && !(ok = mbar_wait(bar(Lay::B_Q_EMPTY), (g - 1) & 1, abort_flag, status, 1)))
          break;
        mbar_arrive_expect_tx(bar(Lay::B_Q_FULL), Lay::NQ * Lay::CHUNK);
        for (int c = 0; c < Lay::NQ; ++c)
          tma_load_3d(qreg + c * Lay::CHUNK, &tm_q, bar(Lay::B_Q_FULL), c * 64, sg.hg * 128, sg.b);
        ++g;
        // Pages kLongPrefetch ahead are pulled into L2, so that the ring's
        // loads (five slots, 80 KB in flight) wait for an L2 hit rather than
        // for DRAM.
        for (int i = sg.lo; i < min(sg.hi, sg.lo + kLongPrefetch); ++i)
          prefetch_page(phys_of(sg, i));
        int pf = sg.lo + kLongPrefetch < sg.hi ? phys_of(sg, sg.lo + kLongPrefetch) : -1;
        int prev = -1;
        int cur = phys_of(sg, sg.lo);
        for (int i = sg.lo; i < sg.hi && ok; ++i) {
          // table entries read one page early: in flight meanwhile
          const int nxt = i + 1 < sg.hi ? phys_of(sg, i + 1) : -1;
          const int i_pf = i + kLongPrefetch + 1;
          const int pf_next = i_pf < sg.hi ? phys_of(sg, i_pf) : -1;
          if (pf >= 0) prefetch_page(pf);  // page i + kLongPrefetch
          pf = pf_next;
          for (int c = 0; c < Lay::KV_CH && ok; ++c) {
            if (c >= Lay::NQ) ok = ring_load(-c - 1, 0, sg);
            if (ok) ok = ring_load(c, cur, sg);
          }
          for (int j = 0; j < Lay::V_CH && ok && prev >= 0; ++j)
            ok = ring_load(4 * half + j, prev, sg, true);
          prev = cur;
          cur = nxt;
        }
        for (int j = 0; j < Lay::V_CH && ok; ++j) ok = ring_load(4 * half + j, prev, sg, true);
      }
      // every copy issued lands before the CTA exits
      drain_ring(bar(Lay::B_FULL), Lay::NSLOT, n_ld);
      if (g > 0) mbar_wait_drain(bar(Lay::B_Q_FULL), (g - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, false);
      const uint32_t id_o = idesc_bf16_f32(128, 64, true);
      const uint32_t id_o2 = idesc_bf16_f32(128, 128, true);
      LongWalk wk = walk0;
      LongSeg sg;
      int n_ld = 0, f = 0, g = 0;
      bool ok = true;
      auto s_page = [&](int ff, bool first) -> bool {
        const int b2 = ff & 1;
        if (ff >= 2 && !mbar_wait(bar(Lay::B_S_FREE + b2), ((ff >> 1) - 1) & 1, abort_flag, status, 1))
          return false;
        if (first && !mbar_wait(bar(Lay::B_Q_FULL), g & 1, abort_flag, status, 1)) return false;
        const uint32_t d = tmem + 128 * b2;
        for (int c = 0; c < Lay::KV_CH; ++c) {
          // Q box c: resident, or the ring slot just before the K box
          int q_slot = -1;
          if (c >= Lay::NQ) {
            q_slot = n_ld % Lay::NSLOT;
            if (!mbar_wait(bar(Lay::B_FULL + q_slot), (n_ld / Lay::NSLOT) & 1, abort_flag, status,
                           1))
              return false;
            ++n_ld;
          }
          const int slot = n_ld % Lay::NSLOT;
          if (!mbar_wait(bar(Lay::B_FULL + slot), (n_ld / Lay::NSLOT) & 1, abort_flag, status, 1))
            return false;
          tc_fence_after();
          const uint32_t kb = ring + slot * Lay::CHUNK;
          const uint32_t qb = q_slot >= 0 ? ring + q_slot * Lay::CHUNK : qreg + c * Lay::CHUNK;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(d, sdesc_sw128(qb + kk * 32, 16, 1024), sdesc_sw128(kb + kk * 32, 16, 1024), id_s,
                   (c > 0 || kk > 0) ? 1u : 0u);
          if (q_slot >= 0) mma_commit(bar(Lay::B_EMPTY + q_slot));
          mma_commit(bar(Lay::B_EMPTY + slot));
          ++n_ld;
        }
        mma_commit(bar(Lay::B_S_FULL + b2));
        return true;
      };
      // O[:, 64j ..] (+)= P V_j over the page's 128 keys, 16 at a time: V box j
      // (128 keys x 64 columns) is an MN-major operand; P words of keys
      // 16kk .. 16kk+15 are columns 8kk .. 8kk+7 of the page's S buffer.
      auto pv_page = [&](int ff, bool first) -> bool {
        const int b2 = ff & 1;
        if (!mbar_wait(bar(Lay::B_P_READY + b2), (ff >> 1) & 1, abort_flag, status, 1))
          return false;
        if (first && g > 0 && !mbar_wait(bar(Lay::B_O_FREE), (g - 1) & 1, abort_flag, status, 1))
          return false;
        for (int j = 0; j < Lay::V_CH;) {
          // two value boxes in adjacent ring slots (no wrap-around) are one
          // N = 128 operand, 64-column chunks one slot apart; else one box
          const int slot = n_ld % Lay::NSLOT;
          const bool two_box = j + 1 < Lay::V_CH && slot + 1 < Lay::NSLOT;
          const uint32_t ph = (n_ld / Lay::NSLOT) & 1;  // the same phase for slot + 1
          if (!mbar_wait(bar(Lay::B_FULL + slot), ph, abort_flag, status, 1) ||
              (two_box && !mbar_wait(bar(Lay::B_FULL + slot + 1), ph, abort_flag, status, 1)))
            return false;
          tc_fence_after();
          const uint32_t vb = ring + slot * Lay::CHUNK;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + Lay::TM_O + 64 * j, tmem + 128 * b2 + 8 * kk,
                   sdesc_sw128(vb + kk * 2048, Lay::CHUNK, 1024), two_box ? id_o2 : id_o,
                   (!first || kk > 0) ? 1u : 0u);
          mma_commit(bar(Lay::B_EMPTY + slot));
          if (two_box) mma_commit(bar(Lay::B_EMPTY + slot + 1));
          n_ld += two_box ? 2 : 1;
          j += two_box ? 2 : 1;
        }
        mma_commit(bar(Lay::B_S_FREE + b2));
        mma_commit(bar(Lay::B_O_DONE));
        return true;
      };
      while (ok && wk.next(sg)) {
        const int f0 = f;
        for (int i = sg.lo; i < sg.hi && ok; ++i, ++f) {
          ok = s_page(f, f == f0);
          if (ok && i == sg.hi - 1) mma_commit(bar(Lay::B_Q_EMPTY));  // Q may be replaced
          if (ok && f > f0) ok = pv_page(f - 1, f - 1 == f0);
        }
        if (ok) ok = pv_page(f - 1, f - 1 == f0);
        // a commit covers every earlier product: the segment's O is final
        if (ok) mma_commit(bar(Lay::B_O_FULL));
        ++g;
      }
      mma_commit(bar(Lay::B_DRAIN));
      mbar_wait_drain(bar(Lay::B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------- softmax + output
    const int r = threadIdx.x - 128;  // head row within the group
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    LongWalk wk = walk0;
    LongSeg sg;
    int f = 0, g = 0;
    bool ok = true;
    while (wk.next(sg)) {
      if (!ok) {
        // a wait gave up: this segment's partial is never written
        if (half == 0) p.lse_part[sg.slot * 128 + r] = __int_as_float(0x7fc00000);
        continue;
      }
      float m_ref = -INFINITY;  // reference max of this segment's exponentials (log2 units)
      float l = 0.f;
      for (int i = sg.lo; i < sg.hi; ++i, ++f) {
        const int b2 = f & 1;
        const int logical = long_listed_page(p, sg.b, sg.w, i);
        const int valid_keys = decode_page(p, sg.b, logical) < 0 ? 0
                                                               : decode_valid_keys(sg.w, logical);
        const bool partial = valid_keys < 128;
        if (!(ok = mbar_wait(bar(Lay::B_S_FULL + b2), (f >> 1) & 1, abort_flag, status, 1))) break;
        tc_fence_after();
        const uint32_t s_col = 128 * b2;
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (valid_keys > 0) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t v[2][32];
            tmem_ld32(t_row + s_col + hf * 64, v[0]);
            tmem_ld32(t_row + s_col + hf * 64 + 32, v[1]);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const uint32_t vm = partial ? decode_chunk_mask(valid_keys, 2 * hf + jj) : 0xffffffffu;
#pragma unroll
              for (int c = 0; c < 32; c += 8)
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                  const int k0 = c + 2 * a;
                  const float x0 = ((vm >> k0) & 1u) ? __uint_as_float(v[jj][k0]) : -INFINITY;
                  const float x1 =
                      ((vm >> (k0 + 1)) & 1u) ? __uint_as_float(v[jj][k0 + 1]) : -INFINITY;
                  mx4[a] = fmax3(mx4[a], x0, x1);
                }
            }
          }
        }
        const float m_page = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;
        // raise the reference max only past the threshold (or from -inf)
        const bool raise = m_page > m_ref + kLongRescaleLog2 || (m_ref == -INFINITY && m_page > m_ref);
        float alpha = 1.f;
        if (raise) {
          alpha = ex2_approx(m_ref - m_page);  // 0 from -inf
          m_ref = m_page;
          l *= alpha;
        }
        // O holds earlier pages' products once this segment's first P V is
        // issued.  Wait for P V of the previous page: S(f) being done means
        // every product issued before it, P V of page f-2 included, is done,
        // and P V of page f waits for this thread's P, so the barrier is one
        // phase behind at most.
        if (__any_sync(0xffffffffu, raise) && i > sg.lo) {
          if (!(ok = mbar_wait(bar(Lay::B_O_DONE), (f - 1) & 1, abort_flag, status, 1))) break;
          tc_fence_after();
#pragma unroll 1
          for (int q = 0; q < 8; ++q) {
            uint32_t o[32];
            tmem_ld32(t_row + Lay::TM_O + 32 * q, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(t_row + Lay::TM_O + 32 * q, o);
          }
          tmem_wait_st();
        }
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
        const uint64_t negm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        // p = exp2(s * scale * log2(e) - m_ref), 32 keys at a time (masked keys
        // 0), packed to bf16 pairs over the S columns this thread has read
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32], pk16[16];
          tmem_ld32(t_row + s_col + ch * 32, v);
          tmem_wait_ld();
          const uint32_t vm = partial ? decode_chunk_mask(valid_keys, ch) : 0xffffffffu;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float y0, y1, p0, p1;
            const float v0 = ((vm >> (2 * c)) & 1u) ? __uint_as_float(v[2 * c]) : -INFINITY;
            const float v1 = ((vm >> (2 * c + 1)) & 1u) ? __uint_as_float(v[2 * c + 1]) : -INFINITY;
            f2_unpack(f2_fma(f2_pack(v0, v1), sl2x2, negm2), y0, y1);
            if ((c & 7) < kDecodePolyPairsPer8) {
              exp2_poly_x2(y0, y1, p0, p1);
              // the polynomial clamps its argument, so a masked key would not be 0
              p0 = v0 == -INFINITY ? 0.f : p0;
              p1 = v1 == -INFINITY ? 0.f : p1;
            } else {
              p0 = ex2_approx(y0);
              p1 = ex2_approx(y1);
            }
            acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
            pk16[c] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_row + s_col + ch * 16, pk16);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_P_READY + b2));
        float a0, a1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
        l += a0 + a1;
      }
      if (!ok) {
        if (half == 0) p.lse_part[sg.slot * 128 + r] = __int_as_float(0x7fc00000);
        continue;
      }
      // ---- segment output: O / l over this CTA's 256 columns
      if (!(ok = mbar_wait(bar(Lay::B_O_FULL), g & 1, abort_flag, status, 1))) {
        if (half == 0) p.lse_part[sg.slot * 128 + r] = __int_as_float(0x7fc00000);
        continue;
      }
      ++g;
      tc_fence_after();
      const bool valid = sg.hg * 128 + r < p.H_q;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(p.o_part) + sg.slot * (64 * 128) + r;
#pragma unroll 1
      for (int q = 0; q < 8; ++q) {
        uint32_t o[32];
        tmem_ld32(t_row + Lay::TM_O + 32 * q, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __half2 hv = __floats2half2_rn(__uint_as_float(o[8 * g4 + 2 * e]) * inv_l,
                                             __uint_as_float(o[8 * g4 + 2 * e + 1]) * inv_l);
              w[e] = *reinterpret_cast<uint32_t*>(&hv);
            }
            dst[(size_t)(32 * half + 4 * q + g4) * 128] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(Lay::B_O_FREE));
      if (valid && half == 0)
        p.lse_part[sg.slot * 128 + r] = l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
    }
    asm volatile("griddepcontrol.launch_dependents;");
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace loza
