// prefill_pair.cuh -- SSA prefill for d_qk <= 128: two query blocks per work
// item sharing their key/value tiles, two softmax warpgroups ping-ponging on
// one tensor core.
//
// A work item is the pair of adjacent query blocks (2p, 2p+1) of one
// (sequence, head).  Their SSA windows (QbitAI article on LongCat LoZA,
// paragraph on the 1024-token sparse window) overlap in all but one block:
// with one sink block and seven local blocks, 2p sees {0, 2p-6..2p} and 2p+1
// sees {0, 2p-5..2p+1}, so the pair reads the union -- 9 key/value tiles --
// once, instead of 16 tiles for the two blocks separately.  That halves the
// L2->SM traffic that bounds the single-block kernel.
//
// Streams: A = query block 2p, B = query block 2p+1 (absent when 2p+1 is past
// the end of the sequence).  For every union tile u in ascending order the MMA
// warp issues, per stream that contains u:
//     O_X += P_X(prev) V(prev)   (the stream's previous tile; P_X overwrote S_X)
//     S_X  = Q_X K(u)^T
// so while warpgroup A computes softmax(S_A), the tensor core works on stream
// B, and vice versa.  Each warpgroup owns whole rows of its stream (thread r =
// query row r = TMEM lane r of its S/O buffers): online softmax with a lazily
// moved running max exactly as in the single-block kernel (prefill.cuh).
//
// Warp roles (320 threads): warps 0-3 stream A softmax/epilogue, warps 4-7
// stream B, warp 8 the TMA producers (lane 0 issues Q and K, lane 1 issues V,
// so a K load never queues behind a V load waiting for its ring slot), warp 9
// TMEM allocator + MMA issuer.
// TMEM: S_A [0,128) S_B [128,256) O_A [256, 256+DV) O_B [256+DV, 256+2DV).
// Shared memory: Q_A Q_B, K ring, V ring (128B-swizzled TMA boxes).
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "prefill.cuh"
#include "ptx.cuh"
#include "schedule.cuh"

namespace loza {

// The pair's union of key tiles, enumerated in ascending block order with a
// flag per stream.  Every role walks it the same way.
struct PairTiles {
  TileRange a, b;
  bool has_b;
  int ia, ib;  // cursors into the two lists
  __device__ __forceinline__ void init(int qa, int n_sink, int n_local, bool with_b) {
    a = tile_range(qa, n_sink, n_local);
    has_b = with_b;
    b = tile_range(qa + 1, n_sink, n_local);
    if (!with_b) b.count = 0;
    ia = ib = 0;
  }
  __device__ __forceinline__ int count() const {
    // |A u B|: B's list is A's list with the diagonal added and possibly the
    // oldest local block removed; count by merging the two ranges.
    int n = 0;
    int x = 0, y = 0;
    while (x < a.count || y < b.count) {
      const int ba = x < a.count ? tile_block(a, x) : 0x7fffffff;
      const int bb = y < b.count ? tile_block(b, y) : 0x7fffffff;
      if (ba <= bb) ++x;
      if (bb <= ba) ++y;
      ++n;
    }
    return n;
  }
  // Next union tile: its key block, and whether stream A / B use it.
  __device__ __forceinline__ int next(bool& in_a, bool& in_b) {
    const int ba = ia < a.count ? tile_block(a, ia) : 0x7fffffff;
    const int bb = ib < b.count ? tile_block(b, ib) : 0x7fffffff;
    in_a = ba <= bb;
    in_b = bb <= ba;
    if (in_a) ++ia;
    if (in_b) ++ib;
    return in_a ? ba : bb;
  }
};

struct PairItem {
  int z, seq_start, len;
  int qa;      // query block of stream A (even)
  bool has_b;  // query block qa+1 exists
};

// Work items: pairs of query blocks.  Dense: (b*H + h) * npair + pair.
// Packed: per sequence H * ceil(nb_s/2) items, found through the prefix.
__device__ __forceinline__ PairItem decode_pair(int item, const PrefillParams& p,
                                                const int* prefix) {
  PairItem w;
  int nb, r;
  if (p.cu_seqlens == nullptr) {
    nb = (p.L + 127) >> 7;
    const int np = (nb + 1) >> 1;
    w.z = item / np;
    r = item - w.z * np;
    w.seq_start = 0;
    w.len = p.L;
  } else {
    int lo = 0, hi = p.n_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int start = __ldg(p.cu_seqlens + lo);
    const int len = __ldg(p.cu_seqlens + lo + 1) - start;
    nb = (len + 127) >> 7;
    const int np = (nb + 1) >> 1;
    const int rr = item - prefix[lo];
    w.z = rr / np;
    r = rr - w.z * np;
    w.seq_start = start;
    w.len = len;
  }
  w.qa = 2 * r;
  w.has_b = w.qa + 1 < nb;
  return w;
}

// Warp 0: pair-item count / packed prefix (H * ceil(ceil(len/128)/2) per sequence).
__device__ __forceinline__ void pair_count_items(const PrefillParams& p, int* prefix,
                                                 uint32_t* misc, int lane) {
  if (p.cu_seqlens == nullptr) {
    if (lane == 0) misc[2] = (uint32_t)p.total_items;
    return;
  }
  const int n = p.n_seqs;
  const int per = (n + 31) / 32;
  const int s0 = min(lane * per, n), s1 = min(s0 + per, n);
  auto items_of = [&](int s) {
    const int len = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
    return p.H * ((((len + 127) >> 7) + 1) >> 1);
  };
  int local = 0, bad = 0;
  for (int s = s0; s < s1; ++s) {
    if (__ldg(p.cu_seqlens + s + 1) < __ldg(p.cu_seqlens + s)) bad = 1;
    else local += items_of(s);
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  int run = incl - local;
  for (int s = s0; s < s1; ++s) {
    prefix[s] = run;
    if (__ldg(p.cu_seqlens + s + 1) >= __ldg(p.cu_seqlens + s)) run += items_of(s);
  }
  if (lane == 0 && (__ldg(p.cu_seqlens) != 0 || __ldg(p.cu_seqlens + n) != p.plane_rows)) bad = 1;
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    prefix[n] = total;
    misc[2] = bad ? 0u : (uint32_t)total;
    if (bad) atomicOr(&g_loza_status, 8);
  }
}

template <int DQK, int DV>
struct PairLayout {
  static constexpr int KCH = DQK / 64;
  static constexpr int VCH = DV / 64;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int Q_BYTES = KCH * CHUNK;  // one query block
  static constexpr int K_BYTES = KCH * CHUNK;
  static constexpr int V_BYTES = VCH * CHUNK;
  static constexpr int KST = 2, VST = 2;
  static constexpr int OFF_Q = 0;  // Q_A then Q_B
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * V_BYTES;
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1;
  static constexpr int B_K_FULL = 2, B_K_EMPTY = B_K_FULL + KST;
  static constexpr int B_V_FULL = B_K_EMPTY + KST, B_V_EMPTY = B_V_FULL + VST;
  static constexpr int B_S_FULL = B_V_EMPTY + VST;  // [2] per stream
  static constexpr int B_P_FULL = B_S_FULL + 2;     // [2]
  static constexpr int B_O_DONE = B_P_FULL + 2;     // [2]
  static constexpr int B_O_EMPTY = B_O_DONE + 2;    // [2]
  static constexpr int B_DRAIN = B_O_EMPTY + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + 256;
  static constexpr int OFF_PREFIX = OFF_MISC + 16;
  static_assert(NBAR * 8 <= 256, "barrier area");
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_O = 256;
  static constexpr int MIN_SMEM = 120 * 1024;
  static constexpr size_t smem_bytes(int n_prefix) {
    size_t need = (size_t)OFF_PREFIX + 4 * (size_t)n_prefix + 1024;
    return need < (size_t)MIN_SMEM ? (size_t)MIN_SMEM : need;
  }
};

constexpr int kPairThreads = 320;

template <int DQK, int DV>
__global__ void __launch_bounds__(kPairThreads, 1)
    ssa_prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using Lay = PairLayout<DQK, DV>;
  static_assert(256 + 2 * DV <= 512, "two O accumulators must fit in TMEM");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* prefix = reinterpret_cast<int*>(smem + Lay::OFF_PREFIX);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::OFF_BAR + 8 * i; };
  int* status = &g_loza_status;

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_Q_FULL), 1);
    mbar_init(bar(Lay::B_Q_EMPTY), 1);
    for (int s = 0; s < Lay::KST; ++s) {
      mbar_init(bar(Lay::B_K_FULL + s), 1);
      mbar_init(bar(Lay::B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < Lay::VST; ++s) {
      mbar_init(bar(Lay::B_V_FULL + s), 1);
      mbar_init(bar(Lay::B_V_EMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(Lay::B_S_FULL + x), 1);
      mbar_init(bar(Lay::B_P_FULL + x), 128);
      mbar_init(bar(Lay::B_O_DONE + x), 1);
      mbar_init(bar(Lay::B_O_EMPTY + x), 128);
    }
    mbar_init(bar(Lay::B_DRAIN), 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 0) pair_count_items(p, prefix, misc, lane);
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 9) {
    tmem_alloc(sb + Lay::OFF_MISC, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int total_items = (int)misc[2];

  if (warp == 8) {
    // ------------------------------------------------------- Q / K producer
    if (lane == 0) {
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const PairItem w = decode_pair(item, p, prefix);
        if (it > 0 && !mbar_wait(bar(Lay::B_Q_EMPTY), (it - 1) & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        // both query blocks in one transaction (block qa+1 past the end of the
        // plane is zero-filled; past the end of a packed sequence it is never stored)
        mbar_arrive_expect_tx(bar(Lay::B_Q_FULL), 2 * Lay::Q_BYTES);
#pragma unroll
        for (int x = 0; x < 2; ++x)
#pragma unroll
          for (int c = 0; c < Lay::KCH; ++c)
            tma_load_3d(sb + Lay::OFF_Q + x * Lay::Q_BYTES + c * Lay::CHUNK, &tm_q,
                        bar(Lay::B_Q_FULL), c * 64, w.seq_start + (w.qa + x) * 128, w.z);
        const int ahead = item + (int)gridDim.x;
        if (ahead < total_items) {
          const PairItem wn = decode_pair(ahead, p, prefix);
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int c = 0; c < Lay::KCH; ++c)
              tma_prefetch_3d(&tm_q, c * 64, wn.seq_start + (wn.qa + x) * 128, wn.z);
        }
        PairTiles pt;
        pt.init(w.qa, p.n_sink, p.n_local, w.has_b);
        const int nu = pt.count();
        for (int u = 0; u < nu; ++u, ++g) {
          bool ia, ib;
          const int row = w.seq_start + pt.next(ia, ib) * 128;
          const int st = g % Lay::KST, use = g / Lay::KST;
          if (use > 0 &&
              !mbar_wait(bar(Lay::B_K_EMPTY + st), (use - 1) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(Lay::B_K_FULL + st), Lay::K_BYTES);
#pragma unroll
          for (int c = 0; c < Lay::KCH; ++c)
            tma_load_3d(sb + Lay::OFF_K + st * Lay::K_BYTES + c * Lay::CHUNK, &tm_k,
                        bar(Lay::B_K_FULL + st), c * 64, row, w.z);
        }
      }
      if (!ok) {
        drain_ring(bar(Lay::B_K_FULL), Lay::KST, g);
        if (it > 0) mbar_wait_drain(bar(Lay::B_Q_FULL), (it - 1) & 1);
      }
    }
  }
  if (warp == 8) {
    // ----------------------------------------------------------- V producer
    if (lane == 1) {
      int g = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const PairItem w = decode_pair(item, p, prefix);
        PairTiles pt;
        pt.init(w.qa, p.n_sink, p.n_local, w.has_b);
        const int nu = pt.count();
        for (int u = 0; u < nu; ++u, ++g) {
          bool ia, ib;
          const int row = w.seq_start + pt.next(ia, ib) * 128;
          const int st = g % Lay::VST, use = g / Lay::VST;
          if (use > 0 &&
              !mbar_wait(bar(Lay::B_V_EMPTY + st), (use - 1) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(Lay::B_V_FULL + st), Lay::V_BYTES);
#pragma unroll
          for (int c = 0; c < Lay::VCH; ++c)
            tma_load_3d(sb + Lay::OFF_V + st * Lay::V_BYTES + c * Lay::CHUNK, &tm_v,
                        bar(Lay::B_V_FULL + st), c * 64, row, w.z);
        }
      }
      if (!ok)
        drain_ring(bar(Lay::B_V_FULL), Lay::VST, g);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, false);
      const uint32_t id_o = idesc_bf16_f32(128, DV, true);
      int g0 = 0, it = 0;
      int sx_a = 0, sx_b = 0;  // tiles each stream has started (global count)
      // readers left of V(g) (1 or 2 streams), one byte per g % 4: a stream's
      // pending tile is never more than two union steps old
      uint32_t vrem = 0;
      bool ok = true;
      // O_X += P_X V(gv), for the stream's tile number n (global count);
      // `first` = the stream's first tile of this item.  The V slot is released
      // after its last reader's P.V.
      auto issue_pv = [&](int x, int n, int gv, bool first) -> bool {
        const int st = gv % Lay::VST;
        if (!mbar_wait(bar(Lay::B_P_FULL + x), n & 1, abort_flag, status, 1)) return false;
        if (!mbar_wait(bar(Lay::B_V_FULL + st), (gv / Lay::VST) & 1, abort_flag, status, 1))
          return false;
        if (first && it > 0 &&
            !mbar_wait(bar(Lay::B_O_EMPTY + x), (it - 1) & 1, abort_flag, status, 1))
          return false;
        tc_fence_after();
        const uint32_t p_tmem = tmem + (uint32_t)(x * 128);
        const uint32_t o_tmem = tmem + Lay::TM_O + x * DV;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sdesc_sw128(
              sb + Lay::OFF_V + st * Lay::V_BYTES + kk * 2048, Lay::CHUNK, 1024);
          mma_ts(o_tmem, p_tmem + kk * 8, bdesc, id_o, (!first || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(Lay::B_O_DONE + x));
        const int sh = (gv & 3) * 8;
        vrem -= 1u << sh;
        if (((vrem >> sh) & 0xffu) == 0) mma_commit(bar(Lay::B_V_EMPTY + st));
        return true;
      };
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const PairItem w = decode_pair(item, p, prefix);
        if (!mbar_wait(bar(Lay::B_Q_FULL), it & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        PairTiles pt;
        pt.init(w.qa, p.n_sink, p.n_local, w.has_b);
        const int nu = pt.count();
        // per stream: tiles started (global), pending tile (global union
        // index, -1 none), and whether that tile is the stream's first of the item
        auto step = [&](int x, int& sx, int& pend, bool& pfirst, bool& started, int g,
                        int st) -> bool {
          if (pend >= 0 && !issue_pv(x, sx - 1, pend, pfirst)) return false;
          tc_fence_after();
          const uint32_t q_base = sb + Lay::OFF_Q + x * Lay::Q_BYTES;
          const uint32_t s_tmem = tmem + (uint32_t)(x * 128);
#pragma unroll
          for (int kk = 0; kk < DQK / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * Lay::CHUNK + (kk & 3) * 32;
            const uint64_t adesc = sdesc_sw128(q_base + koff, 16, 1024);
            const uint64_t bdesc =
                sdesc_sw128(sb + Lay::OFF_K + st * Lay::K_BYTES + koff, 16, 1024);
            mma_ss(s_tmem, adesc, bdesc, id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(Lay::B_S_FULL + x));
          ++sx;
          pend = g;
          pfirst = !started;
          started = true;
          return true;
        };
        int pend_a = -1, pend_b = -1;
        bool first_a = false, first_b = false, started_a = false, started_b = false;
        for (int u = 0; ok && u < nu; ++u) {
          bool in_a, in_b;
          pt.next(in_a, in_b);
          const int g = g0 + u, st = g % Lay::KST;
          if (!mbar_wait(bar(Lay::B_K_FULL + st), (g / Lay::KST) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          const int sh = (g & 3) * 8;
          vrem = (vrem & ~(0xffu << sh)) | ((uint32_t)((in_a ? 1 : 0) + (in_b ? 1 : 0)) << sh);
          if (in_a) ok = step(0, sx_a, pend_a, first_a, started_a, g, st);
          if (ok && in_b) ok = step(1, sx_b, pend_b, first_b, started_b, g, st);
          if (!ok) break;
          mma_commit(bar(Lay::B_K_EMPTY + st));
          if (u == nu - 1) mma_commit(bar(Lay::B_Q_EMPTY));
        }
        if (ok && pend_a >= 0) ok = issue_pv(0, sx_a - 1, pend_a, first_a);
        if (ok && pend_b >= 0) ok = issue_pv(1, sx_b - 1, pend_b, first_b);
        if (!ok) break;
        g0 += nu;
      }
      mma_commit(bar(Lay::B_DRAIN));
      mbar_wait_drain(bar(Lay::B_DRAIN), 0);
    }
  } else {
    // ------------------------------------------ softmax / correction / epilogue
    const int x = warp >> 2;                                      // stream
    const int row = threadIdx.x & 127;                            // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_tmem = tmem + lane_base + (uint32_t)(x * 128);
    const uint32_t o_tmem = tmem + lane_base + Lay::TM_O + x * DV;
    const float sl2 = p.scale_log2;
    int n = 0, it = 0;  // this stream's tiles so far (global), items so far
    for (int item = blockIdx.x; item < total_items; item += gridDim.x, ++it) {
      const PairItem w = decode_pair(item, p, prefix);
      const int qx = w.qa + x;
      if (x == 1 && !w.has_b) {
        // no second block: keep the O-buffer handshake going for the next item
        tc_fence_before();
        mbar_arrive(bar(Lay::B_O_EMPTY + x));
        continue;
      }
      const TileRange tr = tile_range(qx, p.n_sink, p.n_local);
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int t = 0; t < tr.count; ++t, ++n) {
        if (!mbar_wait(bar(Lay::B_S_FULL + x), n & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Diagonal block: key c of the tile is visible to row r iff c <= r
        // (nvis = r + 1 visible keys; a chunk's visibility is one bitmask).
        // Every other tile is unmasked, so the two cases compile separately
        // and the common one carries no per-key selects.
        const bool diag = (t == tr.count - 1);
        const int nvis = row + 1;
        auto chunk_mask = [&](int key0) -> uint32_t {
          const int nk = nvis - key0;
          return nk >= 32 ? 0xffffffffu : (nk <= 0 ? 0u : ((1u << nk) - 1u));
        };
        // Pass 1: row max, 64 columns at a time (ten warps leave a thread 168
        // registers, too few to hold a whole 128-column row alongside the rest).
        auto row_max = [&](auto diag_c) -> float {
          constexpr bool kDiag = decltype(diag_c)::value;
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t v[2][32];
            tmem_ld32(s_tmem + h * 64, v[0]);
            tmem_ld32(s_tmem + h * 64 + 32, v[1]);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t vm = kDiag ? chunk_mask(h * 64 + q * 32) : 0xffffffffu;
#pragma unroll
              for (int c = 0; c < 32; c += 8)
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                  const int k0 = c + 2 * a;
                  float v0 = __uint_as_float(v[q][k0]), v1 = __uint_as_float(v[q][k0 + 1]);
                  if (kDiag) {
                    v0 = ((vm >> k0) & 1u) ? v0 : -INFINITY;
                    v1 = ((vm >> (k0 + 1)) & 1u) ? v1 : -INFINITY;
                  }
                  mx4[a] = fmax3(mx4[a], v0, v1);
                }
            }
          }
          return fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
        };
        const float mx = diag ? row_max(std::true_type{}) : row_max(std::false_type{});
        const float m_tile = mx * sl2;
        const bool first = (t == 0);
        const float m_new = fmaxf(m, m_tile);
        const bool need = !first && (m_new > m + kRescaleThreshold);
        const bool rescale = __any_sync(0xffffffffu, need);
        const float m_use = (first || rescale) ? m_new : m;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        // Pass 2: the row again, 32 keys at a time: p = exp2(s*scale*log2e - m)
        // (masked keys: exp2(-inf) = 0), packed to bf16 pairs.  P words of keys
        // 32c..32c+31 go to columns 16c..16c+15, S columns already read.
        auto exp_pass = [&](auto diag_c) {
          constexpr bool kDiag = decltype(diag_c)::value;
#pragma unroll 1
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t v[32], pk16[16];
            tmem_ld32(s_tmem + ch * 32, v);
            tmem_wait_ld();
            const uint32_t vm = kDiag ? chunk_mask(ch * 32) : 0xffffffffu;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              float v0 = __uint_as_float(v[2 * c]), v1 = __uint_as_float(v[2 * c + 1]);
              if (kDiag) {
                v0 = ((vm >> (2 * c)) & 1u) ? v0 : -INFINITY;
                v1 = ((vm >> (2 * c + 1)) & 1u) ? v1 : -INFINITY;
              }
              float y0, y1, p0, p1;
              f2_unpack(f2_fma(f2_pack(v0, v1), sl2x2, negm2), y0, y1);
              if ((c & 7) < kPolyPairsPer8) {
                exp2_poly_x2(y0, y1, p0, p1);
              } else {
                p0 = ex2_approx(y0);
                p1 = ex2_approx(y1);
              }
              acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
              pk16[c] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_tmem + ch * 16, pk16);
          }
        };
        if (diag) exp_pass(std::true_type{}); else exp_pass(std::false_type{});
        float rsum;
        {
          float a0, a1;
          f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
          rsum = a0 + a1;
        }
        if (!first) {
          // The stream's previous P.V was issued before this S, and the commit
          // that completed S_FULL tracks every earlier tensor-core op of the
          // MMA thread: O already holds that P.V, so it can be rescaled now.
          if (rescale) {
            const float alpha = ex2_approx(m - m_use);
            l *= alpha;
#pragma unroll 1
            for (int ch = 0; ch < DV / 32; ++ch) {
              uint32_t orr[32];
              tmem_ld32(o_tmem + ch * 32, orr);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c)
                orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
              tmem_st32(o_tmem + ch * 32, orr);
            }
          }
        }
        l += rsum;
        m = m_use;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_P_FULL + x));
      }
      if (!ok) break;
      // epilogue: O = acc / l (bf16), LSE = (m + log2 l) ln 2
      if (!mbar_wait(bar(Lay::B_O_DONE + x), (n - 1) & 1, abort_flag, status, 1)) break;
      tc_fence_after();
      const int r_in_seq = qx * 128 + row;
      const bool valid = r_in_seq < w.len;
      const size_t orow = (size_t)w.z * (size_t)p.plane_rows + (size_t)(w.seq_start + r_in_seq);
      const float inv_l = 1.f / l;
#pragma unroll 1
      for (int ch = 0; ch < DV / 32; ++ch) {
        uint32_t orr[32];
        tmem_ld32(o_tmem + ch * 32, orr);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + orow * DV + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t* r8 = &orr[8 * v];
            uint4 pkt;
            pkt.x = pack_bf16x2(__uint_as_float(r8[0]) * inv_l, __uint_as_float(r8[1]) * inv_l);
            pkt.y = pack_bf16x2(__uint_as_float(r8[2]) * inv_l, __uint_as_float(r8[3]) * inv_l);
            pkt.z = pack_bf16x2(__uint_as_float(r8[4]) * inv_l, __uint_as_float(r8[5]) * inv_l);
            pkt.w = pack_bf16x2(__uint_as_float(r8[6]) * inv_l, __uint_as_float(r8[7]) * inv_l);
            dst[v] = pkt;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(Lay::B_O_EMPTY + x));
      if (valid) p.lse[orow] = (m + __log2f(l)) * kLn2;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace loza
