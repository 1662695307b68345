// prefill.cuh -- SSA prefill on sm_100a: TMA + tcgen05 (TMEM accumulators),
// warp-specialised, persistent.
//
// One CTA per SM walks a static stride of work items (sequence, head, 128-row
// query block).  For each item the tile scheduler lists the key blocks of the
// SSA window (sink block(s) first, then the local run, the causal diagonal
// block last).  Per key tile j:
//
//     S_j   = Q K_j^T                       tcgen05.mma, smem x smem -> TMEM (fp32)
//     P_j   = exp2(S_j*scale*log2e - m)     softmax warps: tcgen05.ld, row max,
//                                           exp2, row sum; P (bf16) written back
//                                           into the S columns with tcgen05.st
//     O    += P_j V_j                       tcgen05.mma, TMEM x smem -> TMEM (fp32)
//
// which is the max-subtracted ("CSA/HCA tutorial" §7.1) masked softmax of
// "LoZA：ZigZag稀疏注意力机制" §2.1, computed online over the window's tiles:
// the running max m only moves when a row's new maximum exceeds it by more
// than kRescaleThreshold (log2 units); then the warp rescales its rows of O
// in TMEM by exp2(m_old - m_new) before the next P.V.  The final O = acc / l
// and LSE = (m + log2 l) ln 2 are exact for any choice of m.
//
// Warp roles (512 threads):
//   warps 0-7  softmax + correction + epilogue.  Warp w reads TMEM lanes
//              32*(w%4)..+31 (a warp may only touch its own lane quarter), so
//              query row r is shared by thread r of warpgroup 0 (key columns
//              0-63 of every tile, O columns [0, DV/2)) and thread r of
//              warpgroup 1 (key columns 64-127, O columns [DV/2, DV)); the two
//              halves exchange their row maxima through shared memory once per
//              tile and their row sums once per item.
//   warp 8     TMA producer of Q and K (one elected lane)
//   warp 9     TMEM allocator + issuer of the S = Q K^T MMAs (one elected lane)
//   warp 10    TMA producer of V (one elected lane)
//   warp 11    issuer of the O += P V MMAs (one elected lane)
//   warps 12-15 the epilogue: the softmax warps hand each item's row max and
//              row sums over through shared memory and go straight on to the
//              next item; these warps wait for the item's last P.V, read O
//              from TMEM, normalise it and send it out through swizzled
//              staging boxes and TMA stores (the staging is a buffer of its
//              own for d_qk <= 128, else the V ring slot of the item's last
//              key tile).  The 512 threads launch with 128 registers each and
//              rebalance with setmaxnreg: 152 for the softmax warpgroups, 104
//              for the other two.
// K and V have their own producers so a K load never queues behind a V load
// that is waiting for its ring slot: S consumes K_{j+1} before P.V reads V_j.
// S and P.V have their own issuers because an issuer blocks on its barrier
// waits: with a single issuer the wait for P_j also held back the S MMAs of
// later tiles, so the chain P_j ready -> P_j V_j issued -> S_{j+2} issued sat
// on the softmax's critical path.  (Issue rate itself is not the limit: a
// lone lane starts a 128x128x16 MMA every ~86 SM cycles in a tight loop,
// measured on B200.)
//
// TMEM (512 columns x 128 lanes, fp32): S buffers [0,128), [128,256),
// [256,384), O buffers from 384 (two of them when 2*DV <= 128, so the next
// item's first P.V never waits for this item's epilogue).  P_j (bf16 pairs)
// overwrites the first 64 columns of its S buffer.  With three S buffers the
// tensor core computes S_{j+1} and S_{j+2} while the softmax warps work on
// S_j; S_{j+3} waits until P_j V_j has read buffer j's P.
//
// Shared memory (1024-byte aligned, 128B-swizzled TMA boxes of 64 bf16
// columns x 128 rows = 16 KB "chunks"):  Q ring, K ring, V ring, mbarriers,
// the softmax exchange buffer and, for packed varlen input, the per-sequence
// work-item prefix.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace loza {

constexpr float kRescaleThreshold = 8.0f;  // log2 units: P values stay <= 2^8

// Of every 8 exp2 pairs a softmax thread evaluates, this many run as a
// polynomial on the FMA pipe (exp2_poly_x2) and the rest on the MUFU unit
// (16 exp2 per clock per SM).  Measured on B200 with the mha workload:
// 0 -> 0.566 ms, 1 -> 0.558, 2 -> 0.555, 3 -> 0.565, 4 -> 0.608.
#ifndef LOZA_POLY_PAIRS
#define LOZA_POLY_PAIRS 2
#endif
constexpr int kPolyPairsPer8 = LOZA_POLY_PAIRS;

struct PrefillParams {
  __nv_bfloat16* o;
  float* lse;
  const int* cu_seqlens;  // nullptr: dense [B,H,L,d]; else packed [H,total,d]
  int n_seqs;             // dense: B
  int H;
  int L;                  // dense sequence length
  int plane_rows;         // rows of one TMA plane: dense L, packed total_tokens
  int n_sink;
  int n_local;
  float scale_log2;       // scale * log2(e)
  int total_items;        // dense: B*H*ceil(L/128); packed: computed on the device
};

template <int DQK, int DV>
struct PrefillLayout {
  static constexpr int KCH = DQK / 64;
  static constexpr int VCH = DV / 64;
  static constexpr int CHUNK = 128 * 128;  // one swizzled [128 rows x 64 bf16] box
  static constexpr int Q_BYTES = KCH * CHUNK;
  static constexpr int K_BYTES = KCH * CHUNK;
  static constexpr int V_BYTES = VCH * CHUNK;
  // Q ring depth: one stage measured as fast as two (the S issuer runs ahead of
  // the softmax by two tiles, which covers the next item's Q load)
  static constexpr int QST = DQK <= 64 ? 2 : 1;
  static constexpr int KST = 2;                   // K ring depth
  static constexpr int VST = 2;                   // V ring depth
  static constexpr int NSB = 3;                   // S buffers in TMEM (128 columns each)
  static constexpr int TM_O = NSB * 128;          // O buffers after the S buffers
  static constexpr int NOB = TM_O + 2 * DV <= 512 ? 2 : 1;  // O buffers in TMEM
  static_assert(TM_O + DV <= 512, "S buffers and one O buffer must fit in TMEM");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QST * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * K_BYTES;
  // O goes out through TMA stores from a staging area: a buffer of its own
  // where one fits beside the rings (d_qk <= 128), else the V ring slot of the
  // item's last key tile (d_qk = 192), which that tile's P.V has read by the
  // time O is final and which is handed back to the V producer once the stores
  // have read it (holding a V slot measured slower where a buffer fits).
  static constexpr bool TMA_OUT = true;
  static constexpr bool OWN_STAGE = DQK <= 128;
  static constexpr int OFF_OST = OFF_V + VST * V_BYTES;
  static constexpr int OFF_BAR = OFF_OST + (OWN_STAGE ? VCH * CHUNK : 0);
  // barrier indices
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = B_Q_FULL + QST;
  static constexpr int B_K_FULL = B_Q_EMPTY + QST, B_K_EMPTY = B_K_FULL + KST;
  static constexpr int B_V_FULL = B_K_EMPTY + KST, B_V_EMPTY = B_V_FULL + VST;
  static constexpr int B_S_FULL = B_V_EMPTY + VST;  // NSB
  static constexpr int B_P_FULL = B_S_FULL + NSB;   // NSB
  // NSB: committed after P_j V_j, so it also says "O holds P_j V_j": the
  // softmax waits on it only to rescale O and before the epilogue reads O.
  // A waiter for tile j is never more than one phase behind (S_{j} was issued
  // after P_{j-NSB} V_{j-NSB} finished) nor ahead (P_{j+NSB} is not yet written).
  static constexpr int B_S_FREE = B_P_FULL + NSB;
  static constexpr int B_O_EMPTY = B_S_FREE + NSB;  // NOB
  static constexpr int B_DRAIN = B_O_EMPTY + NOB;   // 2: one per MMA issuer
  // (the two softmax warpgroups' row exchange uses named barriers 1-4, one
  // per pair of warps (w, w + 4) that share TMEM lanes)
  static constexpr int B_OST_FULL = B_DRAIN + 2;    // 2, per warpgroup: box written (128)
  static constexpr int B_OST_FREE = B_OST_FULL + 2; // 2, per warpgroup: box read by its store
  // With an epilogue warpgroup: the softmax warps hand each item's row max
  // and row sums over in shared memory and go on to the next item; warps
  // 12-15 normalise O and store it.
  static constexpr bool EPI_WG = true;
  static constexpr int THREADS = EPI_WG ? 512 : 384;
  static constexpr int B_O_FULL = B_OST_FREE + 2;    // NOB: the item's last P.V done (commit)
  static constexpr int B_ROWS_FULL = B_O_FULL + NOB; // 2: rows published (256)
  static constexpr int B_ROWS_EMPTY = B_ROWS_FULL + 2;  // 2: rows read by the epilogue (128)
  static constexpr int NBAR = EPI_WG ? B_ROWS_EMPTY + 2 : B_OST_FREE + 2;
  static constexpr int BAR_BYTES = EPI_WG ? 512 : 256;
  static constexpr int OFF_MISC = OFF_BAR + BAR_BYTES;  // [0] tmem base, [1] abort, [2] items
  static constexpr int OFF_RED = OFF_MISC + 16;       // float [2 buffers][2 halves][128 rows]
  static constexpr int OFF_ROWS = OFF_RED + 2 * 2 * 128 * 4;  // float [2 items][m, l0, l1][128]
  static constexpr int OFF_PREFIX = OFF_ROWS + (EPI_WG ? 2 * 3 * 128 * 4 : 0);
  static_assert(NBAR * 8 <= BAR_BYTES, "barrier area");
  static constexpr int TMEM_COLS = 512;
  static constexpr int MIN_SMEM = 120 * 1024;  // keeps one CTA (and one TMEM owner) per SM
  // largest prefix (sequences + 1) that fits the 227 KB of shared memory
  static constexpr int MAX_PREFIX = (227 * 1024 - 1024 - OFF_PREFIX) / 4;
  static constexpr size_t smem_bytes(int n_prefix) {
    size_t need = (size_t)OFF_PREFIX + 4 * (size_t)n_prefix + 1024;  // + alignment slack
    return need < (size_t)MIN_SMEM ? (size_t)MIN_SMEM : need;
  }
};

struct WorkItem {
  int z;          // TMA plane: dense b*H + h, packed h
  int seq_start;  // first row of the sequence inside the plane
  int len;        // sequence length
  int qb;         // query block
};

__device__ __forceinline__ WorkItem decode_item(int item, const PrefillParams& p,
                                                const int* prefix) {
  WorkItem w;
  if (p.cu_seqlens == nullptr) {
    const int nb = (p.L + 127) >> 7;
    w.qb = item % nb;
    w.z = item / nb;
    w.seq_start = 0;
    w.len = p.L;
  } else {
    int lo = 0, hi = p.n_seqs - 1;  // largest s with prefix[s] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int start = __ldg(p.cu_seqlens + lo);
    const int len = __ldg(p.cu_seqlens + lo + 1) - start;
    const int nb = (len + 127) >> 7;
    const int r = item - prefix[lo];
    w.z = r / nb;
    w.qb = r - w.z * nb;
    w.seq_start = start;
    w.len = len;
  }
  return w;
}

// Warp 0: work-item count (and, for packed input, the per-sequence prefix of
// H * ceil(len/128) items).  Invalid cu_seqlens -> 0 items + status bit.
__device__ __forceinline__ void prefill_count_items(const PrefillParams& p, int* prefix,
                                                    uint32_t* misc, int lane) {
  if (p.cu_seqlens == nullptr) {
    if (lane == 0) misc[2] = (uint32_t)p.total_items;
    return;
  }
  const int n = p.n_seqs;
  const int per = (n + 31) / 32;
  const int s0 = min(lane * per, n), s1 = min(s0 + per, n);
  int local = 0, bad = 0;
  for (int s = s0; s < s1; ++s) {
    const int a = __ldg(p.cu_seqlens + s), b = __ldg(p.cu_seqlens + s + 1);
    if (b < a) bad = 1;
    local += p.H * ((b - a + 127) >> 7);
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
    run += p.H * ((__ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s) + 127) >> 7);
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

constexpr int kSoftmaxThreads = 256;

template <int DQK, int DV>
__global__ void __launch_bounds__(PrefillLayout<DQK, DV>::THREADS, 1)
    ssa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
  using Lay = PrefillLayout<DQK, DV>;
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
    for (int s = 0; s < Lay::QST; ++s) {
      mbar_init(bar(Lay::B_Q_FULL + s), 1);
      mbar_init(bar(Lay::B_Q_EMPTY + s), 1);
    }
    for (int s = 0; s < Lay::KST; ++s) {
      mbar_init(bar(Lay::B_K_FULL + s), 1);
      mbar_init(bar(Lay::B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < Lay::VST; ++s) {
      mbar_init(bar(Lay::B_V_FULL + s), 1);
      mbar_init(bar(Lay::B_V_EMPTY + s), 1);
    }
    for (int s = 0; s < Lay::NSB; ++s) {
      mbar_init(bar(Lay::B_S_FULL + s), 1);
      mbar_init(bar(Lay::B_P_FULL + s), kSoftmaxThreads);
      mbar_init(bar(Lay::B_S_FREE + s), 1);
    }
    for (int s = 0; s < Lay::NOB; ++s)
      mbar_init(bar(Lay::B_O_EMPTY + s), Lay::EPI_WG ? 128 : kSoftmaxThreads);
    mbar_init(bar(Lay::B_DRAIN), 1);
    mbar_init(bar(Lay::B_DRAIN + 1), 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(Lay::B_OST_FULL + w), kSoftmaxThreads / 2);
      mbar_init(bar(Lay::B_OST_FREE + w), 1);
    }
    if (Lay::EPI_WG) {
      for (int s = 0; s < Lay::NOB; ++s) mbar_init(bar(Lay::B_O_FULL + s), 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(Lay::B_ROWS_FULL + s), kSoftmaxThreads);
        mbar_init(bar(Lay::B_ROWS_EMPTY + s), 128);
      }
    }
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 0) prefill_count_items(p, prefix, misc, lane);
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
  }
  if (warp == 10 && lane == 0) {
    prefetch_tensormap(&tm_v);
    if (Lay::TMA_OUT) prefetch_tensormap(&tm_o);
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
  if constexpr (Lay::EPI_WG) {
    // 512 threads launch with 128 registers each: the softmax warpgroups take
    // 152, the producer / issuer and epilogue warpgroups keep 104
    // (2 x 128 x 152 + 2 x 128 x 104 = 65536, the launch's total)
    if (warp < 8) asm volatile("setmaxnreg.inc.sync.aligned.u32 152;");
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 104;");
  }

  if (warp == 8) {
    // ------------------------------------------------------- Q / K producer
    if (lane == 0) {
      int g = 0, it = 0;
      int q_issued[Lay::QST] = {}, k_issued[Lay::KST] = {};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const WorkItem w = decode_item(item, p, prefix);
        const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
        const int qs = it % Lay::QST;
        if (it >= Lay::QST && !mbar_wait(bar(Lay::B_Q_EMPTY + qs), (it / Lay::QST - 1) & 1,
                                         abort_flag, status, 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(Lay::B_Q_FULL + qs), Lay::Q_BYTES);
        ++q_issued[qs];
#pragma unroll
        for (int c = 0; c < Lay::KCH; ++c)
          tma_load_3d(sb + Lay::OFF_Q + qs * Lay::Q_BYTES + c * Lay::CHUNK, &tm_q,
                      bar(Lay::B_Q_FULL + qs), c * 64, w.seq_start + w.qb * 128, w.z);
        // the item after the ring's reach is first-touch HBM data: start
        // pulling its Q into L2 now
        const int ahead = item + Lay::QST * (int)gridDim.x;
        if (ahead < total_items) {
          const WorkItem wn = decode_item(ahead, p, prefix);
#pragma unroll
          for (int c = 0; c < Lay::KCH; ++c)
            tma_prefetch_3d(&tm_q, c * 64, wn.seq_start + wn.qb * 128, wn.z);
        }
        for (int t = 0; t < tr.count; ++t, ++g) {
          const int row = w.seq_start + tile_block(tr, t) * 128;
          const int st = g % Lay::KST, use = g / Lay::KST;
          if (use > 0 &&
              !mbar_wait(bar(Lay::B_K_EMPTY + st), (use - 1) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(Lay::B_K_FULL + st), Lay::K_BYTES);
          ++k_issued[st];
#pragma unroll
          for (int c = 0; c < Lay::KCH; ++c)
            tma_load_3d(sb + Lay::OFF_K + st * Lay::K_BYTES + c * Lay::CHUNK, &tm_k,
                        bar(Lay::B_K_FULL + st), c * 64, row, w.z);
        }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA's smem goes away:
        // a slot holds at most one unconsumed load, its newest phase.
        for (int s = 0; s < Lay::KST; ++s)
          if (k_issued[s] > 0) mbar_wait_drain(bar(Lay::B_K_FULL + s), (k_issued[s] - 1) & 1);
        for (int s = 0; s < Lay::QST; ++s)
          if (q_issued[s] > 0) mbar_wait_drain(bar(Lay::B_Q_FULL + s), (q_issued[s] - 1) & 1);
      }
    }
  } else if (warp == 10) {
    // ----------------------------------------------------------- V producer
    if (lane == 0) {
      int g = 0;
      int v_issued[Lay::VST] = {};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const WorkItem w = decode_item(item, p, prefix);
        const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
        for (int t = 0; t < tr.count; ++t, ++g) {
          const int row = w.seq_start + tile_block(tr, t) * 128;
          const int st = g % Lay::VST, use = g / Lay::VST;
          if (use > 0 &&
              !mbar_wait(bar(Lay::B_V_EMPTY + st), (use - 1) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(Lay::B_V_FULL + st), Lay::V_BYTES);
          ++v_issued[st];
#pragma unroll
          for (int c = 0; c < Lay::VCH; ++c)
            tma_load_3d(sb + Lay::OFF_V + st * Lay::V_BYTES + c * Lay::CHUNK, &tm_v,
                        bar(Lay::B_V_FULL + st), c * 64, row, w.z);
        }
      }
      if (!ok)
        for (int s = 0; s < Lay::VST; ++s)
          if (v_issued[s] > 0) mbar_wait_drain(bar(Lay::B_V_FULL + s), (v_issued[s] - 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------ MMA issuer: S
    // S and P.V have an issuer each, so a wait for P never holds back S; with
    // three S buffers the S issuer runs up to two tiles ahead of the softmax.
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, false);
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const WorkItem w = decode_item(item, p, prefix);
        const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
        const int qs = it % Lay::QST;
        const uint32_t q_base = sb + Lay::OFF_Q + qs * Lay::Q_BYTES;
        if (!mbar_wait(bar(Lay::B_Q_FULL + qs), (it / Lay::QST) & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        for (int t = 0; t < tr.count; ++t, ++g) {
          const int st = g % Lay::KST, sbuf = g % Lay::NSB;
          // S buffer sbuf last held P_{g-NSB}: wait until its P.V has read it
          if (!mbar_wait(bar(Lay::B_K_FULL + st), (g / Lay::KST) & 1, abort_flag, status, 1) ||
              (g >= Lay::NSB && !mbar_wait(bar(Lay::B_S_FREE + sbuf), (g / Lay::NSB - 1) & 1,
                                           abort_flag, status, 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t s_tmem = tmem + (uint32_t)(sbuf * 128);
#pragma unroll
          for (int kk = 0; kk < DQK / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * Lay::CHUNK + (kk & 3) * 32;
            const uint64_t adesc = sdesc_sw128(q_base + koff, 16, 1024);
            const uint64_t bdesc = sdesc_sw128(sb + Lay::OFF_K + st * Lay::K_BYTES + koff, 16, 1024);
            mma_ss(s_tmem, adesc, bdesc, id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(Lay::B_S_FULL + sbuf));
          mma_commit(bar(Lay::B_K_EMPTY + st));
          if (t == tr.count - 1) mma_commit(bar(Lay::B_Q_EMPTY + qs));
        }
      }
      // every tcgen05.mma issued above has finished before TMEM is released
      mma_commit(bar(Lay::B_DRAIN));
      mbar_wait_drain(bar(Lay::B_DRAIN), 0);
    }
  } else if (warp == 11) {
    // ---------------------------------------------------- MMA issuer: P.V
    if (lane == 0) {
      const uint32_t id_o = idesc_bf16_f32(128, DV, true);
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const WorkItem w = decode_item(item, p, prefix);
        const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
        const int ob = it % Lay::NOB;
        const uint32_t o_tmem = tmem + Lay::TM_O + ob * DV;
        for (int t = 0; t < tr.count; ++t, ++g) {
          // O_ob += P_g V_g
          const int st = g % Lay::VST, sbuf = g % Lay::NSB;
          if (!mbar_wait(bar(Lay::B_P_FULL + sbuf), (g / Lay::NSB) & 1, abort_flag, status, 1) ||
              !mbar_wait(bar(Lay::B_V_FULL + st), (g / Lay::VST) & 1, abort_flag, status, 1) ||
              (t == 0 && it >= Lay::NOB &&
               !mbar_wait(bar(Lay::B_O_EMPTY + ob), (it / Lay::NOB - 1) & 1, abort_flag, status,
                          1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t p_tmem = tmem + (uint32_t)(sbuf * 128);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bdesc = sdesc_sw128(
                sb + Lay::OFF_V + st * Lay::V_BYTES + kk * 2048, Lay::CHUNK, 1024);
            mma_ts(o_tmem, p_tmem + kk * 8, bdesc, id_o, (t > 0 || kk > 0) ? 1u : 0u);
          }
          // without a staging buffer the item's last V slot stages O: the
          // epilogue warpgroup frees it
          if (Lay::OWN_STAGE || t != tr.count - 1) mma_commit(bar(Lay::B_V_EMPTY + st));
          mma_commit(bar(Lay::B_S_FREE + sbuf));
          if (Lay::EPI_WG && t == tr.count - 1) mma_commit(bar(Lay::B_O_FULL + ob));
        }
      }
      mma_commit(bar(Lay::B_DRAIN + 1));
      mbar_wait_drain(bar(Lay::B_DRAIN + 1), 0);
    }
  } else if (Lay::EPI_WG && warp >= 12) {
    // ------------------------------------------------------ epilogue warpgroup
    // Per item: the softmax warps' row max and row sums, then O from TMEM once
    // the item's last P.V is done: O / l as bf16 through the staging boxes and
    // TMA stores (rows past a packed sequence's end through plain stores),
    // LSE = (m + log2 l) ln 2.
    const int row = threadIdx.x - 12 * 32;                        // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float* rows_all = reinterpret_cast<const float*>(smem + Lay::OFF_ROWS);
    int it = 0, n_out = 0, g = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
      const WorkItem w = decode_item(item, p, prefix);
      const int pr = it & 1, ob = it % Lay::NOB;
      g += tile_range(w.qb, p.n_sink, p.n_local).count;
      const int v_slot = (g - 1) % Lay::VST;  // V slot of the item's last tile
      uint8_t* stage = smem + (Lay::OWN_STAGE ? Lay::OFF_OST : Lay::OFF_V + v_slot * Lay::V_BYTES);
      if (!mbar_wait(bar(Lay::B_ROWS_FULL + pr), (it >> 1) & 1, abort_flag, status, 1)) break;
      const float* rows = rows_all + pr * 384;
      const float m = rows[row];
      const float l_row = rows[128 + row] + rows[256 + row];
      mbar_arrive(bar(Lay::B_ROWS_EMPTY + pr));
      if (!mbar_wait(bar(Lay::B_O_FULL + ob), (it / Lay::NOB) & 1, abort_flag, status, 1)) break;
      tc_fence_after();
      const int r_in_seq = w.qb * 128 + row;
      const bool valid = r_in_seq < w.len;
      const size_t orow = (size_t)w.z * (size_t)p.plane_rows + (size_t)(w.seq_start + r_in_seq);
      const float inv_l = 1.f / l_row;
      // dense rows past L fall outside the tensor map and are not written; a
      // packed sequence's last block would spill into the next sequence
      const bool tma_out = p.cu_seqlens == nullptr || (w.qb + 1) * 128 <= w.len;
      // an own staging buffer: the previous store has read it (its issuer checks,
      // then tells the rest)
      if (Lay::OWN_STAGE && tma_out && n_out > 0 &&
          !mbar_wait(bar(Lay::B_OST_FREE), (n_out - 1) & 1, abort_flag, status, 1))
        break;
#pragma unroll 1
      for (int q4 = 0; q4 < 2 * Lay::VCH; ++q4) {  // 32 columns at a time
        uint32_t orr[32];
        tmem_ld32(tmem + lane_base + Lay::TM_O + ob * DV + q4 * 32, orr);
        tmem_wait_ld();
        if (q4 == 2 * Lay::VCH - 1) {
          // O buffer free for the item NOB after this one
          tc_fence_before();
          mbar_arrive(bar(Lay::B_O_EMPTY + ob));
        }
        if (tma_out) {
          // row `row` of box q4/2 in the 128B-swizzled layout the tensor map
          // reads: 16-byte unit j at j ^ (row & 7)
          uint8_t* rowp = stage + (q4 >> 1) * Lay::CHUNK + row * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = (q4 & 1) * 4 + u;
            const uint32_t* r8 = &orr[u * 8];
            *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) =
                make_uint4(pack_bf16x2(__uint_as_float(r8[0]) * inv_l, __uint_as_float(r8[1]) * inv_l),
                           pack_bf16x2(__uint_as_float(r8[2]) * inv_l, __uint_as_float(r8[3]) * inv_l),
                           pack_bf16x2(__uint_as_float(r8[4]) * inv_l, __uint_as_float(r8[5]) * inv_l),
                           pack_bf16x2(__uint_as_float(r8[6]) * inv_l, __uint_as_float(r8[7]) * inv_l));
          }
        } else if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + orow * DV + q4 * 32);
#pragma unroll
          for (int v = 0; v < 4; v += 2) {
            uint32_t w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w8[e] = pack_bf16x2(__uint_as_float(orr[8 * v + 2 * e]) * inv_l,
                                  __uint_as_float(orr[8 * v + 2 * e + 1]) * inv_l);
            st_global_v8(dst + v, w8);
          }
        }
      }
      if (tma_out) {
        fence_async_shared();
        mbar_arrive(bar(Lay::B_OST_FULL));
        if (row == 0) {
          if (!(ok = mbar_wait(bar(Lay::B_OST_FULL), n_out & 1, abort_flag, status, 1))) break;
#pragma unroll
          for (int hh = 0; hh < Lay::VCH; ++hh)
            tma_store_3d(&tm_o, smem_u32(stage) + hh * Lay::CHUNK, hh * 64,
                         w.seq_start + w.qb * 128, w.z);
          tma_store_commit();
          // the staging may be rewritten (own buffer) or refilled by the V
          // producer (V slot) once these stores have read it
          tma_store_wait_read();
          mbar_arrive(bar(Lay::OWN_STAGE ? Lay::B_OST_FREE : Lay::B_V_EMPTY + v_slot));
        }
        ++n_out;
      } else if (!Lay::OWN_STAGE && row == 0) {
        mbar_arrive(bar(Lay::B_V_EMPTY + v_slot));  // nothing staged: the slot is free
      }
      if (valid) p.lse[orow] = (m + __log2f(l_row)) * kLn2;
    }
    if (row == 0) tma_store_wait_all();  // stores done before the CTA exits
  } else {
    // -------------------------------------------- softmax / correction / epilogue
    const int wg = warp >> 2;                                     // column half
    const int row = threadIdx.x & 127;                            // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16; // this warp's lane quarter
    const int col0 = wg * 64;                                     // first key column of the half
    constexpr int OH = DV / 2;                                    // O columns per half
    float* red = reinterpret_cast<float*>(smem + Lay::OFF_RED);
    const float sl2 = p.scale_log2;
    int g0 = 0, it = 0;
    uint32_t xc = 0;  // exchanges done (selects the red buffer)
    // Publish v for this row; the other half's value for the same row comes
    // back in `other`.  Warps w and w + 4 (the same TMEM lanes) meet at named
    // barrier 1 + (w & 3); the buffer alternates, so an exchange never
    // overwrites a value the partner has still to read.  The barrier has no
    // timeout: a thread that leaves the loops early (a failed wait) makes up
    // the exchanges it skipped before it finishes (see the end of this branch).
    auto exchange = [&](float v, float& other) -> bool {
      float* buf = red + (xc & 1) * 256;
      buf[wg * 128 + row] = v;
      named_bar_sync(1 + (warp & 3), 64);
      other = buf[(wg ^ 1) * 128 + row];
      ++xc;
      return true;
    };
    for (int item = blockIdx.x; item < total_items; item += gridDim.x, ++it) {
      const WorkItem w = decode_item(item, p, prefix);
      const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
      const int ob = it % Lay::NOB;
      const uint32_t o_tmem = tmem + lane_base + Lay::TM_O + ob * DV + wg * OH;
      float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
      bool ok = true;
      for (int t = 0; t < tr.count; ++t) {
        const int g = g0 + t;
        const int sbuf = g % Lay::NSB;
        const uint32_t s_tmem = tmem + lane_base + (uint32_t)(sbuf * 128);
        if (!mbar_wait(bar(Lay::B_S_FULL + sbuf), (g / Lay::NSB) & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[2][32];
        tmem_ld32(s_tmem + col0, sr[0]);
        tmem_ld32(s_tmem + col0 + 32, sr[1]);
        tmem_wait_ld();
        if (t == tr.count - 1) {
          // diagonal block: key c of the tile is visible to row r iff c <= r
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (col0 + ch * 32 + c > row) sr[ch][c] = __float_as_uint(-INFINITY);
        }
        // this half's row max: four independent 3-input max chains
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8)
#pragma unroll
          for (int a = 0; a < 4; ++a)
            mx4[a] = fmax3(mx4[a], __uint_as_float(sr[(c + 2 * a) >> 5][(c + 2 * a) & 31]),
                           __uint_as_float(sr[(c + 2 * a + 1) >> 5][(c + 2 * a + 1) & 31]));
        float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
        float mx_other;
        if (!exchange(mx, mx_other)) {
          ok = false;
          break;
        }
        mx = fmaxf(mx, mx_other);
        const float m_tile = mx * sl2;
        const bool first = (t == 0);
        const float m_new = fmaxf(m, m_tile);
        // both halves see the same row maxima, so they take the same decision
        const bool need = !first && (m_new > m + kRescaleThreshold);
        const bool rescale = __any_sync(0xffffffffu, need);
        const float m_use = (first || rescale) ? m_new : m;
        // p = exp2(s*scale*log2e - m): packed FMA for the affine part, four
        // independent packed row-sum accumulators
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const uint64_t xx = f2_pack(__uint_as_float(sr[c >> 4][(2 * c) & 31]),
                                      __uint_as_float(sr[c >> 4][(2 * c + 1) & 31]));
          float y0, y1, p0, p1;
          f2_unpack(f2_fma(xx, sl2x2, negm2), y0, y1);
          if ((c & 7) < kPolyPairsPer8) {
            exp2_poly_x2(y0, y1, p0, p1);
          } else {
            p0 = ex2_approx(y0);
            p1 = ex2_approx(y1);
          }
          acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
        // P (bf16 pairs) over the first 64 columns of the S buffer: keys 2c, 2c+1
        // of this half land in column col0/2 + c
        tmem_st32(s_tmem + col0 / 2, pk);
        float rsum;
        {
          float a0, a1;
          f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
          rsum = a0 + a1;
        }
        if (!first) {
          if (rescale) {
            // O must hold P_{g-1} V_{g-1} before it is rescaled
            const int gp = g - 1;
            if (!mbar_wait(bar(Lay::B_S_FREE + gp % Lay::NSB), (gp / Lay::NSB) & 1, abort_flag,
                           status, 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float alpha = ex2_approx(m - m_use);
            l *= alpha;
#pragma unroll 1
            for (int ch = 0; ch < OH / 32; ++ch) {
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
        mbar_arrive(bar(Lay::B_P_FULL + sbuf));
      }
      if (!ok) break;
      {
        // hand the item's row max and this half's row sums to the epilogue
        // warpgroup (rows buffer it & 1, read back two items ago)
        const int pr = it & 1;
        if (it >= 2 &&
            !mbar_wait(bar(Lay::B_ROWS_EMPTY + pr), ((it >> 1) - 1) & 1, abort_flag, status, 1))
          break;
        float* rows = reinterpret_cast<float*>(smem + Lay::OFF_ROWS) + pr * 384;
        if (wg == 0) rows[row] = m;
        rows[128 + wg * 128 + row] = l;
        mbar_arrive(bar(Lay::B_ROWS_FULL + pr));
      }
      g0 += tr.count;
    }
    // Every softmax thread performs the same number of exchanges -- one per
    // tile of each of this CTA's items -- so that no partner is left at a
    // named barrier: a thread that left the loops early makes up the rest here.
    if (*abort_flag) {
      uint32_t total = 0;
      for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
        const WorkItem w = decode_item(item, p, prefix);
        total += (uint32_t)tile_range(w.qb, p.n_sink, p.n_local).count;
      }
      float unused;
      while (xc < total) exchange(-INFINITY, unused);
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
