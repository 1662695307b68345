// backward.cuh -- gradients of the SSA prefill on sm_100a, for (d_qk, d_v) in
// {(64, 64), (128, 128), (192, 128)} (dense and packed layouts).
//
// For a loss with upstream gradient dO = dL/dO, differentiating the masked
// softmax attention of "LoZA：ZigZag稀疏注意力机制" §2.1 over the SSA key sets
// J(i) (QbitAI LoZA article, 1024-token window paragraph) gives, with
// P_ij = exp(s_ij - LSE_i) for j in J(i) and s_ij = scale * q_i . k_j:
//
//     D_i   = sum_c dO_ic O_ic                 (= sum_j P_ij dP_ij)
//     dP_ij = dO_i . v_j
//     dS_ij = P_ij (dP_ij - D_i)
//     dQ_i  = scale sum_j dS_ij k_j
//     dK_j  = scale sum_i dS_ij q_i            (over the i with j in J(i))
//     dV_j  = sum_i P_ij dO_i
//
// Three kernels:
//   ssa_bwd_preprocess_kernel  D_i for every row (CUDA cores; reads O and dO once).
//   ssa_bwd_dq_kernel          per query block: for each key tile of its window
//                              S = Q K^T and dP = dO V^T on tcgen05 into TMEM,
//                              dS in registers, dQ += dS K as a TMEM x smem MMA.
//   ssa_bwd_dkdv_kernel        per key block: for each query block whose window
//                              holds it, S^T = K Q^T and dP^T = V dO^T (TMEM lanes =
//                              keys), P^T and dS^T in registers, then
//                              dV += P^T dO and dK += dS^T Q as TMEM x smem MMAs.
//                              The sink blocks are seen by every later query
//                              block, so their query lists are cut into chunks
//                              of kSinkChunk blocks whose fp32 partial dK / dV
//                              ssa_bwd_sink_reduce_kernel adds up.
// LSE_i = ln sum_j exp(s_ij) comes from the forward pass, so no row max is
// recomputed: P is exact up to rounding and dS goes to the MMAs as bf16.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace loza {

// warps 0-7 compute, 8 TMA producer, 9, 10 and 11 MMA issuers
constexpr int kBwdThreads = 384;
constexpr int kBwdComputeThreads = 256;
constexpr int kSinkChunk = 8;        // query blocks per sink work item

struct BwdParams {
  const float* lse;        // [planes * plane_rows], natural log, from the forward pass
  const float* dsum;       // [planes * plane_rows], D_i
  __nv_bfloat16* dq;       // [planes, plane_rows, d_qk]; dk likewise, dv [.., d_v]
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* part;             // sink partials: [sink slots] x (dK [128][d_qk], dV [128][d_v])
  int L, planes, n_sink, n_local;
  int nb;                  // dense: query / key blocks per plane
  int sink_items;          // dense: sink work items per plane
  float scale, scale_log2;
  // Packed variable-length input (cu_seqlens != nullptr): planes = heads,
  // plane_rows = total tokens, and pfx holds three exclusive prefixes over the
  // sequences, [3][n_seqs + 1]: dQ work items, dK/dV work items and sink
  // partial slots (each counted over all heads).
  const int* cu_seqlens;
  const int* pfx;
  int n_seqs;
  int plane_rows;          // dense: L
};

// Largest s with a[s] <= x, for a non-decreasing a[0..n] with a[0] = 0 <= x.
__device__ __forceinline__ int bwd_find(const int* a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a + mid) <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// A dQ work item: one query block of one (sequence, head).
struct BwdQItem {
  int plane, seq_start, len, qb;
};

__device__ __forceinline__ int bwd_q_items(const BwdParams& p) {
  return p.cu_seqlens == nullptr ? p.planes * p.nb : __ldg(p.pfx + p.n_seqs);
}

__device__ __forceinline__ BwdQItem bwd_q_item(const BwdParams& p, int item) {
  BwdQItem w;
  if (p.cu_seqlens == nullptr) {
    w.plane = item / p.nb;
    w.qb = item - w.plane * p.nb;
    w.seq_start = 0;
    w.len = p.L;
  } else {
    const int s = bwd_find(p.pfx, p.n_seqs, item);
    w.seq_start = __ldg(p.cu_seqlens + s);
    w.len = __ldg(p.cu_seqlens + s + 1) - w.seq_start;
    const int nb = (w.len + 127) >> 7;
    const int r = item - __ldg(p.pfx + s);
    w.plane = r / nb;
    w.qb = r - w.plane * nb;
  }
  return w;
}

// Sink work items of one plane: key block j < min(n_sink, nb) is seen by
// query blocks j .. nb-1, cut into chunks of kSinkChunk.
__host__ __device__ __forceinline__ int bwd_sink_chunks(int j, int nb) {
  return (nb - j + kSinkChunk - 1) / kSinkChunk;
}
__host__ __device__ __forceinline__ int bwd_sink_items(int n_sink, int nb) {
  int n = 0;
  for (int j = 0; j < n_sink && j < nb; ++j) n += bwd_sink_chunks(j, nb);
  return n;
}

// A dK/dV work item: one key block of one (sequence, head) with its query
// blocks q_lo .. q_hi (a sink block's list is cut into chunks).
struct BwdKItem {
  int plane, seq_start, len, kb;
  int q_lo, q_hi;    // query blocks q_lo .. q_hi (inclusive)
  int slot;          // sink partial slot, -1 for a regular key block (written directly)
};

__device__ __forceinline__ int bwd_kv_items(const BwdParams& p) {
  return p.cu_seqlens == nullptr
             ? p.planes * (p.sink_items + (p.nb > p.n_sink ? p.nb - p.n_sink : 0))
             : __ldg(p.pfx + (p.n_seqs + 1) + p.n_seqs);
}

__device__ __forceinline__ BwdKItem bwd_kv_item(const BwdParams& p, int item) {
  BwdKItem w;
  int nb, sink_items, r, slot0;
  if (p.cu_seqlens == nullptr) {
    nb = p.nb;
    sink_items = p.sink_items;
    const int per_plane = sink_items + (nb > p.n_sink ? nb - p.n_sink : 0);
    w.plane = item / per_plane;
    r = item - w.plane * per_plane;
    w.seq_start = 0;
    w.len = p.L;
    slot0 = w.plane * sink_items;
  } else {
    const int* pfx_kv = p.pfx + (p.n_seqs + 1);
    const int* pfx_sink = pfx_kv + (p.n_seqs + 1);
    const int s = bwd_find(pfx_kv, p.n_seqs, item);
    w.seq_start = __ldg(p.cu_seqlens + s);
    w.len = __ldg(p.cu_seqlens + s + 1) - w.seq_start;
    nb = (w.len + 127) >> 7;
    sink_items = bwd_sink_items(p.n_sink, nb);
    const int per_plane = sink_items + (nb > p.n_sink ? nb - p.n_sink : 0);
    r = item - __ldg(pfx_kv + s);
    w.plane = r / per_plane;
    r -= w.plane * per_plane;
    slot0 = __ldg(pfx_sink + s) + w.plane * sink_items;
  }
  if (r < sink_items) {
    w.slot = slot0 + r;
    int j = 0;
    while (r >= bwd_sink_chunks(j, nb)) {
      r -= bwd_sink_chunks(j, nb);
      ++j;
    }
    w.kb = j;
    w.q_lo = j + r * kSinkChunk;
    w.q_hi = min(nb - 1, w.q_lo + kSinkChunk - 1);
  } else {
    w.slot = -1;
    w.kb = p.n_sink + (r - sink_items);
    w.q_lo = w.kb;
    w.q_hi = min(nb - 1, w.kb + p.n_local - 1);
  }
  return w;
}

// Packed input: the three prefixes of BwdParams::pfx from cu_seqlens, one CTA
// of 1024 threads.  Invalid cu_seqlens (not starting at 0, not ending at
// total, decreasing), or more sink slots than the workspace holds, give zero
// work everywhere and set a device status bit.
__global__ void __launch_bounds__(1024) ssa_bwd_varlen_setup_kernel(const int* cu, int n_seqs,
                                                                    int total, int H, int n_sink,
                                                                    long long slot_capacity,
                                                                    int* pfx) {
  __shared__ int warp_tot[3][32];
  __shared__ int bad;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t == 0) bad = (__ldg(cu) != 0 || __ldg(cu + n_seqs) != total) ? 1 : 0;
  __syncthreads();
  const int per = (n_seqs + 1023) / 1024;
  const int s0 = min(t * per, n_seqs), s1 = min(s0 + per, n_seqs);
  int loc[3] = {0, 0, 0};
  for (int s = s0; s < s1; ++s) {
    const int len = __ldg(cu + s + 1) - __ldg(cu + s);
    if (len < 0) bad = 1;
    const int nb = len > 0 ? (len + 127) >> 7 : 0;
    const int si = bwd_sink_items(n_sink, nb);
    loc[0] += H * nb;
    loc[1] += H * (si + (nb > n_sink ? nb - n_sink : 0));
    loc[2] += H * si;
  }
  int inc[3];
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    inc[a] = loc[a];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc[a], off);
      if (lane >= off) inc[a] += v;
    }
    if (lane == 31) warp_tot[a][warp] = inc[a];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      int v = warp_tot[a][lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
      }
      warp_tot[a][lane] = v;  // inclusive over warps
    }
  }
  __syncthreads();
  const bool invalid = bad != 0 || (long long)warp_tot[2][31] > slot_capacity;
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    int run = inc[a] - loc[a] + (warp > 0 ? warp_tot[a][warp - 1] : 0);
    for (int s = s0; s < s1; ++s) {
      pfx[a * (n_seqs + 1) + s] = invalid ? 0 : run;
      const int len = __ldg(cu + s + 1) - __ldg(cu + s);
      const int nb = len > 0 ? (len + 127) >> 7 : 0;
      const int si = bwd_sink_items(n_sink, nb);
      run += a == 0 ? H * nb : a == 1 ? H * (si + (nb > n_sink ? nb - n_sink : 0)) : H * si;
    }
    if (t == 1023) pfx[a * (n_seqs + 1) + n_seqs] = invalid ? 0 : warp_tot[a][31];
  }
  if (t == 0 && invalid) atomicOr(&g_loza_status, 8);
}

// ---------------------------------------------------------------- D_i

// D_i = dO_i . O_i for every row (DIM = d_v); DIM / 8 lanes share a row (16
// bytes each).
template <int DIM>
__global__ void __launch_bounds__(256) ssa_bwd_preprocess_kernel(const __nv_bfloat16* o,
                                                                  const __nv_bfloat16* dout,
                                                                  float* dsum, long long rows) {
  constexpr int LPR = DIM / 8;  // lanes per row
  constexpr int RPW = 32 / LPR;  // rows per warp step
  const int lane = threadIdx.x & 31;
  const long long warp = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r0 = warp * RPW; r0 < rows; r0 += n_warps * RPW) {
    const long long r = r0 + lane / LPR;
    float acc = 0.f;
    if (r < rows) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + r * DIM) + (lane % LPR));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + r * DIM) + (lane % LPR));
      const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* bh = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = __bfloat1622float2(ah[e]), y = __bfloat1622float2(bh[e]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < rows && lane % LPR == 0) dsum[r] = acc;
  }
}

// ------------------------------------------------------------------ dQ

template <int DQK, int DV>
struct BwdDqLayout {
  static constexpr int QCH = DQK / 64, VCH = DV / 64;
  static constexpr int CHUNK = 128 * 128;     // one swizzled [128 rows x 64 bf16] box
  static constexpr int QTILE = QCH * CHUNK;   // [128 rows x d_qk]: Q, K
  static constexpr int VTILE = VCH * CHUNK;   // [128 rows x d_v]: dO, V
  static constexpr int KST = 2;
  // two V stages where they fit in shared memory (not beside the d_qk = 192 tiles)
  static constexpr int VST = 2 * QTILE + 3 * VTILE + KST * QTILE <= 220 * 1024 ? 2 : 1;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = QTILE;
  static constexpr int OFF_K = QTILE + VTILE;
  static constexpr int OFF_V = OFF_K + KST * QTILE;
  static constexpr int OFF_BAR = OFF_V + VST * VTILE;
  // TMEM columns: S, dP, dS (bf16 pairs, 64 columns), dQ (d_qk columns) at the end
  static constexpr int TM_S = 0, TM_DP = 128, TM_DS = 256, TM_DQ = 512 - DQK;
  static_assert(TM_DS + 64 <= TM_DQ, "TMEM");
  // barriers
  static constexpr int B_QD_FULL = 0, B_QD_EMPTY = 1;
  static constexpr int B_K_FULL = 2, B_K_EMPTY = B_K_FULL + KST;
  static constexpr int B_V_FULL = B_K_EMPTY + KST, B_V_EMPTY = B_V_FULL + VST;
  static constexpr int B_S_FULL = B_V_EMPTY + VST;    // S and dP of a tile issued (commit)
  static constexpr int B_SDP_FREE = B_S_FULL + 1;     // compute warps have loaded S and dP
  static constexpr int B_DS_FULL = B_SDP_FREE + 1;    // dS written to TMEM
  static constexpr int B_DS_FREE = B_DS_FULL + 1;     // dQ MMA of the tile done
  static constexpr int B_DQ_FULL = B_DS_FREE + 1;     // the item's last dQ MMA done
  static constexpr int B_DQ_EMPTY = B_DQ_FULL + 1;    // epilogue has read dQ
  static constexpr int B_DRAIN = B_DQ_EMPTY + 1;     // 3: one per MMA issuer
  static constexpr int NBAR = B_DRAIN + 3;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // [0] tmem base, [1] abort
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int DQK, int DV>
__global__ void __launch_bounds__(kBwdThreads, 1)
    ssa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using Lay = BwdDqLayout<DQK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::OFF_BAR + 8 * i; };
  int* status = &g_loza_status;
  const int total_items = bwd_q_items(p);

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_QD_FULL), 1);
    mbar_init(bar(Lay::B_QD_EMPTY), 2);  // the S and the dP issuer
    for (int s = 0; s < Lay::KST; ++s) {
      mbar_init(bar(Lay::B_K_FULL + s), 1);
      mbar_init(bar(Lay::B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < Lay::VST; ++s) {
      mbar_init(bar(Lay::B_V_FULL + s), 1);
      mbar_init(bar(Lay::B_V_EMPTY + s), 1);
    }
    mbar_init(bar(Lay::B_S_FULL), 2);  // S and dP, one commit from each issuer
    mbar_init(bar(Lay::B_SDP_FREE), kBwdComputeThreads);
    mbar_init(bar(Lay::B_DS_FULL), kBwdComputeThreads);
    mbar_init(bar(Lay::B_DS_FREE), 1);
    mbar_init(bar(Lay::B_DQ_FULL), 1);
    mbar_init(bar(Lay::B_DQ_EMPTY), kBwdComputeThreads);
    mbar_init(bar(Lay::B_DRAIN), 1);
    mbar_init(bar(Lay::B_DRAIN + 1), 1);
    mbar_init(bar(Lay::B_DRAIN + 2), 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  if (warp == 9) {
    tmem_alloc(sb + Lay::OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int g = 0, it = 0, qd_issued = 0;
      int k_issued[Lay::KST] = {}, v_issued[Lay::VST] = {};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const BwdQItem w = bwd_q_item(p, item);
        const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
        if (it > 0 && !mbar_wait(bar(Lay::B_QD_EMPTY), (it - 1) & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(Lay::B_QD_FULL), Lay::QTILE + Lay::VTILE);
        ++qd_issued;
#pragma unroll
        for (int c = 0; c < Lay::QCH; ++c)
          tma_load_3d(sb + Lay::OFF_Q + c * Lay::CHUNK, &tm_q, bar(Lay::B_QD_FULL), c * 64,
                      w.seq_start + w.qb * 128, w.plane);
#pragma unroll
        for (int c = 0; c < Lay::VCH; ++c)
          tma_load_3d(sb + Lay::OFF_DO + c * Lay::CHUNK, &tm_do, bar(Lay::B_QD_FULL), c * 64,
                      w.seq_start + w.qb * 128, w.plane);
        for (int t = 0; t < tr.count; ++t, ++g) {
          const int row = w.seq_start + tile_block(tr, t) * 128;
          const int st = g % Lay::KST, use = g / Lay::KST;
          if (use > 0 &&
              !mbar_wait(bar(Lay::B_K_EMPTY + st), (use - 1) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(Lay::B_K_FULL + st), Lay::QTILE);
          ++k_issued[st];
#pragma unroll
          for (int c = 0; c < Lay::QCH; ++c)
            tma_load_3d(sb + Lay::OFF_K + st * Lay::QTILE + c * Lay::CHUNK, &tm_k,
                        bar(Lay::B_K_FULL + st), c * 64, row, w.plane);
          const int vs = g % Lay::VST, vuse = g / Lay::VST;
          if (vuse > 0 &&
              !mbar_wait(bar(Lay::B_V_EMPTY + vs), (vuse - 1) & 1, abort_flag, status, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(Lay::B_V_FULL + vs), Lay::VTILE);
          ++v_issued[vs];
#pragma unroll
          for (int c = 0; c < Lay::VCH; ++c)
            tma_load_3d(sb + Lay::OFF_V + vs * Lay::VTILE + c * Lay::CHUNK, &tm_v,
                        bar(Lay::B_V_FULL + vs), c * 64, row, w.plane);
        }
      }
      if (!ok) {
        // let the copies in flight land before the CTA's shared memory goes away
        for (int s = 0; s < Lay::KST; ++s)
          if (k_issued[s] > 0) mbar_wait_drain(bar(Lay::B_K_FULL + s), (k_issued[s] - 1) & 1);
        for (int s = 0; s < Lay::VST; ++s)
          if (v_issued[s] > 0) mbar_wait_drain(bar(Lay::B_V_FULL + s), (v_issued[s] - 1) & 1);
        if (qd_issued > 0) mbar_wait_drain(bar(Lay::B_QD_FULL), (qd_issued - 1) & 1);
      }
    }
  } else if (warp == 9 || warp == 11) {
    // --------------------------------- MMA issuers: S (warp 9) and dP (warp 11)
    // S/dP of tile g+1 go out as soon as the compute warps have loaded tile
    // g's S and dP; the dQ products have their own issuer (warp 10), so a
    // wait for dS never holds them back.  S and dP come from two threads: a
    // lone thread issues these shared x shared products below the tensor rate.
    if (lane == 0) {
      const bool is_s = warp == 9;
      const uint32_t id_s = idesc_bf16_f32(128, 128, false);
      const uint64_t q_desc = sdesc_sw128(sb + Lay::OFF_Q, 16, 1024);
      const uint64_t do_desc = sdesc_sw128(sb + Lay::OFF_DO, 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(sb + Lay::OFF_K, 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(sb + Lay::OFF_V, 16, 1024);
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const TileRange tr = tile_range(bwd_q_item(p, item).qb, p.n_sink, p.n_local);
        if (!(ok = mbar_wait(bar(Lay::B_QD_FULL), it & 1, abort_flag, status, 1))) break;
        for (int t = 0; t < tr.count; ++t, ++g) {
          const int st = g % Lay::KST, vs = g % Lay::VST;
          if ((g > 0 &&
               !(ok = mbar_wait(bar(Lay::B_SDP_FREE), (g - 1) & 1, abort_flag, status, 1))) ||
              (is_s && !(ok = mbar_wait(bar(Lay::B_K_FULL + st), (g / Lay::KST) & 1, abort_flag,
                                        status, 1))) ||
              (!is_s && !(ok = mbar_wait(bar(Lay::B_V_FULL + vs), (g / Lay::VST) & 1, abort_flag,
                                         status, 1))))
            break;
          tc_fence_after();
          if (is_s) {
            const uint64_t k_desc = k_desc0 + (uint64_t)(st * (Lay::QTILE >> 4));
#pragma unroll
            for (int kk = 0; kk < DQK / 16; ++kk) {
              const uint64_t koff = (uint64_t)(((kk >> 2) * Lay::CHUNK + (kk & 3) * 32) >> 4);
              mma_ss(tmem + Lay::TM_S, q_desc + koff, k_desc + koff, id_s, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar(Lay::B_S_FULL));
          } else {
            const uint64_t v_desc = v_desc0 + (uint64_t)(vs * (Lay::VTILE >> 4));
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk) {
              const uint64_t koff = (uint64_t)(((kk >> 2) * Lay::CHUNK + (kk & 3) * 32) >> 4);
              mma_ss(tmem + Lay::TM_DP, do_desc + koff, v_desc + koff, id_s, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar(Lay::B_S_FULL));
            mma_commit(bar(Lay::B_V_EMPTY + vs));
          }
          if (t == tr.count - 1) mma_commit(bar(Lay::B_QD_EMPTY));
        }
      }
      const uint32_t drain = bar(Lay::B_DRAIN + (is_s ? 0 : 2));
      mma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp == 10) {
    // ------------------------------------------------- MMA issuer: dQ += dS K
    if (lane == 0) {
      const uint32_t id_q = idesc_bf16_f32(128, DQK, true);
      // K read MN-major: keys 16kk .. 16kk+15 of each 64-column box are 2048 bytes in
      const uint64_t k_desc0 = sdesc_sw128(sb + Lay::OFF_K, Lay::CHUNK, 1024);
      int g = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const TileRange tr = tile_range(bwd_q_item(p, item).qb, p.n_sink, p.n_local);
        for (int t = 0; t < tr.count; ++t, ++g) {
          const int st = g % Lay::KST;
          // K(g) is in place (its slot is released only by this issuer) and
          // dS(g) is in TMEM; the item's first product overwrites dQ, which
          // the previous item's epilogue must have read
          if (!(ok = mbar_wait(bar(Lay::B_K_FULL + st), (g / Lay::KST) & 1, abort_flag, status,
                               1)) ||
              !(ok = mbar_wait(bar(Lay::B_DS_FULL), g & 1, abort_flag, status, 1)) ||
              (t == 0 && it > 0 &&
               !(ok = mbar_wait(bar(Lay::B_DQ_EMPTY), (it - 1) & 1, abort_flag, status, 1))))
            break;
          tc_fence_after();
          const uint64_t k_desc = k_desc0 + (uint64_t)(st * (Lay::QTILE >> 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + Lay::TM_DQ, tmem + Lay::TM_DS + kk * 8,
                   k_desc + (uint64_t)(kk * (2048 >> 4)), id_q, (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(Lay::B_DS_FREE));
          mma_commit(bar(Lay::B_K_EMPTY + st));
          if (t == tr.count - 1) mma_commit(bar(Lay::B_DQ_FULL));
        }
      }
      mma_commit(bar(Lay::B_DRAIN + 1));
      mbar_wait_drain(bar(Lay::B_DRAIN + 1), 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------- compute warps
    const int wg = warp >> 2;                                      // key-column half
    const int row = threadIdx.x & 127;                             // query row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int col0 = wg * 64;
    const float sl2 = p.scale_log2;
    int g = 0, it = 0;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x, ++it) {
      const BwdQItem w = bwd_q_item(p, item);
      const TileRange tr = tile_range(w.qb, p.n_sink, p.n_local);
      const int r_in_seq = w.qb * 128 + row;
      const bool valid = r_in_seq < w.len;
      const size_t grow = (size_t)w.plane * p.plane_rows + w.seq_start + r_in_seq;
      // rows past the sequence: P = 0 here, and their dQ is not written
      const float lse2 = valid ? __ldg(p.lse + grow) * 1.4426950408889634f : INFINITY;
      const float dsum = valid ? __ldg(p.dsum + grow) : 0.f;
      bool ok = true;
      for (int t = 0; t < tr.count; ++t, ++g) {
        if (!mbar_wait(bar(Lay::B_S_FULL), g & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool diag = (t == tr.count - 1);
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_base + Lay::TM_S + col0 + h * 32, sr);
          tmem_ld32(tmem + lane_base + Lay::TM_DP + col0 + h * 32, dr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int key0 = col0 + h * 32 + c;
            float p0 = ex2_approx(__uint_as_float(sr[c]) * sl2 - lse2);
            float p1 = ex2_approx(__uint_as_float(sr[c + 1]) * sl2 - lse2);
            if (diag && key0 > row) p0 = 0.f;
            if (diag && key0 + 1 > row) p1 = 0.f;
            const float ds0 = p0 * (__uint_as_float(dr[c]) - dsum);
            const float ds1 = p1 * (__uint_as_float(dr[c + 1]) - dsum);
            pk[h * 16 + c / 2] = pack_bf16x2(ds0, ds1);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(Lay::B_SDP_FREE));
        // the previous tile's dQ MMA has read the dS columns
        if (g > 0 && !mbar_wait(bar(Lay::B_DS_FREE), (g - 1) & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem + lane_base + Lay::TM_DS + col0 / 2, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_DS_FULL));
      }
      if (!ok) break;
      // epilogue: dQ = scale * acc, bf16
      if (!mbar_wait(bar(Lay::B_DQ_FULL), it & 1, abort_flag, status, 1)) break;
      tc_fence_after();
      constexpr int OH = DQK / 2;
      uint32_t orr[OH / 32][32];
#pragma unroll
      for (int ch = 0; ch < OH / 32; ++ch)
        tmem_ld32(tmem + lane_base + Lay::TM_DQ + wg * OH + ch * 32, orr[ch]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(Lay::B_DQ_EMPTY));
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(p.dq + grow * DQK + wg * OH);
#pragma unroll
        for (int ch = 0; ch < OH / 32; ++ch)
#pragma unroll
          for (int v = 0; v < 4; v += 2) {
            uint32_t w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w8[e] = pack_bf16x2(__uint_as_float(orr[ch][8 * v + 2 * e]) * p.scale,
                                  __uint_as_float(orr[ch][8 * v + 2 * e + 1]) * p.scale);
            st_global_v8(dst + ch * 4 + v, w8);
          }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV
//
// Each query block is taken as two half-steps of 64 queries; half-step k = 2s
// + h (query step s, half h) belongs to compute warpgroup h.  Its S^T (keys on
// the TMEM lanes, 64 query columns) goes to TMEM region k mod 3 and its dP^T
// to region (k + 1) mod 3, 64 columns each.  The warpgroup reads both, then
// writes P^T and dS^T as bf16 pairs over the 64 columns of S^T's region, from
// where the dV and dK products read them.  dP^T's region is free once the
// warpgroup has read it, and it is the next half-step's S^T region, so the
// tensor core computes half-step k+1's products while warpgroup h turns
// half-step k into P^T and dS^T.  Three regions (192 columns) beside dV (d_v
// columns) and dK (d_qk columns) fit the 512 columns for d_qk up to 192.
// Q and dO stream through a ring of half-step slots, [Q | dO] rows of 64
// queries each, so that the d_qk = 192 tiles fit shared memory with three
// half-steps in flight.

template <int DQK, int DV>
struct BwdKvLayout {
  static constexpr int QCH = DQK / 64, VCH = DV / 64;
  static constexpr int CHUNK = 128 * 128;   // [128 rows x 64 bf16] box: K, V
  static constexpr int HCHUNK = 64 * 128;   // [64 rows x 64 bf16] box: Q, dO of a half-step
  static constexpr int KTILE = QCH * CHUNK, VTILE = VCH * CHUNK;
  static constexpr int HSLOT = (QCH + VCH) * HCHUNK;  // [Q_h | dO_h]
  static constexpr int NHS = KTILE + VTILE + 4 * HSLOT <= 200 * 1024 ? 4 : 3;  // half-step slots
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KTILE;
  static constexpr int OFF_Q = KTILE + VTILE;           // NHS x [Q_h | dO_h]
  static constexpr int OFF_ROW = OFF_Q + NHS * HSLOT;   // float [2 steps][2 halves][lse2, D][64]
  static constexpr int OFF_BAR = OFF_ROW + 2 * 2 * 2 * 64 * 4;
  // TMEM: regions 0..2 of 64 columns at 64 r, then dV and dK
  static constexpr int TM_DV = 192, TM_DK = 192 + DV;
  static_assert(TM_DK + DQK <= 512, "TMEM");
  // barriers
  static constexpr int B_KV_FULL = 0, B_KV_EMPTY = 1;
  static constexpr int B_Q_FULL = 2, B_Q_EMPTY = B_Q_FULL + NHS;  // per half-step slot
  static constexpr int B_ST_FULL = B_Q_EMPTY + NHS;  // [2] S^T of warpgroup h's half-step done
  static constexpr int B_DPT_FULL = B_ST_FULL + 2;   // [2] dP^T of warpgroup h's half-step done
  static constexpr int B_SYNC = B_DPT_FULL + 2;      // [2] warpgroup h: its rows staged
  static constexpr int B_READ = B_SYNC + 2;          // [2] warpgroup h has read S^T and dP^T
  static constexpr int B_PDS_FULL = B_READ + 2;      // [2] P^T, dS^T written
  static constexpr int B_PDS_FREE = B_PDS_FULL + 2;  // [2] their dV, dK products done
  static constexpr int B_ACC_FULL = B_PDS_FREE + 2;  // the item's last dV, dK products done
  static constexpr int B_ACC_EMPTY = B_ACC_FULL + 1; // epilogue has read dV, dK
  static constexpr int B_DRAIN = B_ACC_EMPTY + 1;    // [3] one per issuer
  static constexpr int NBAR = B_DRAIN + 3;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Epilogue of one accumulator row (D columns; warpgroup h takes columns
// h D/2 .. h D/2 + D/2 - 1): mul * acc as fp32 to part_row (a sink chunk's
// partial) or, when part_row is null, as bf16 to out_row if `valid`.
template <int D>
__device__ __forceinline__ void bwd_kv_store(uint32_t acc_tmem, int h, float mul, float* part_row,
                                             __nv_bfloat16* out_row, bool valid) {
  constexpr int OH = D / 2;
  uint32_t ar[OH / 32][32];
#pragma unroll
  for (int ch = 0; ch < OH / 32; ++ch) tmem_ld32(acc_tmem + h * OH + ch * 32, ar[ch]);
  tmem_wait_ld();
  if (part_row) {
    float* dst = part_row + h * OH;
#pragma unroll
    for (int ch = 0; ch < OH / 32; ++ch)
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + ch * 32 + e) =
            make_float4(__uint_as_float(ar[ch][e]) * mul, __uint_as_float(ar[ch][e + 1]) * mul,
                        __uint_as_float(ar[ch][e + 2]) * mul, __uint_as_float(ar[ch][e + 3]) * mul);
  } else if (valid) {
    uint4* dst = reinterpret_cast<uint4*>(out_row + h * OH);
#pragma unroll
    for (int ch = 0; ch < OH / 32; ++ch)
#pragma unroll
      for (int v = 0; v < 4; v += 2) {
        uint32_t a8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          a8[e] = pack_bf16x2(__uint_as_float(ar[ch][8 * v + 2 * e]) * mul,
                              __uint_as_float(ar[ch][8 * v + 2 * e + 1]) * mul);
        st_global_v8(dst + ch * 4 + v, a8);
      }
  }
}

// TMEM regions of half-step k: S^T (then P^T | dS^T) and dP^T.
__device__ __forceinline__ uint32_t bwd_region_s(int k) { return 64u * (uint32_t)(k % 3); }
__device__ __forceinline__ uint32_t bwd_region_dp(int k) { return 64u * (uint32_t)((k + 1) % 3); }

// tm_q and tm_do here have boxes of 64 rows (a half-step); tm_k and tm_v of 128.
template <int DQK, int DV>
__global__ void __launch_bounds__(kBwdThreads, 1)
    ssa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using Lay = BwdKvLayout<DQK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::OFF_BAR + 8 * i; };
  int* status = &g_loza_status;
  const int total_items = bwd_kv_items(p);

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_KV_FULL), 1);
    mbar_init(bar(Lay::B_KV_EMPTY), 2);  // the S^T and the dP^T issuer
    for (int s = 0; s < Lay::NHS; ++s) {
      mbar_init(bar(Lay::B_Q_FULL + s), 1);
      mbar_init(bar(Lay::B_Q_EMPTY + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(Lay::B_ST_FULL + h), 1);
      mbar_init(bar(Lay::B_DPT_FULL + h), 1);
      mbar_init(bar(Lay::B_SYNC + h), kBwdComputeThreads / 2);
      mbar_init(bar(Lay::B_READ + h), kBwdComputeThreads / 2);
      mbar_init(bar(Lay::B_PDS_FULL + h), kBwdComputeThreads / 2);
      mbar_init(bar(Lay::B_PDS_FREE + h), 1);
      mbar_init(bar(Lay::B_DRAIN + h), 1);
    }
    mbar_init(bar(Lay::B_DRAIN + 2), 1);
    mbar_init(bar(Lay::B_ACC_FULL), 1);
    mbar_init(bar(Lay::B_ACC_EMPTY), kBwdComputeThreads);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_do);
  }
  if (warp == 9) {
    tmem_alloc(sb + Lay::OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0, it = 0, kv_issued = 0;  // k: half-steps issued
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const BwdKItem w = bwd_kv_item(p, item);
        if (it > 0 && !mbar_wait(bar(Lay::B_KV_EMPTY), (it - 1) & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(Lay::B_KV_FULL), Lay::KTILE + Lay::VTILE);
        ++kv_issued;
#pragma unroll
        for (int c = 0; c < Lay::QCH; ++c)
          tma_load_3d(sb + Lay::OFF_K + c * Lay::CHUNK, &tm_k, bar(Lay::B_KV_FULL), c * 64,
                      w.seq_start + w.kb * 128, w.plane);
#pragma unroll
        for (int c = 0; c < Lay::VCH; ++c)
          tma_load_3d(sb + Lay::OFF_V + c * Lay::CHUNK, &tm_v, bar(Lay::B_KV_FULL), c * 64,
                      w.seq_start + w.kb * 128, w.plane);
        for (int qi = w.q_lo; ok && qi <= w.q_hi; ++qi) {
#pragma unroll 1
          for (int h = 0; h < 2; ++h, ++k) {
            const int slot = k % Lay::NHS, use = k / Lay::NHS;
            if (use > 0 &&
                !mbar_wait(bar(Lay::B_Q_EMPTY + slot), (use - 1) & 1, abort_flag, status, 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(Lay::B_Q_FULL + slot), Lay::HSLOT);
            const uint32_t base = sb + Lay::OFF_Q + slot * Lay::HSLOT;
            const int row = w.seq_start + qi * 128 + h * 64;
#pragma unroll
            for (int c = 0; c < Lay::QCH; ++c)
              tma_load_3d(base + c * Lay::HCHUNK, &tm_q, bar(Lay::B_Q_FULL + slot), c * 64, row,
                          w.plane);
#pragma unroll
            for (int c = 0; c < Lay::VCH; ++c)
              tma_load_3d(base + (Lay::QCH + c) * Lay::HCHUNK, &tm_do, bar(Lay::B_Q_FULL + slot),
                          c * 64, row, w.plane);
          }
        }
      }
      // let the copies in flight land before the CTA's shared memory goes away:
      // a slot holds at most one unconsumed load, its newest phase
      if (!ok) {
        drain_ring(bar(Lay::B_Q_FULL), Lay::NHS, k);
        if (kv_issued > 0) mbar_wait_drain(bar(Lay::B_KV_FULL), (kv_issued - 1) & 1);
      }
    }
  } else if (warp == 9 || warp == 11) {
    // ----------------------------- MMA issuers: S^T (warp 9) and dP^T (warp 11)
    // Two issuing threads: a lone thread starts these N = 64 shared x shared
    // products at about half the tensor rate, two together at ~2/3 of it.
    if (lane == 0) {
      const bool is_s = warp == 9;
      const uint32_t id_s = idesc_bf16_f32(128, 64, false);   // M = keys, N = 64 queries
      const uint64_t k_desc = sdesc_sw128(sb + Lay::OFF_K, 16, 1024);
      const uint64_t v_desc = sdesc_sw128(sb + Lay::OFF_V, 16, 1024);
      const uint64_t q_desc0 = sdesc_sw128(sb + Lay::OFF_Q, 16, 1024);
      int k = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const BwdKItem w = bwd_kv_item(p, item);
        if (!(ok = mbar_wait(bar(Lay::B_KV_FULL), it & 1, abort_flag, status, 1))) break;
        for (int qi = w.q_lo; ok && qi <= w.q_hi; ++qi) {
#pragma unroll 1
          for (int h = 0; h < 2; ++h, ++k) {
            const int slot = k % Lay::NHS;
            // S^T's region was the previous half-step's dP^T region: its
            // warpgroup has read it (and that dP^T went in only after the
            // region's P^T / dS^T of half-step k - 3 were consumed); and the
            // warpgroup that takes this half-step has written P^T / dS^T of
            // half-step k - 2, so it has waited for that half-step's S^T and
            // ST_FULL[h] never runs two phases ahead of it.  dP^T's region
            // held P^T / dS^T of half-step k - 2: their dV / dK products are
            // done (which also keeps DPT_FULL[h] within a phase).
            if (!(ok = mbar_wait(bar(Lay::B_Q_FULL + slot), (k / Lay::NHS) & 1, abort_flag,
                                 status, 1)) ||
                (is_s && k >= 1 &&
                 !(ok = mbar_wait(bar(Lay::B_READ + ((k - 1) & 1)), ((k - 1) >> 1) & 1,
                                  abort_flag, status, 1))) ||
                (is_s && k >= 2 &&
                 !(ok = mbar_wait(bar(Lay::B_PDS_FULL + (k & 1)), ((k - 2) >> 1) & 1,
                                  abort_flag, status, 1))) ||
                (!is_s && k >= 2 &&
                 !(ok = mbar_wait(bar(Lay::B_PDS_FREE + (k & 1)), ((k - 2) >> 1) & 1,
                                  abort_flag, status, 1))))
              break;
            tc_fence_after();
            const uint64_t q_desc = q_desc0 + (uint64_t)((slot * Lay::HSLOT) >> 4);
            const uint64_t do_desc = q_desc + (uint64_t)((Lay::QCH * Lay::HCHUNK) >> 4);
            if (is_s) {
              const uint32_t st_t = tmem + bwd_region_s(k);
#pragma unroll
              for (int kk = 0; kk < DQK / 16; ++kk) {
                const uint64_t koff = (uint64_t)(((kk >> 2) * Lay::CHUNK + (kk & 3) * 32) >> 4);
                const uint64_t hoff = (uint64_t)(((kk >> 2) * Lay::HCHUNK + (kk & 3) * 32) >> 4);
                mma_ss(st_t, k_desc + koff, q_desc + hoff, id_s, kk > 0 ? 1u : 0u);
              }
              mma_commit(bar(Lay::B_ST_FULL + h));
            } else {
              const uint32_t dpt_t = tmem + bwd_region_dp(k);
#pragma unroll
              for (int kk = 0; kk < DV / 16; ++kk) {
                const uint64_t koff = (uint64_t)(((kk >> 2) * Lay::CHUNK + (kk & 3) * 32) >> 4);
                const uint64_t hoff = (uint64_t)(((kk >> 2) * Lay::HCHUNK + (kk & 3) * 32) >> 4);
                mma_ss(dpt_t, v_desc + koff, do_desc + hoff, id_s, kk > 0 ? 1u : 0u);
              }
              mma_commit(bar(Lay::B_DPT_FULL + h));
            }
          }
          if (ok && qi == w.q_hi) mma_commit(bar(Lay::B_KV_EMPTY));  // K, V read for the last time
        }
      }
      const uint32_t drain = bar(Lay::B_DRAIN + (is_s ? 0 : 2));
      mma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else if (warp == 10) {
    // ------------------------------------ MMA issuer: dV += P^T dO, dK += dS^T Q
    if (lane == 0) {
      const uint32_t id_v = idesc_bf16_f32(128, DV, true);   // B = dO_h, MN-major
      const uint32_t id_k = idesc_bf16_f32(128, DQK, true);  // B = Q_h, MN-major
      // queries 16kk .. 16kk+15 of a half-step: rows 16kk of every 64-row box
      // (2048 bytes in); consecutive 64-column boxes HCHUNK apart
      const uint64_t q_desc0 = sdesc_sw128(sb + Lay::OFF_Q, Lay::HCHUNK, 1024);
      int k = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x, ++it) {
        const BwdKItem w = bwd_kv_item(p, item);
        for (int qi = w.q_lo; ok && qi <= w.q_hi; ++qi) {
#pragma unroll 1
          for (int h = 0; h < 2; ++h, ++k) {
            const int slot = k % Lay::NHS;
            const uint64_t q_desc = q_desc0 + (uint64_t)((slot * Lay::HSLOT) >> 4);
            const uint64_t do_desc = q_desc + (uint64_t)((Lay::QCH * Lay::HCHUNK) >> 4);
            const bool first = (qi == w.q_lo && h == 0);
            if (!(ok = mbar_wait(bar(Lay::B_Q_FULL + slot), (k / Lay::NHS) & 1, abort_flag,
                                 status, 1)) ||
                !(ok = mbar_wait(bar(Lay::B_PDS_FULL + h), (k >> 1) & 1, abort_flag, status, 1)) ||
                (first && it > 0 &&
                 !(ok = mbar_wait(bar(Lay::B_ACC_EMPTY), (it - 1) & 1, abort_flag, status, 1))))
              break;
            tc_fence_after();
            const uint32_t pt_t = tmem + bwd_region_s(k), dst_t = pt_t + 32;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tmem + Lay::TM_DV, pt_t + kk * 8, do_desc + (uint64_t)((2048 * kk) >> 4),
                     id_v, (!first || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tmem + Lay::TM_DK, dst_t + kk * 8, q_desc + (uint64_t)((2048 * kk) >> 4),
                     id_k, (!first || kk > 0) ? 1u : 0u);
            mma_commit(bar(Lay::B_PDS_FREE + h));
            mma_commit(bar(Lay::B_Q_EMPTY + slot));
          }
          if (!ok) break;
          if (qi == w.q_hi) mma_commit(bar(Lay::B_ACC_FULL));
        }
      }
      mma_commit(bar(Lay::B_DRAIN + 1));
      mbar_wait_drain(bar(Lay::B_DRAIN + 1), 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------- compute warps
    const int h = warp >> 2;                                       // query half of every step
    const int r = threadIdx.x & 127;                               // key row = TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    float* rows_smem = reinterpret_cast<float*>(smem + Lay::OFF_ROW);
    int s = 0, it = 0;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x, ++it) {
      const BwdKItem w = bwd_kv_item(p, item);
      const int key = w.kb * 128 + r;
      bool ok = true;
      for (int qi = w.q_lo; qi <= w.q_hi; ++qi, ++s) {
        const int k = 2 * s + h;  // this warpgroup's half-step
        // stage lse2 and D of this half's 64 queries; rows past the sequence
        // (zero fill, or the next packed sequence) get lse2 = +inf: P = 0
        float* lse_s = rows_smem + ((s & 1) * 2 + h) * 128;
        float* d_s = lse_s + 64;
        {
          const int t = r & 63;
          const int qrow = qi * 128 + h * 64 + t;
          const size_t gq = (size_t)w.plane * p.plane_rows + w.seq_start + qrow;
          if (r < 64) lse_s[t] = qrow < w.len ? __ldg(p.lse + gq) * 1.4426950408889634f : INFINITY;
          else d_s[t] = qrow < w.len ? __ldg(p.dsum + gq) : 0.f;
        }
        mbar_arrive(bar(Lay::B_SYNC + h));
        if (!mbar_wait(bar(Lay::B_SYNC + h), s & 1, abort_flag, status, 1) ||
            !mbar_wait(bar(Lay::B_ST_FULL + h), s & 1, abort_flag, status, 1) ||
            !mbar_wait(bar(Lay::B_DPT_FULL + h), s & 1, abort_flag, status, 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool diag = (qi == w.kb);
        const uint32_t st_t = tmem + lane_base + bwd_region_s(k);
        const uint32_t dpt_t = tmem + lane_base + bwd_region_dp(k);
        uint32_t pk[32], dk_[32];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t st_r[32], dp_r[32];
          tmem_ld32(st_t + c2 * 32, st_r);
          tmem_ld32(dpt_t + c2 * 32, dp_r);
          tmem_wait_ld();
          if (c2 == 1) {
            // all of dP^T is read: its region may take the next half-step's S^T
            tc_fence_before();
            mbar_arrive(bar(Lay::B_READ + h));
          }
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const int qc = c2 * 32 + c;                 // query within the half
            // the staged rows are read four at a time (every thread reads the
            // same address: one broadcast per warp)
            const float4 l4 = *reinterpret_cast<const float4*>(lse_s + qc);
            const float4 d4 = *reinterpret_cast<const float4*>(d_s + qc);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv4[4] = {d4.x, d4.y, d4.z, d4.w};
            float pp[4], dd[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              pp[e] = ex2_approx(__uint_as_float(st_r[c + e]) * sl2 - lv[e]);
              if (diag && h * 64 + qc + e < r) pp[e] = 0.f;  // the key comes after the query
              dd[e] = pp[e] * (__uint_as_float(dp_r[c + e]) - dv4[e]);
            }
            pk[c2 * 16 + c / 2] = pack_bf16x2(pp[0], pp[1]);
            pk[c2 * 16 + c / 2 + 1] = pack_bf16x2(pp[2], pp[3]);
            dk_[c2 * 16 + c / 2] = pack_bf16x2(dd[0], dd[1]);
            dk_[c2 * 16 + c / 2 + 1] = pack_bf16x2(dd[2], dd[3]);
          }
        }
        // P^T and dS^T over the 64 columns of S^T's region
        tmem_st32(st_t, pk);
        tmem_st32(st_t + 32, dk_);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_PDS_FULL + h));
      }
      if (!ok) break;
      // epilogue: dK = scale * acc, then dV = acc, one accumulator at a time;
      // sink chunks go out as fp32 partials that the reduce kernel adds up
      if (!mbar_wait(bar(Lay::B_ACC_FULL), it & 1, abort_flag, status, 1)) break;
      tc_fence_after();
      const size_t grow = (size_t)w.plane * p.plane_rows + w.seq_start + key;
      // slot layout: dK [128 keys][d_qk], then dV [128 keys][d_v]
      float* part = w.slot >= 0 ? p.part + (size_t)w.slot * 128 * (DQK + DV) : nullptr;
      bwd_kv_store<DQK>(tmem + lane_base + Lay::TM_DK, h, p.scale,
                        part ? part + (size_t)r * DQK : nullptr, p.dk + grow * DQK,
                        key < w.len);
      bwd_kv_store<DV>(tmem + lane_base + Lay::TM_DV, h, 1.f,
                       part ? part + (size_t)128 * DQK + (size_t)r * DV : nullptr,
                       p.dv + grow * DV, key < w.len);
      tc_fence_before();
      mbar_arrive(bar(Lay::B_ACC_EMPTY));
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The sink blocks' dK, dV: the sum of their chunks' fp32 partials, as bf16.
// A slot holds dK [128 keys][d_qk] then dV [128 keys][d_v].  Dense: one thread
// per (plane, sink block, key row, 4 columns of dK or dV).  Packed: blockIdx.y
// is the sequence and the threads of its column of CTAs walk its (head, sink
// block, key row, 4 columns).
template <int DQK, int DV>
__global__ void __launch_bounds__(256) ssa_bwd_sink_reduce_kernel(const BwdParams p) {
  constexpr int C4 = (DQK + DV) / 4;  // 4-column groups of a key row: dK's, then dV's
  int n_sink, nb, len, seq_start, planes;
  long long slot_base;  // slot of chunk 0 of sink block 0 of head 0
  int per_head;         // sink slots per head
  if (p.cu_seqlens == nullptr) {
    nb = p.nb;
    len = p.L;
    seq_start = 0;
    planes = p.planes;
    slot_base = 0;
    per_head = p.sink_items;
  } else {
    const int sq = blockIdx.y;
    seq_start = __ldg(p.cu_seqlens + sq);
    len = __ldg(p.cu_seqlens + sq + 1) - seq_start;
    if (len <= 0) return;
    nb = (len + 127) >> 7;
    planes = p.planes;
    const int* pfx_sink = p.pfx + 2 * (p.n_seqs + 1);
    slot_base = __ldg(pfx_sink + sq);
    per_head = bwd_sink_items(p.n_sink, nb);
    if (__ldg(pfx_sink + p.n_seqs) == 0) return;  // invalid cu_seqlens: nothing was computed
  }
  n_sink = min(p.n_sink, nb);
  const long long quads = (long long)planes * n_sink * 128 * C4;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < quads;
       x += (long long)gridDim.x * blockDim.x) {
    const int c4 = (int)(x % C4);
    const int r = (int)((x / C4) % 128);
    const int j = (int)((x / C4 / 128) % n_sink);
    const int plane = (int)(x / C4 / 128 / n_sink);
    const int key = j * 128 + r;
    if (key >= len) continue;
    long long slot = slot_base + (long long)plane * per_head;
    for (int j2 = 0; j2 < j; ++j2) slot += bwd_sink_chunks(j2, nb);
    const bool is_k = c4 < DQK / 4;
    const size_t in_slot = is_k ? (size_t)r * DQK + 4 * c4
                                : (size_t)128 * DQK + (size_t)r * DV + 4 * (c4 - DQK / 4);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < bwd_sink_chunks(j, nb); ++c) {
      const float4 v4 = *reinterpret_cast<const float4*>(
          p.part + (size_t)(slot + c) * 128 * (DQK + DV) + in_slot);
      a.x += v4.x; a.y += v4.y; a.z += v4.z; a.w += v4.w;
    }
    const size_t grow = (size_t)plane * p.plane_rows + seq_start + key;
    uint2 out;
    out.x = pack_bf16x2(a.x, a.y);
    out.y = pack_bf16x2(a.z, a.w);
    if (is_k)
      *reinterpret_cast<uint2*>(p.dk + grow * DQK + 4 * c4) = out;
    else
      *reinterpret_cast<uint2*>(p.dv + grow * DV + 4 * (c4 - DQK / 4)) = out;
  }
}

}  // namespace loza
