// decode.cuh -- paged SSA decode on sm_100a (absorbed-MLA layout).
//
// One new query token per sequence; H_q query heads (a group of up to 128 is
// the M dimension of the MMA) share one latent key/value row of 576 bf16 per
// token (512 latent + 64 rope); the value is the first 512 entries of the
// same row.  The window of the query at t = seq_len - 1 is the sink page(s)
// plus the n_local pages ending at t's page (QbitAI article on LongCat LoZA,
// paragraph on the 1024-token sparse window), read through the page table.
//
// Split kernel: one CTA per (window page, head group, sequence).
//   TMA     the 128-token page (9 swizzled boxes of 64 columns = 144 KB) into
//           smem, Q of the head group streamed in 64-column boxes (4-deep ring)
//   MMA     S[128 heads x 128 keys] = Q K^T   (K = 576: 9 boxes x 4 k-steps)
//   softmax mask keys past t, row max, exp2, row sum; P (bf16) -> smem over
//           the first two (by then consumed) Q ring slots
//   MMA     O[128 x 512] = P V, two N=256 halves, V = the page's first 8 boxes
//           read as an MN-major operand (no transpose copy)
//   out     normalised partial O (fp16), staged in the page buffer (free once
//           P V is done) in the TMA layout and written with 8 bulk-tensor
//           stores; its LSE (fp32) with plain stores
// TMEM: S uses columns [0,128); O uses [0,512) once S has been read.
//
// Merge kernel (programmatic dependent launch after the split kernel):
// LSE = logsumexp_s LSE_s, O = sum_s exp(LSE_s - LSE) O_s.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace loza {

constexpr int kDecodeDqk = 576;
constexpr int kDecodeDv = 512;
// Of every 8 exp2 pairs in the decode softmax, this many run as a polynomial on
// the FMA pipe: with one softmax warp per SM sub-partition the 16 exp2/clock of
// the MUFU unit bound this step (128 x 128 exponentials per page).
constexpr int kDecodePolyPairsPer8 = 3;

struct DecodeParams {
  const int* page_table;  // [B, max_pages]
  const int* seq_lens;    // [B]
  __half* o_part;         // [B, HG, n_split, 128, 512]
  float* lse_part;        // [B, HG, n_split, 128]
  __nv_bfloat16* o;       // [B, H_q, 512]
  float* lse;             // [B, H_q]
  int B, H_q, HG, max_pages, n_pages, n_sink, n_local, n_split;
  int wave;  // CTAs resident at once (one per SM): the CTA `wave` later runs on a freed SM
  float scale_log2;
};

// The decode window of sequence b, as the kernels select it.
struct DecodeWindow {
  int t;       // query position
  int qb;      // logical page of the query
  TileRange tr;
};

// False for a seq_len outside [1, max_pages * 128].
__device__ __forceinline__ bool decode_window(const DecodeParams& p, int b, DecodeWindow& w) {
  const int len = __ldg(p.seq_lens + b);
  if (len < 1 || (long long)len > (long long)p.max_pages * 128) return false;
  w.t = len - 1;
  w.qb = w.t >> 7;
  w.tr = tile_range(w.qb, p.n_sink, p.n_local);
  return true;
}

// Physical page of window tile `i`, or -1 if the table entry is outside the pool.
__device__ __forceinline__ int decode_page(const DecodeParams& p, int b, const DecodeWindow& w,
                                           int i) {
  const int logical = tile_block(w.tr, i);
  const int phys = __ldg(p.page_table + (size_t)b * p.max_pages + logical);
  return (phys >= 0 && phys < p.n_pages) ? phys : -1;
}

struct DecodeLayout {
  static constexpr int CHUNK = 128 * 128;  // [128 rows x 64 bf16], 128B swizzle
  static constexpr int KV_CH = kDecodeDqk / 64;  // 9
  static constexpr int QST = 4;                  // Q ring depth
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_Q = OFF_KV + KV_CH * CHUNK;
  static constexpr int OFF_P = OFF_Q;  // P [128 x 128] bf16 (2 boxes) reuses Q slots 0-1
  static constexpr int OFF_BAR = OFF_Q + QST * CHUNK;
  static constexpr int B_KV_FULL = 0;                    // 9
  static constexpr int B_Q_FULL = B_KV_FULL + KV_CH;     // QST
  static constexpr int B_Q_EMPTY = B_Q_FULL + QST;       // QST
  static constexpr int B_S_FULL = B_Q_EMPTY + QST;
  static constexpr int B_P_FULL = B_S_FULL + 1;
  static constexpr int B_O_FULL = B_P_FULL + 1;
  static constexpr int B_DRAIN = B_O_FULL + 1;
  static constexpr int B_EPI = B_DRAIN + 1;  // staged partial O complete (128 arrivals)
  static constexpr int NBAR = B_EPI + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
};

__global__ void __launch_bounds__(192, 1)
    ssa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_kv,
                            const __grid_constant__ CUtensorMap tm_part, const DecodeParams p) {
  using Lay = DecodeLayout;
  const int sp = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t part = ((size_t)(b * p.HG + hg) * p.n_split + sp) * 128;

  // ---- which page this CTA reads (uniform across the CTA; exits before any barrier)
  DecodeWindow win;
  int phys = -1, valid_keys = 0;
  if (!decode_window(p, b, win)) {
    if (threadIdx.x == 0 && sp == 0 && hg == 0) atomicOr(&g_loza_status, 4);
  } else if (sp < win.tr.count) {
    phys = decode_page(p, b, win, sp);
    if (phys < 0) {
      if (threadIdx.x == 0) atomicOr(&g_loza_status, 2);
    } else {
      const int logical = tile_block(win.tr, sp);
      valid_keys = min(128, win.t - logical * 128 + 1);
    }
  }
  if (phys < 0) {
    if (threadIdx.x < 128) p.lse_part[part + threadIdx.x] = -INFINITY;  // empty split
    asm volatile("griddepcontrol.launch_dependents;");
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::OFF_BAR + 8 * i; };
  int* status = &g_loza_status;

  if (threadIdx.x == 0) {
    for (int c = 0; c < Lay::KV_CH; ++c) mbar_init(bar(Lay::B_KV_FULL + c), 1);
    for (int s = 0; s < Lay::QST; ++s) {
      mbar_init(bar(Lay::B_Q_FULL + s), 1);
      mbar_init(bar(Lay::B_Q_EMPTY + s), 1);
    }
    mbar_init(bar(Lay::B_S_FULL), 1);
    mbar_init(bar(Lay::B_P_FULL), 128);
    mbar_init(bar(Lay::B_O_FULL), 1);
    mbar_init(bar(Lay::B_DRAIN), 1);
    mbar_init(bar(Lay::B_EPI), 128);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_kv);
    prefetch_tensormap(&tm_part);
  }
  if (warp == 5) {
    tmem_alloc(sb + Lay::OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int q_issued = 0;
      bool ok = true;
      auto load_q = [&](int c) -> bool {
        const int st = c % Lay::QST;
        if (c >= Lay::QST &&
            !mbar_wait(bar(Lay::B_Q_EMPTY + st), (c / Lay::QST - 1) & 1, abort_flag, status, 1))
          return false;
        mbar_arrive_expect_tx(bar(Lay::B_Q_FULL + st), Lay::CHUNK);
        tma_load_3d(sb + Lay::OFF_Q + st * Lay::CHUNK, &tm_q, bar(Lay::B_Q_FULL + st), c * 64,
                    hg * 128, b);
        ++q_issued;
        return true;
      };
      // interleave the first Q boxes with the page so the first MMAs can start
      // early; then the rest of the page; then Q boxes as ring slots free up
      for (int c = 0; c < Lay::KV_CH; ++c) {
        if (c < Lay::QST) load_q(c);
        mbar_arrive_expect_tx(bar(Lay::B_KV_FULL + c), Lay::CHUNK);
        tma_load_2d(sb + Lay::OFF_KV + c * Lay::CHUNK, &tm_kv, bar(Lay::B_KV_FULL + c), c * 64,
                    phys * 128);
      }
      for (int c = Lay::QST; ok && c < Lay::KV_CH; ++c) ok = load_q(c);
      // The CTA one wave later starts only when an SM frees up: pull its page
      // and query boxes into L2 now so that its loads hit L2 instead of paying
      // a cold HBM (and page-table) latency after this wave.
      const int lin = (b * p.HG + hg) * p.n_split + sp;
      const int nxt = lin + p.wave;
      if (ok && nxt < p.B * p.HG * p.n_split) {
        const int sp2 = nxt % p.n_split, hg2 = (nxt / p.n_split) % p.HG, b2 = nxt / (p.n_split * p.HG);
        DecodeWindow w2;
        if (decode_window(p, b2, w2) && sp2 < w2.tr.count) {
          const int phys2 = decode_page(p, b2, w2, sp2);
          if (phys2 >= 0) {
            for (int c = 0; c < Lay::KV_CH; ++c) {
              tma_prefetch_2d(&tm_kv, c * 64, phys2 * 128);
              tma_prefetch_3d(&tm_q, c * 64, hg2 * 128, b2);
            }
          }
        }
      }
      // every copy issued lands before the CTA exits (normally already consumed)
      for (int c = 0; c < Lay::KV_CH; ++c) mbar_wait_drain(bar(Lay::B_KV_FULL + c), 0);
      for (int st = 0; st < Lay::QST; ++st) {
        const int n = (q_issued - st + Lay::QST - 1) / Lay::QST;  // loads issued into slot st
        if (n > 0) mbar_wait_drain(bar(Lay::B_Q_FULL + st), (n - 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, false);
      const uint32_t id_o = idesc_bf16_f32(128, 256, true);
      bool ok = true;
      for (int c = 0; ok && c < Lay::KV_CH; ++c) {
        const int st = c % Lay::QST;
        ok = mbar_wait(bar(Lay::B_KV_FULL + c), 0, abort_flag, status, 1) &&
             mbar_wait(bar(Lay::B_Q_FULL + st), (c / Lay::QST) & 1, abort_flag, status, 1);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adesc = sdesc_sw128(sb + Lay::OFF_Q + st * Lay::CHUNK + kk * 32, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(sb + Lay::OFF_KV + c * Lay::CHUNK + kk * 32, 16, 1024);
          mma_ss(tmem, adesc, bdesc, id_s, (c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(Lay::B_Q_EMPTY + st));
      }
      if (ok) {
        mma_commit(bar(Lay::B_S_FULL));
        ok = mbar_wait(bar(Lay::B_P_FULL), 0, abort_flag, status, 1);
      }
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t adesc =
                sdesc_sw128(sb + Lay::OFF_P + (kk >> 2) * Lay::CHUNK + (kk & 3) * 32, 16, 1024);
            const uint64_t bdesc = sdesc_sw128(
                sb + Lay::OFF_KV + half * 4 * Lay::CHUNK + kk * 2048, Lay::CHUNK, 1024);
            mma_ss(tmem + half * 256, adesc, bdesc, id_o, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar(Lay::B_O_FULL));
      }
      mma_commit(bar(Lay::B_DRAIN));
      mbar_wait_drain(bar(Lay::B_DRAIN), 0);
    }
  } else {
    // ----------------------------------------------------- softmax + output
    const int h = threadIdx.x;  // head row within the group
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    do {
      if (!mbar_wait(bar(Lay::B_S_FULL), 0, abort_flag, status, 1)) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(tmem + lane_base + ch * 32, sr[ch]);
      tmem_wait_ld();
      if (valid_keys < 128) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (ch * 32 + c >= valid_keys) sr[ch][c] = __float_as_uint(-INFINITY);
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 128; c += 8)
#pragma unroll
        for (int a = 0; a < 4; ++a)
          mx4[a] = fmax3(mx4[a], __uint_as_float(sr[(c + 2 * a) >> 5][(c + 2 * a) & 31]),
                         __uint_as_float(sr[(c + 2 * a + 1) >> 5][(c + 2 * a + 1) & 31]));
      const float m = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m, -m);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      // P row h -> smem, K-major 128B-swizzled: box (key/64), row h, 16-byte unit u
      // holding keys 8u..8u+7 lands at unit u ^ (h & 7).
      uint8_t* prow = smem + Lay::OFF_P + h * 128;
#pragma unroll
      for (int box = 0; box < 2; ++box) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = box * 64 + u * 8 + 2 * e;
            const uint64_t xx = f2_pack(__uint_as_float(sr[col >> 5][col & 31]),
                                        __uint_as_float(sr[(col + 1) >> 5][(col + 1) & 31]));
            float y0, y1, p0, p1;
            f2_unpack(f2_fma(xx, sl2x2, negm2), y0, y1);
            if (((u * 4 + e) & 7) < kDecodePolyPairsPer8) {
              exp2_poly_x2(y0, y1, p0, p1);
            } else {
              p0 = ex2_approx(y0);
              p1 = ex2_approx(y1);
            }
            acc[e] = f2_add(acc[e], f2_pack(p0, p1));
            w4[e] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + box * Lay::CHUNK + ((u ^ (h & 7)) << 4)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      float l;
      {
        float a0, a1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
        l = a0 + a1;
      }
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(bar(Lay::B_P_FULL));

      if (!mbar_wait(bar(Lay::B_O_FULL), 0, abort_flag, status, 1)) break;
      tc_fence_after();
      asm volatile("griddepcontrol.launch_dependents;");
      const bool valid = hg * 128 + h < p.H_q;
      const float inv_l = 1.f / l;
      // Stage row h of the partial O (fp16) in the page buffer, laid out as the
      // 128B-swizzled [128 rows x 64 columns] boxes a TMA store reads:
      // 16-byte unit u of box c, row h, sits at unit u ^ (h & 7).
      uint8_t* srow = smem + Lay::OFF_KV + h * 128;
#pragma unroll 1
      for (int j = 0; j < kDecodeDv / 64; ++j) {
        uint32_t orr[2][32];
        tmem_ld32(tmem + lane_base + j * 64, orr[0]);
        tmem_ld32(tmem + lane_base + j * 64 + 32, orr[1]);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t* r8 = &orr[u >> 2][(u & 3) * 8];
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __half2 hv = __floats2half2_rn(__uint_as_float(r8[2 * e]) * inv_l,
                                           __uint_as_float(r8[2 * e + 1]) * inv_l);
            w[e] = *reinterpret_cast<uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(srow + j * Lay::CHUNK + ((u ^ (h & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_async_shared();
      mbar_arrive(bar(Lay::B_EPI));
      if (h == 0 && mbar_wait(bar(Lay::B_EPI), 0, abort_flag, status, 1)) {
        // rows part..part+127 of the [rows x 512] fp16 workspace, 8 boxes
#pragma unroll
        for (int j = 0; j < kDecodeDv / 64; ++j)
          tma_store_2d(&tm_part, sb + Lay::OFF_KV + j * Lay::CHUNK, j * 64, (int)part);
        tma_store_commit_and_wait_read();  // smem is read before the CTA exits
      }
      if (valid) p.lse_part[part + h] = (m + __log2f(l)) * kLn2;
    } while (false);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One CTA of 64 threads per (sequence, head): each thread merges 8 of the 512
// output columns (one 16-byte fp16 load per split).  Launched as a programmatic
// dependent of the split kernel; it waits for the split kernel's results
// before reading.  Splits whose LSE is -inf are empty and contribute nothing
// (their partial O is never read into the sum).
constexpr int kMergeThreads = kDecodeDv / 8;

__global__ void __launch_bounds__(kMergeThreads)
    ssa_decode_merge_kernel(const DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x / p.H_q, h = blockIdx.x % p.H_q;
  const int hg = h >> 7, hr = h & 127;
  const size_t base = (size_t)(b * p.HG + hg) * p.n_split;
  const float* lsep = p.lse_part + base * 128 + hr;              // split stride 128
  const uint4* op = reinterpret_cast<const uint4*>(p.o_part + (base * 128 + hr) * kDecodeDv) +
                    threadIdx.x;                                // split stride 128*512/8
  constexpr size_t kSplitStride = 128 * kDecodeDv / 8;
  float lmax = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < p.n_split; ++s) lmax = fmaxf(lmax, __ldg(lsep + s * 128));
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float denom = 0.f;
  if (lmax > -INFINITY) {
#pragma unroll 8
    for (int s = 0; s < p.n_split; ++s) {
      const float ls = __ldg(lsep + s * 128);
      const uint4 raw = __ldg(op + s * kSplitStride);
      if (ls == -INFINITY) continue;
      const float wgt = __expf(ls - lmax);
      denom += wgt;
      const __half2* hv = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hv[e]);
        acc[2 * e] += wgt * f.x;
        acc[2 * e + 1] += wgt * f.y;
      }
    }
  }
  const float inv = denom > 0.f ? 1.f / denom : 0.f;
  uint4 pk;
  pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *(reinterpret_cast<uint4*>(p.o + ((size_t)b * p.H_q + h) * kDecodeDv) + threadIdx.x) = pk;
  if (threadIdx.x == 0)
    p.lse[(size_t)b * p.H_q + h] = denom > 0.f ? lmax + __logf(denom) : -INFINITY;
}

}  // namespace loza
