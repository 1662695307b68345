// decode.cuh -- paged SSA decode on sm_100a (absorbed-MLA layout).
//
// One new query token per sequence; H_q query heads (a group of up to 128 is
// the M dimension of the MMA) share one latent key/value row of 576 bf16 per
// token (512 latent + 64 rope); the value is the first 512 entries of the
// same row.  The window of the query at t = seq_len - 1 is the sink page(s)
// plus the n_local pages ending at t's page (QbitAI article on LongCat LoZA,
// paragraph on the 1024-token sparse window), read through the page table.
//
// Split kernel: one CTA (one per SM) per (pair of window pages, head group,
// sequence).  The two pages A and B share the query, so S over both is one
// 128 x 256 product and their softmax is joint (no rescaling).
//   TMA     a 4-stage ring of 48 KB stages (Q box | K_A box | K_B box):
//             9 S stages, K boxes in the order 8, 0, 1, .., 7 (576 columns)
//           The last four S stages hold K boxes 4..7, which are also V columns
//           256..511: they stay in the ring for O half 1.  V columns 0..255
//           are read again (L2 hits): page A's boxes into the Q slots (free
//           once S is done), page B's into the K_A slots (free once O half
//           1's page-A products are done).
//   MMA     S[128 heads x 256 keys] = Q [K_A; K_B]^T into TMEM columns
//           [0,256) -- K_A and K_B boxes sit side by side, one N=256 operand
//   softmax warpgroup 0 takes page A's 128 keys of every head row, warpgroup 1
//           page B's; the row max and row sum are exchanged through shared
//           memory; P (bf16 pairs) goes over the first half of each page's
//           S columns (P_A in [0,64), P_B in [128,192)) with tcgen05.st
//   MMA     O half = P [V_A; V_B][:, 256 columns] (A = P in TMEM, N = 256) into
//           TMEM columns [256,512): half 1 first, then half 0
//   out     each half, normalised, as fp16 to the workspace in the layout
//           [CTA][64 groups of 8 columns][128 heads][8] (a warp's stores of
//           a group are 512 contiguous bytes); the LSE as fp32
//
// FP8 cache (template argument FP8): each latent row is 576 e4m3 codes with
// one fp32 scale per token, K_j = s_j k8_j.  The TMA puts a page's 64-channel
// e4m3 box (8 KB) in the upper half of its 16 KB bf16 slot; the softmax
// warpgroups, idle while S is built, expand it in place to the bf16 swizzled
// box the MMA reads (e4m3 values are exact in bf16) and arrive on a second
// barrier the MMA waits for.  The scale stays out of the products: S column j
// is multiplied by s_j before the softmax, and P_ij s_j is what goes to TMEM
// for the P V product, so O = sum_j p_ij s_j v8_j / l with l = sum_j p_ij.
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
constexpr int kDecodePagesPerSplit = 2;
// Of every 8 exp2 pairs in the decode softmax, this many run as a polynomial
// on the FMA pipe instead of the MUFU unit.
constexpr int kDecodePolyPairsPer8 = 3;

// Rows of the decode: one per (sequence, query token).  With q_len query
// tokens per sequence, row v is token v % q_len of sequence v / q_len, at
// position seq_len - q_len + v % q_len; q, o and lse are indexed by row.
struct DecodeParams {
  const int* page_table;  // [sequences, max_pages]
  const int* seq_lens;    // [sequences]
  __half* o_part;         // [B*HG*n_split CTAs][64 column groups][128 heads][8]
  float* lse_part;        // [B*HG*n_split CTAs][128 heads]
  __nv_bfloat16* o;       // [B rows, H_q, 512]
  float* lse;             // [B rows, H_q]
  int B;                  // rows: sequences * q_len
  int q_len;              // query tokens per sequence (1: plain decode)
  int H_q, HG, max_pages, n_pages, n_sink, n_local;
  int n_split;  // split CTAs per (sequence, head group): ceil(listed pages / 2)
  // Optional pages chosen per sequence on top of the window (nullptr: none):
  // [B, max_extra] logical page ids.
  const int* extra_pages;
  int max_extra;
  int wave;     // CTAs resident at once: the CTA `wave` later runs on a freed SM
  float scale_log2;
  // FP8 cache only: fp32 scale of every token, [n_pages, 128] by physical page.
  const float* kv_scale;
  // 1: the n_split splits of a (row, head group) run as one thread-block
  // cluster and merge their partials in the split kernel (no merge kernel).
  int cluster_merge;
  // Long-window kernel (decode_long.cuh; nullptr otherwise): plan[u] = pages
  // listed by the (row, head group) units before u, plan[B * HG] = all of
  // them; the pages are shared out over n_pairs CTA pairs; then, from
  // plan + B * HG + 1, each unit's first partial slot and slot count.
  const int* plan;
  int n_pairs;
};

__device__ __forceinline__ int decode_seq(const DecodeParams& p, int row) {
  return p.q_len == 1 ? row : row / p.q_len;
}

// The decode window of row b, as the kernels select it.
struct DecodeWindow {
  int t;       // query position
  int qb;      // logical page of the query
  TileRange tr;
};

// False for a seq_len outside [q_len, max_pages * 128].
__device__ __forceinline__ bool decode_window(const DecodeParams& p, int b, DecodeWindow& w) {
  const int s = decode_seq(p, b);
  const int len = __ldg(p.seq_lens + s);
  if (len < p.q_len || (long long)len > (long long)p.max_pages * 128) return false;
  w.t = len - p.q_len + (b - s * p.q_len);
  w.qb = w.t >> 7;
  w.tr = tile_range(w.qb, p.n_sink, p.n_local);
  return true;
}

// Logical pages of split `sp` of row b: entries 2sp and 2sp+1 of the
// sequence's page list, which holds the window's tiles in order, then the
// sequence's extra pages that lie strictly between the sink pages and the local
// run (others are in the window or after the query) and were not listed
// before.  Returns how many of the two entries exist (0..2).  The extra pages
// are the page-level selection of the LongCat sparse-attention article (机制 1:
// fixed sink + sliding window plus indexer-chosen tokens; 机制 3: chosen in
// pages of P = 128).  One pass over the list; the duplicate check makes it
// O(max_extra^2) loads at worst, all from one small L1-resident row.
__device__ __forceinline__ int decode_split_pages(const DecodeParams& p, int b,
                                                  const DecodeWindow& w, int sp, int (&lg)[2]) {
  int n = 0, i = kDecodePagesPerSplit * sp;
  for (; i < w.tr.count && n < 2; ++i) lg[n++] = tile_block(w.tr, i);
  if (n == 2 || p.max_extra == 0) return n;
  int k = i - w.tr.count;  // index among the extra pages of the next entry wanted
  const int* ex = p.extra_pages + (size_t)decode_seq(p, b) * p.max_extra;
  for (int j = 0; j < p.max_extra && n < 2; ++j) {
    const int e = __ldg(ex + j);
    if (e < p.n_sink || e >= w.tr.local_lo) continue;
    bool dup = false;
    for (int j2 = 0; j2 < j && !dup; ++j2) dup = __ldg(ex + j2) == e;
    if (dup) continue;
    if (k == 0) lg[n++] = e;
    else --k;
  }
  return n;
}

// Chosen pages of row b that count, in the list's order: those strictly
// between the sink pages and the local run (others are in the window or after
// the query's page), each page once.  decode_extra_count: how many there are;
// decode_extra_page: the k-th of them (0-based), or -1.  O(max_extra^2) loads
// at worst, from one small L1-resident row.
__device__ __forceinline__ bool decode_extra_counts(const DecodeParams& p, const int* ex, int j,
                                                    const DecodeWindow& w) {
  const int e = __ldg(ex + j);
  if (e < p.n_sink || e >= w.tr.local_lo) return false;
  for (int j2 = 0; j2 < j; ++j2)
    if (__ldg(ex + j2) == e) return false;
  return true;
}
__device__ __forceinline__ int decode_extra_count(const DecodeParams& p, int b,
                                                  const DecodeWindow& w) {
  if (p.max_extra == 0) return 0;
  const int* ex = p.extra_pages + (size_t)decode_seq(p, b) * p.max_extra;
  int n = 0;
  for (int j = 0; j < p.max_extra; ++j) n += decode_extra_counts(p, ex, j, w) ? 1 : 0;
  return n;
}
__device__ __forceinline__ int decode_extra_page(const DecodeParams& p, int b,
                                                 const DecodeWindow& w, int k) {
  const int* ex = p.extra_pages + (size_t)decode_seq(p, b) * p.max_extra;
  for (int j = 0; j < p.max_extra; ++j)
    if (decode_extra_counts(p, ex, j, w) && k-- == 0) return __ldg(ex + j);
  return -1;
}

// Physical page of a logical page of row b's sequence, or -1 if the table entry is
// outside the pool.
__device__ __forceinline__ int decode_page(const DecodeParams& p, int b, int logical) {
  if (logical < 0) return -1;
  const int phys = __ldg(p.page_table + (size_t)decode_seq(p, b) * p.max_pages + logical);
  return (phys >= 0 && phys < p.n_pages) ? phys : -1;
}

// Keys of a logical page at or before the query (1..128).
__device__ __forceinline__ int decode_valid_keys(const DecodeWindow& w, int logical) {
  return min(128, w.t - logical * 128 + 1);
}

// Pair that owns flat page x of T, with P pairs: pair k owns [k T / P, (k+1) T / P).
__host__ __device__ __forceinline__ int long_pair_of(long long x, long long T, int P) {
  return (int)(((x + 1) * P + T - 1) / T) - 1;
}
__host__ __device__ __forceinline__ long long long_pair_start(int k, long long T, int P) {
  return (long long)k * T / P;
}
// Pairs that share T pages when `launched` pairs run: at most one per page, so
// that every pair's range [k T / P, (k+1) T / P) holds at least one page.
__host__ __device__ __forceinline__ int long_pairs(int launched, long long T) {
  return (int)(T < launched ? (T > 0 ? T : 1) : launched);
}
// Partial slots of unit u, whose pages are [lo, lo + n) of the T listed, with P
// pairs: one per pair its pages reach, slots u + k for those pairs k
// (consecutive), so *first = u + (first pair) and *count = the pairs reached
// (0 for a unit without pages).
__host__ __device__ __forceinline__ void long_unit_slot_range(int u, long long lo, int n,
                                                              long long T, int P, int* first,
                                                              int* count) {
  if (n <= 0) {
    *first = 0;
    *count = 0;
    return;
  }
  const int kf = long_pair_of(lo, T, P), kl = long_pair_of(lo + n - 1, T, P);
  *first = u + kf;
  *count = kl - kf + 1;
}

struct DecodeLayout {
  static constexpr int CHUNK = 128 * 128;        // [128 rows x 64 bf16], 128B swizzle
  static constexpr int KV_CH = kDecodeDqk / 64;  // 9 boxes per 576-wide row block
  static constexpr int NST = 4;                  // ring stages
  static constexpr int STAGE = 3 * CHUNK;        // slots: Q box | K_A box | K_B box
  static constexpr int N_KEEP = 4;               // last S stages kept for P V (boxes 4..7)
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_XCHG = NST * STAGE;  // float [2 warpgroups][128 rows] x (max, sum)
  static constexpr int OFF_BAR = OFF_XCHG + 2 * 2 * 128 * 4;
  static constexpr int B_FULL = 0;              // NST
  static constexpr int B_EMPTY = B_FULL + NST;  // NST
  static constexpr int B_VA_FULL = B_EMPTY + NST;  // V_A boxes 0..3 in the Q slots
  static constexpr int B_VB_FULL = B_VA_FULL + 1;  // V_B boxes 0..3 in the K_A slots
  static constexpr int B_S_FULL = B_VB_FULL + 1;
  static constexpr int B_P_FULL = B_S_FULL + 1;   // 256 arrivals
  static constexpr int B_XCHG = B_P_FULL + 1;     // 256 arrivals; phase 0 max, 1 sum
  // O output buffers: bf16 cache, two 128-column TMEM regions (quarters 3 and
  // 1 in region 1, 2 and 0 in region 0; one phase per use); FP8 cache, index 0
  // only (phase 0: O half 1, phase 1: O half 0)
  static constexpr int B_O_FULL = B_XCHG + 1;      // 2
  static constexpr int B_O_EMPTY = B_O_FULL + 2;   // 2, 256 arrivals
  static constexpr int B_KA_FREE = B_O_EMPTY + 2;  // page A's products over boxes 4..7 done
  static constexpr int B_DRAIN = B_KA_FREE + 1;
  // FP8 cache: a stage's K boxes expanded to bf16, the V_A and the V_B boxes
  // expanded
  static constexpr int B_CONV = B_DRAIN + 1;  // NST
  static constexpr int B_VA_CONV = B_CONV + NST;  // 256 arrivals: both warpgroups convert
  static constexpr int B_VB_CONV = B_VA_CONV + 1;  // 256 arrivals
  static constexpr int B_XP = B_VB_CONV + 1;  // 2, 128 arrivals: a warpgroup read its e4m3 box
  static constexpr int NBAR = B_XP + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // FP8 cache: float [2 pages][128 tokens] of s_j * scale * log2(e), then of s_j
  static constexpr int OFF_SCALE = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_SCALE + 2 * 2 * 128 * 4 + 1024;
  static constexpr int CHUNK8 = CHUNK / 2;  // one e4m3 box: 128 rows x 64 bytes
  static constexpr int TMEM_COLS = 512;  // S [0,256) (P inside it), O [256,512)
  static constexpr int TM_O = 256;
};

// S stage i (0..8) loads K box decode_s_box(i) -- the rope box first, then the
// latent boxes in order -- into ring stage decode_s_stage(i), numbered so that
// the last N_KEEP stages (boxes 4..7 = V columns 256..511) land in stages
// 0..3 in order, one STAGE apart: an MN-major operand with a constant stride.
__host__ __device__ constexpr int decode_s_box(int i) { return i == 0 ? 8 : i - 1; }
__host__ __device__ constexpr int decode_s_stage(int i) { return (i + 3) & 3; }
// How many earlier S stages used the same ring stage (the mbarrier phase).
__host__ __device__ constexpr int decode_s_round(int i) {
  return (i + 3) / 4 - (decode_s_stage(i) != 3 ? 1 : 0);
}

// Bit k set: key 32*ch + k of the page is at or before the query.
__device__ __forceinline__ uint32_t decode_chunk_mask(int valid_keys, int ch) {
  const int n = valid_keys - 32 * ch;
  return n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : (1u << n) - 1u);
}

// Two e4m3 codes (bytes `sel` of w, picked by a byte permute) to a bf16x2
// word, exactly: the code's magnitude bits placed at bf16 bits 4..10 read as
// exponent e and mantissa m, i.e. 2^(e-127) (1 + m/8) (a bf16 subnormal m/8
// 2^-126 when e = 0); one multiply by 2^120 (no rounding, subnormal inputs
// supported) gives the e4m3 value 2^(e-7) (1 + m/8), or m/8 2^-6, and the
// sign bit moves from bit 7 to bit 15.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w) {
  uint32_t y, r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(y) : "r"(w), "n"(SEL));  // code bytes -> bytes 0, 2
  const uint32_t bits = ((y << 4) & 0x07F007F0u) | ((y << 8) & 0x80008000u);
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(bits), "r"(0x7B807B80u));  // x 2^120
  return r;
}

// FP8 cache: expand one e4m3 box (128 rows x 64 channels; row r at byte 64 r
// of the slot's upper half, as the TMA wrote it) in place into the bf16
// 128-byte-swizzled box the MMA reads (row r at byte 128 r, 16-byte chunk c
// at chunk c ^ (r & 7)).  Thread `row` of a warpgroup takes one row.  The
// bf16 rows 64.. overlap the e4m3 rows, so every row is read before any is
// written: the warpgroup's threads arrive on `xp` (128 arrivals) once they
// have read, and write only after the phase completes.  The wait is bounded,
// so a thread that left early (its own wait failed) ends the others' wait
// with the abort flag rather than holding them.  `uses` counts this
// thread's uses of `xp` (its phase).
__device__ __forceinline__ bool decode_expand_fp8_box(uint32_t slot, int row, uint32_t xp,
                                                      uint32_t& uses, volatile int* abort_flag,
                                                      int* status) {
  uint32_t in[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) lds_v4(slot + DecodeLayout::CHUNK8 + 64 * row + 16 * j, in + 4 * j);
  mbar_arrive(xp);
  const bool ok = mbar_wait(xp, uses & 1, abort_flag, status, 1);
  ++uses;
  if (!ok) return false;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    sts_v4(slot + 128 * row + 16 * (c ^ (row & 7)), e4m3x2_to_bf16x2<0x4140>(in[2 * c]),
           e4m3x2_to_bf16x2<0x4342>(in[2 * c]), e4m3x2_to_bf16x2<0x4140>(in[2 * c + 1]),
           e4m3x2_to_bf16x2<0x4342>(in[2 * c + 1]));
  return true;
}

template <bool FP8>
__device__ __forceinline__ void decode_split_body(const CUtensorMap* tm_q_p,
                                                  const CUtensorMap* tm_kv_p,
                                                  const DecodeParams& p, int sp, int hg, int b,
                                                  size_t cta, int phys_a, int phys_b, int valid_a,
                                                  int valid_b);

// Merge of the split partials of row b, head group hg (n_split <= 4), for the
// 8-column groups [g0, g1) of O: LSE = logsumexp_s LSE_s, O = sum_s exp(LSE_s -
// LSE) O_s.  Splits whose LSE is -inf are empty and contribute nothing (their
// partial O is never read into the sum); a NaN LSE marks a split that gave up
// on a wait, and makes the head's O and LSE NaN.  256 threads: thread (set,
// head) = (tid / 128, tid % 128) takes groups g0 + set, g0 + set + 2, ... in
// passes of 8, with every load of a pass in flight at once (one L2 round trip
// per pass); a warp's loads of one group of one split are 32 heads' 16-byte
// pieces, 512 contiguous bytes.  The partials are read from L2 (ld.global.cg).
constexpr int kClusterMergeMaxSplits = 4;

__device__ __forceinline__ void decode_merge_groups(const DecodeParams& p, int b, int hg, int g0,
                                                    int g1, bool write_lse, int tid) {
  constexpr int NS = kClusterMergeMaxSplits, PASS = 8;
  const int n = p.n_split;
  const int h = tid & 127, set = tid >> 7;
  const int hq = hg * 128 + h;
  if (tid >= 256 || hq >= p.H_q) return;
  const size_t cta0 = ((size_t)b * p.HG + hg) * n;
  const uint4* op = reinterpret_cast<const uint4*>(p.o_part) + cta0 * (64 * 128) + h;
  float ls[NS];
  float mx = -INFINITY;
  bool poisoned = false;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    ls[s] = s < n ? __ldcg(p.lse_part + (cta0 + s) * 128 + h) : -INFINITY;
    poisoned |= ls[s] != ls[s];
    mx = fmaxf(mx, ls[s]);  // fmaxf skips a NaN operand
  }
  float wgt[NS];
  float den = 0.f;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    // empty split, or one that gave up: weight 0 (its partial O is not read)
    wgt[s] = (s < n && ls[s] != -INFINITY && ls[s] == ls[s]) ? __expf(ls[s] - mx) : 0.f;
    den += wgt[s];
  }
  const float inv = poisoned ? __int_as_float(0x7fc00000) : (den > 0.f ? 1.f / den : 0.f);
  uint4* orow = reinterpret_cast<uint4*>(p.o + ((size_t)b * p.H_q + hq) * kDecodeDv);
  for (int gb = g0 + set; gb < g1; gb += 2 * PASS) {
    uint4 raw[PASS][NS];
#pragma unroll
    for (int k = 0; k < PASS; ++k)
#pragma unroll
      for (int s = 0; s < NS; ++s)
        if (gb + 2 * k < g1 && wgt[s] != 0.f)
          raw[k][s] = __ldcg(op + ((size_t)s * 64 + gb + 2 * k) * 128);
#pragma unroll
    for (int k = 0; k < PASS; ++k) {
      if (gb + 2 * k >= g1) break;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        if (wgt[s] == 0.f) continue;
        const __half2* hv = reinterpret_cast<const __half2*>(&raw[k][s]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          acc[2 * e] += wgt[s] * f.x;
          acc[2 * e + 1] += wgt[s] * f.y;
        }
      }
      uint4 pk;
      pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      pk.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      pk.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      orow[gb + 2 * k] = pk;
    }
  }
  if (write_lse && set == 0)
    p.lse[(size_t)b * p.H_q + hq] = poisoned ? __int_as_float(0x7fc00000)
                                    : den > 0.f ? mx + __logf(den) : -INFINITY;
}

template <bool FP8>
__global__ void __launch_bounds__(320, 1)
    ssa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_kv, const DecodeParams p) {
  const int sp = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const size_t cta = ((size_t)b * p.HG + hg) * p.n_split + sp;  // partial-result slot

  // The query boxes do not depend on the page table: start pulling them into
  // L2 while the table is read.
  if (threadIdx.x == 256)
    for (int c = 0; c < kDecodeDqk / 64; ++c) tma_prefetch_3d(&tm_q, c * 64, hg * 128, b);

  // ---- which pages this CTA reads (uniform across the CTA; exits before any barrier).
  // A page whose table entry is bad is skipped (and flagged); if only one page
  // is left it is page A.
  DecodeWindow win;
  int phys_a = -1, phys_b = -1, valid_a = 0, valid_b = 0;
  if (!decode_window(p, b, win)) {
    if (threadIdx.x == 0 && sp == 0 && hg == 0) atomicOr(&g_loza_status, 4);
  } else {
    int lg[2];
    const int n_lg = decode_split_pages(p, b, win, sp, lg);
    for (int i = 0; i < n_lg; ++i) {
      const int logical = lg[i];
      const int ph = decode_page(p, b, logical);
      if (ph < 0) {
        if (threadIdx.x == 0) atomicOr(&g_loza_status, 2);
      } else if (phys_a < 0) {
        phys_a = ph;
        valid_a = decode_valid_keys(win, logical);
      } else {
        phys_b = ph;
        valid_b = decode_valid_keys(win, logical);
      }
    }
  }
  if (phys_a < 0) {
    if (threadIdx.x < 128) p.lse_part[cta * 128 + threadIdx.x] = -INFINITY;  // empty split
    if (!p.cluster_merge) {
      asm volatile("griddepcontrol.launch_dependents;");
      return;
    }
  } else {
    decode_split_body<FP8>(&tm_q, &tm_kv, p, sp, hg, b, cta, phys_a, phys_b, valid_a, valid_b);
  }
  if (p.cluster_merge) {
    // The splits of this (row, head group) are the CTAs of this cluster, all
    // resident at once.  Every thread of every split arrives once its writes
    // of the partials are done (every wait before this point is bounded, and
    // an empty split arrives straight away), then each split merges its share
    // of the 64 column groups; split 0 also writes the LSE.
    cluster_arrive_release();
    cluster_wait_acquire();
    const int n = p.n_split;
    decode_merge_groups(p, b, hg, 64 * sp / n, 64 * (sp + 1) / n, sp == 0, threadIdx.x);
  }
}

template <bool FP8>
__device__ __forceinline__ void decode_split_body(const CUtensorMap* tm_q_p,
                                                  const CUtensorMap* tm_kv_p,
                                                  const DecodeParams& p, int sp, int hg, int b,
                                                  size_t cta, int phys_a, int phys_b, int valid_a,
                                                  int valid_b) {
  using Lay = DecodeLayout;
  const CUtensorMap& tm_q = *tm_q_p;
  const CUtensorMap& tm_kv = *tm_kv_p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool two = phys_b >= 0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t ring = sb + Lay::OFF_RING;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::OFF_BAR + 8 * i; };
  int* status = &g_loza_status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Lay::NST; ++s) {
      mbar_init(bar(Lay::B_FULL + s), 1);
      mbar_init(bar(Lay::B_EMPTY + s), 1);
    }
    mbar_init(bar(Lay::B_VA_FULL), 1);
    mbar_init(bar(Lay::B_VB_FULL), 1);
    mbar_init(bar(Lay::B_S_FULL), 1);
    mbar_init(bar(Lay::B_P_FULL), 256);
    mbar_init(bar(Lay::B_XCHG), 256);
    for (int r = 0; r < 2; ++r) {
      mbar_init(bar(Lay::B_O_FULL + r), 1);
      mbar_init(bar(Lay::B_O_EMPTY + r), 256);
    }
    mbar_init(bar(Lay::B_KA_FREE), 1);
    mbar_init(bar(Lay::B_DRAIN), 1);
    if (FP8) {
      for (int s = 0; s < Lay::NST; ++s) mbar_init(bar(Lay::B_CONV + s), 256);
      mbar_init(bar(Lay::B_VA_CONV), 256);
      mbar_init(bar(Lay::B_VB_CONV), 256);
      mbar_init(bar(Lay::B_XP), 128);
      mbar_init(bar(Lay::B_XP + 1), 128);
    }
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_kv);
  }
  if (warp == 9) {
    tmem_alloc(sb + Lay::OFF_MISC, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // K boxes: bf16 (a whole slot) or e4m3 (the slot's upper half)
      const uint32_t kbox = FP8 ? Lay::CHUNK8 : Lay::CHUNK;
      const uint32_t koff = FP8 ? Lay::CHUNK8 : 0;
      const uint32_t s_bytes = Lay::CHUNK + (two ? 2 : 1) * kbox;
      int issued = 0;        // S stages issued
      bool va = false, vb = false;
      // With one head group and one token per sequence no other CTA reads this
      // CTA's pages (unless the page table maps two sequences to one page): the
      // boxes it reads for the last time (boxes 4..8 in S, 0..3 when reloaded as
      // values) are marked first to leave L2.  The policy only orders evictions;
      // a shared page read again later comes from DRAM, with the same values.
      const bool once = p.HG == 1 && p.q_len == 1;
      const uint64_t pol = l2_policy_evict_first();
      auto load_k = [&](uint32_t dst_k, uint32_t fb, int c, int page, bool last_read) {
        if (once && last_read) tma_load_2d_hint(dst_k, &tm_kv, fb, c * 64, page * 128, pol);
        else tma_load_2d(dst_k, &tm_kv, fb, c * 64, page * 128);
      };
      do {
        for (int i = 0; i < Lay::KV_CH; ++i) {
          const int st = decode_s_stage(i), r = decode_s_round(i);
          if (r > 0 && !mbar_wait(bar(Lay::B_EMPTY + st), (r - 1) & 1, abort_flag, status, 1))
            break;
          const int c = decode_s_box(i);
          const uint32_t dst = ring + st * Lay::STAGE, full = bar(Lay::B_FULL + st);
          mbar_arrive_expect_tx(full, s_bytes);
          tma_load_3d(dst, &tm_q, full, c * 64, hg * 128, b);
          load_k(dst + Lay::CHUNK + koff, full, c, phys_a, c >= 4);
          if (two) load_k(dst + 2 * Lay::CHUNK + koff, full, c, phys_b, c >= 4);
          ++issued;
          if (i == 0) {
            // A CTA one wave later starts only when an SM frees up: pull its
            // pages into L2 now so that its loads hit L2.
            const long long nxt = (long long)cta + p.wave;
            if (nxt < (long long)p.B * p.HG * p.n_split) {
              const int n2 = (int)nxt;
              const int sp2 = n2 % p.n_split, hg2 = (n2 / p.n_split) % p.HG;
              const int b2 = n2 / (p.n_split * p.HG);
              DecodeWindow w2;
              if (decode_window(p, b2, w2)) {
                int lg2[2];
                const int n_lg2 = decode_split_pages(p, b2, w2, sp2, lg2);
                for (int i2 = 0; i2 < n_lg2; ++i2) {
                  const int ph2 = decode_page(p, b2, lg2[i2]);
                  if (ph2 < 0) continue;
                  for (int c2 = 0; c2 < Lay::KV_CH; ++c2)
                    tma_prefetch_2d(&tm_kv, c2 * 64, ph2 * 128);
                }
                for (int c2 = 0; c2 < Lay::KV_CH; ++c2)
                  tma_prefetch_3d(&tm_q, c2 * 64, hg2 * 128, b2);
              }
            }
          }
        }
        if (issued < Lay::KV_CH) break;
        // V columns 0..255 (boxes 0..3) again: page A's into the Q slots, free
        // once S is done; page B's into the K_A slots, free once O half 1's
        // page-A products (which read boxes 4..7 there) are done.  Box e goes
        // to stage e.
        if (!mbar_wait(bar(Lay::B_S_FULL), 0, abort_flag, status, 1)) break;
        mbar_arrive_expect_tx(bar(Lay::B_VA_FULL), 4 * kbox);
        for (int e = 0; e < 4; ++e)
          load_k(ring + e * Lay::STAGE + koff, bar(Lay::B_VA_FULL), e, phys_a, true);
        va = true;
        if (!two) break;
        if (!mbar_wait(bar(Lay::B_KA_FREE), 0, abort_flag, status, 1)) break;
        mbar_arrive_expect_tx(bar(Lay::B_VB_FULL), 4 * kbox);
        for (int e = 0; e < 4; ++e)
          load_k(ring + e * Lay::STAGE + Lay::CHUNK + koff, bar(Lay::B_VB_FULL), e, phys_b, true);
        vb = true;
      } while (false);
      // every copy issued lands before the CTA exits
      for (int s = 0; s < Lay::NST; ++s) {
        int last = -1;  // newest S stage issued into ring stage s
        for (int i = 0; i < issued; ++i)
          if (decode_s_stage(i) == s) last = i;
        if (last >= 0) mbar_wait_drain(bar(Lay::B_FULL + s), decode_s_round(last) & 1);
      }
      if (va) mbar_wait_drain(bar(Lay::B_VA_FULL), 0);
      if (vb) mbar_wait_drain(bar(Lay::B_VB_FULL), 0);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, two ? 256 : 128, false);
      const uint32_t id_o = idesc_bf16_f32(128, 256, true);
      const uint32_t o_tm = tmem + Lay::TM_O;
      bool ok = true;
      for (int i = 0; i < Lay::KV_CH; ++i) {
        const int st = decode_s_stage(i);
        if (!(ok = mbar_wait(bar(Lay::B_FULL + st), decode_s_round(i) & 1, abort_flag, status, 1)))
          break;
        if (FP8 && !(ok = mbar_wait(bar(Lay::B_CONV + st), decode_s_round(i) & 1, abort_flag,
                                    status, 1)))
          break;
        tc_fence_after();
        const uint32_t base = ring + st * Lay::STAGE;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // A: the Q box; B: the K_A box and the K_B box right after it, one
          // K-major operand of 256 rows.
          const uint64_t adesc = sdesc_sw128(base + kk * 32, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(base + Lay::CHUNK + kk * 32, 16, 1024);
          mma_ss(tmem, adesc, bdesc, id_s, (i > 0 || kk > 0) ? 1u : 0u);
        }
        if (i < Lay::KV_CH - Lay::N_KEEP) mma_commit(bar(Lay::B_EMPTY + st));  // else kept
      }
      if (ok) {
        mma_commit(bar(Lay::B_S_FULL));
        ok = mbar_wait(bar(Lay::B_P_FULL), 0, abort_flag, status, 1);
      }
      if constexpr (FP8) {
        // O in halves of 256 columns through TMEM columns [256, 512): O half
        // = P V[:, 256 columns]: V rows (keys) 16kk .. 16kk+15 of page A (then
        // B) across four 64-column boxes one STAGE apart, MN-major; the P_A /
        // P_B words of those keys are TMEM columns 8kk .. (128 + 8kk ..).
        auto pv_page = [&](uint32_t v_base, uint32_t p_col, bool first) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(o_tm, tmem + p_col + kk * 8, sdesc_sw128(v_base + kk * 2048, Lay::STAGE, 1024),
                   id_o, (!first || kk > 0) ? 1u : 0u);
        };
        if (ok) {  // half 1 (columns 256..511): the kept S stages
          tc_fence_after();
          pv_page(ring + Lay::CHUNK, 0, true);
          mma_commit(bar(Lay::B_KA_FREE));  // the K_A slots may take page B's V boxes 0..3
          if (two) pv_page(ring + 2 * Lay::CHUNK, 128, false);
          mma_commit(bar(Lay::B_O_FULL));
          ok = mbar_wait(bar(Lay::B_VA_FULL), 0, abort_flag, status, 1) &&
               mbar_wait(bar(Lay::B_VA_CONV), 0, abort_flag, status, 1) &&
               mbar_wait(bar(Lay::B_O_EMPTY), 0, abort_flag, status, 1);
        }
        if (ok) {  // half 0 (columns 0..255): the reloaded boxes
          tc_fence_after();
          pv_page(ring, 0, true);
          if (two && (ok = mbar_wait(bar(Lay::B_VB_FULL), 0, abort_flag, status, 1) &&
                           mbar_wait(bar(Lay::B_VB_CONV), 0, abort_flag, status, 1))) {
            tc_fence_after();
            pv_page(ring + Lay::CHUNK, 128, false);
          }
          if (ok) mma_commit(bar(Lay::B_O_FULL));
        }
      } else {
        // O in quarters of 128 columns: quarter q (V columns 128q .., boxes 2q
        // and 2q+1) goes to TMEM region q & 1 (columns 256 + 128 (q & 1) ..),
        // so that a quarter's products run while the output warps read the
        // quarter before.  Quarters 3 and 2 (boxes 4..7: the kept S stages,
        // box e in stage e - 4) first, then 1 and 0 (boxes 0..3 reloaded, box e
        // in stage e: page A's into the Q slots, page B's into the K_A slots)
        // as the output warps finish reading 3 and 2.  Page A's products over
        // the kept boxes go first, so that the K_A slots are handed back for
        // page B's reload early.  P_A / P_B words of keys 16kk .. 16kk+15 are
        // TMEM columns 8kk .. (128 + 8kk ..).
        const uint32_t id_q = idesc_bf16_f32(128, 128, true);
        auto pv_quarter = [&](int q, bool page_b, bool first) {
          const uint32_t v_base =
              q >= 2 ? ring + (2 * q - 4) * Lay::STAGE + (page_b ? 2 : 1) * Lay::CHUNK
                     : ring + 2 * q * Lay::STAGE + (page_b ? Lay::CHUNK : 0);
          const uint32_t d = o_tm + 128 * (q & 1);
          const uint32_t p_col = page_b ? 128 : 0;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(d, tmem + p_col + kk * 8, sdesc_sw128(v_base + kk * 2048, Lay::STAGE, 1024),
                   id_q, (!first || kk > 0) ? 1u : 0u);
        };
        if (ok) {
          tc_fence_after();
          pv_quarter(3, false, true);
          pv_quarter(2, false, true);
          mma_commit(bar(Lay::B_KA_FREE));  // the K_A slots may take page B's V boxes 0..3
          if (two) pv_quarter(3, true, false);
          mma_commit(bar(Lay::B_O_FULL + 1));  // quarter 3
          if (two) pv_quarter(2, true, false);
          mma_commit(bar(Lay::B_O_FULL + 0));  // quarter 2
          ok = mbar_wait(bar(Lay::B_VA_FULL), 0, abort_flag, status, 1) &&
               mbar_wait(bar(Lay::B_O_EMPTY + 1), 0, abort_flag, status, 1);
        }
        if (ok) {
          tc_fence_after();
          pv_quarter(1, false, true);
          ok = mbar_wait(bar(Lay::B_O_EMPTY + 0), 0, abort_flag, status, 1);
        }
        if (ok) {
          tc_fence_after();
          pv_quarter(0, false, true);
          if (two && (ok = mbar_wait(bar(Lay::B_VB_FULL), 0, abort_flag, status, 1))) {
            tc_fence_after();
            pv_quarter(1, true, false);
            mma_commit(bar(Lay::B_O_FULL + 1));  // quarter 1
            pv_quarter(0, true, false);
            mma_commit(bar(Lay::B_O_FULL + 0));  // quarter 0
          } else if (ok) {
            mma_commit(bar(Lay::B_O_FULL + 1));
            mma_commit(bar(Lay::B_O_FULL + 0));
          }
        }
      }
      mma_commit(bar(Lay::B_DRAIN));
      mbar_wait_drain(bar(Lay::B_DRAIN), 0);
    }
  } else {
    // ----------------------------------------------------- softmax + output
    const int wg = warp >> 2;             // 0: page A, 1: page B
    const int h = threadIdx.x & 127;      // head row within the group
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = wg * 128;
    const int valid_keys = wg == 0 ? valid_a : (two ? valid_b : 0);  // warp-uniform
    const bool partial = valid_keys < 128;
    float* xmax = reinterpret_cast<float*>(smem + Lay::OFF_XCHG);
    float* xsum = xmax + 256;
    const float sl2 = p.scale_log2;
    // FP8: this page's s_j * scale * log2(e) (ksl) and s_j (ksc)
    const float* ksl = reinterpret_cast<const float*>(smem + Lay::OFF_SCALE) + wg * 128;
    const float* ksc = ksl + 256;
    const uint32_t xp = bar(Lay::B_XP + wg);
    uint32_t xp_uses = 0;
    bool done = false;  // this split's LSE slot was written with its result
    do {
      if constexpr (FP8) {
        // this page's token scales, then its K boxes as they land
        const bool mine = wg == 0 || two;
        if (mine) {
          const float sj = __ldg(p.kv_scale + (size_t)(wg == 0 ? phys_a : phys_b) * 128 + h);
          float* st_sc = reinterpret_cast<float*>(smem + Lay::OFF_SCALE) + wg * 128 + h;
          st_sc[0] = sj * sl2;
          st_sc[256] = sj;
        }
        bool okc = true;
        for (int i = 0; i < Lay::KV_CH; ++i) {
          const int st = decode_s_stage(i);
          if (!(okc = mbar_wait(bar(Lay::B_FULL + st), decode_s_round(i) & 1, abort_flag, status,
                                1)))
            break;
          if (mine && !(okc = decode_expand_fp8_box(ring + st * Lay::STAGE + Lay::CHUNK * (1 + wg),
                                                    h, xp, xp_uses, abort_flag, status)))
            break;
          fence_async_shared();
          mbar_arrive(bar(Lay::B_CONV + st));
        }
        if (!okc) break;
      }
      if (!mbar_wait(bar(Lay::B_S_FULL), 0, abort_flag, status, 1)) break;
      tc_fence_after();
      // Pass 1: this page's row max, 64 keys at a time.
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
                float s0 = __uint_as_float(v[jj][k0]), s1 = __uint_as_float(v[jj][k0 + 1]);
                if constexpr (FP8) {  // already in log2 units
                  s0 *= ksl[64 * hf + 32 * jj + k0];
                  s1 *= ksl[64 * hf + 32 * jj + k0 + 1];
                }
                const float x0 = ((vm >> k0) & 1u) ? s0 : -INFINITY;
                const float x1 = ((vm >> (k0 + 1)) & 1u) ? s1 : -INFINITY;
                mx4[a] = fmax3(mx4[a], x0, x1);
              }
          }
        }
      }
      const float mloc = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
      xmax[wg * 128 + h] = mloc;
      mbar_arrive(bar(Lay::B_XCHG));
      if (!mbar_wait(bar(Lay::B_XCHG), 0, abort_flag, status, 1)) break;
      // finite: page A has a key (FP8: the maxima are already in log2 units)
      const float m = fmaxf(mloc, xmax[(wg ^ 1) * 128 + h]) * (FP8 ? 1.f : sl2);
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m, -m);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      // Pass 2: p = exp2(s * scale * log2(e) - m) 32 keys at a time (masked
      // keys: exp2(-inf) = 0), packed to bf16 pairs.  The P words of keys
      // 32ch .. 32ch+31 go to columns 16ch .. 16ch+15 of this page's S
      // columns, which this thread has already read.
      if (valid_keys > 0) {
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32], pk16[16];
          tmem_ld32(t_row + s_col + ch * 32, v);
          tmem_wait_ld();
          const uint32_t vm = partial ? decode_chunk_mask(valid_keys, ch) : 0xffffffffu;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float y0, y1, p0, p1;
            if constexpr (FP8) {
              // y = s * (s_j scale log2 e) - m; the mask after the product, so
              // that a zero s_j never meets -inf
              const uint64_t kl = *reinterpret_cast<const uint64_t*>(ksl + 32 * ch + 2 * c);
              f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])),
                               kl, negm2),
                        y0, y1);
              y0 = ((vm >> (2 * c)) & 1u) ? y0 : -INFINITY;
              y1 = ((vm >> (2 * c + 1)) & 1u) ? y1 : -INFINITY;
            } else {
              const float v0 = ((vm >> (2 * c)) & 1u) ? __uint_as_float(v[2 * c]) : -INFINITY;
              const float v1 =
                  ((vm >> (2 * c + 1)) & 1u) ? __uint_as_float(v[2 * c + 1]) : -INFINITY;
              f2_unpack(f2_fma(f2_pack(v0, v1), sl2x2, negm2), y0, y1);
            }
            if ((c & 7) < kDecodePolyPairsPer8) {
              exp2_poly_x2(y0, y1, p0, p1);
            } else {
              p0 = ex2_approx(y0);
              p1 = ex2_approx(y1);
            }
            acc[c & 3] = f2_add(acc[c & 3], f2_pack(p0, p1));
            if constexpr (FP8)
              pk16[c] = pack_bf16x2(p0 * ksc[32 * ch + 2 * c], p1 * ksc[32 * ch + 2 * c + 1]);
            else
              pk16[c] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_row + s_col + ch * 16, pk16);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(Lay::B_P_FULL));
      float lloc;
      {
        float a0, a1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
        lloc = a0 + a1;
      }
      xsum[wg * 128 + h] = lloc;
      mbar_arrive(bar(Lay::B_XCHG));
      if (!mbar_wait(bar(Lay::B_XCHG), 1, abort_flag, status, 1)) break;
      const float l = lloc + xsum[(wg ^ 1) * 128 + h];
      if constexpr (FP8) {
        // page A's V columns 0..255, reloaded into the Q slots, to bf16: boxes
        // 2wg and 2wg+1 by warpgroup wg (this overlaps the MMAs of O half 1)
        bool okv = mbar_wait(bar(Lay::B_VA_FULL), 0, abort_flag, status, 1);
        for (int e = 2 * wg; e < 2 * wg + 2 && okv; ++e)
          okv = decode_expand_fp8_box(ring + e * Lay::STAGE, h, xp, xp_uses, abort_flag, status);
        if (!okv) break;
        fence_async_shared();
        mbar_arrive(bar(Lay::B_VA_CONV));
      }

      const bool valid = hg * 128 + h < p.H_q;
      const float inv_l = 1.f / l;
      uint4* dst = reinterpret_cast<uint4*>(p.o_part) + cta * (64 * 128) + h;
      // 64 columns of O (registers orr) as fp16 into the row's 8-column groups
      // g0 .. g0+7
      auto emit = [&](const uint32_t (&orr)[2][32], int g0) {
        if (!valid) return;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint32_t* r8 = &orr[g >> 2][(g & 3) * 8];
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            __half2 hv = __floats2half2_rn(__uint_as_float(r8[2 * q]) * inv_l,
                                           __uint_as_float(r8[2 * q + 1]) * inv_l);
            w[q] = *reinterpret_cast<uint32_t*>(&hv);
          }
          dst[(size_t)(g0 + g) * 128] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      };
      bool ok = true;
      if constexpr (FP8) {
        // O half hf (1 first): warpgroup wg takes its 128 columns 128wg .. of
        // the half, i.e. 8-column groups 32hf + 16wg + g of the row.
#pragma unroll 1
        for (int n = 0; n < 2; ++n) {
          const int hf = 1 - n;
          if (!(ok = mbar_wait(bar(Lay::B_O_FULL), n, abort_flag, status, 1))) break;
          tc_fence_after();
          if (n == 1) asm volatile("griddepcontrol.launch_dependents;");
#pragma unroll 1
          for (int part = 0; part < 2; ++part) {  // 64 columns at a time
            uint32_t orr[2][32];
            tmem_ld32(t_row + Lay::TM_O + 128 * wg + 64 * part, orr[0]);
            tmem_ld32(t_row + Lay::TM_O + 128 * wg + 64 * part + 32, orr[1]);
            tmem_wait_ld();
            if (part == 1) {
              tc_fence_before();
              mbar_arrive(bar(Lay::B_O_EMPTY));  // the MMA may reuse the buffer now
            }
            emit(orr, 32 * hf + 16 * wg + 8 * part);
          }
          // page B's V columns 0..255, reloaded into the K_A slots, to bf16
          // (once O half 1 is done, so page A's boxes there are read): boxes
          // 2wg and 2wg+1 by warpgroup wg
          if (n == 0 && two) {
            bool okv = mbar_wait(bar(Lay::B_VB_FULL), 0, abort_flag, status, 1);
            for (int e = 2 * wg; e < 2 * wg + 2 && okv; ++e)
              okv = decode_expand_fp8_box(ring + e * Lay::STAGE + Lay::CHUNK, h, xp, xp_uses,
                                          abort_flag, status);
            if (!(ok = okv)) break;
            fence_async_shared();
            mbar_arrive(bar(Lay::B_VB_CONV));
          }
        }
      } else {
        // O quarter q (3 first) in TMEM region q & 1: warpgroup wg takes its 64
        // columns 64wg .. of the quarter, i.e. 8-column groups 16q + 8wg + g of
        // the row; reading quarters 3 and 2 frees their region for 1 and 0.
#pragma unroll 1
        for (int n = 0; n < 4; ++n) {
          const int q = 3 - n, r = q & 1;
          if (!(ok = mbar_wait(bar(Lay::B_O_FULL + r), n >> 1, abort_flag, status, 1))) break;
          tc_fence_after();
          if (n == 3) asm volatile("griddepcontrol.launch_dependents;");
          uint32_t orr[2][32];
          tmem_ld32(t_row + Lay::TM_O + 128 * r + 64 * wg, orr[0]);
          tmem_ld32(t_row + Lay::TM_O + 128 * r + 64 * wg + 32, orr[1]);
          tmem_wait_ld();
          if (n < 2) {
            tc_fence_before();
            mbar_arrive(bar(Lay::B_O_EMPTY + r));  // the MMA may write quarter q - 2 here
          }
          emit(orr, 16 * q + 8 * wg);
        }
      }
      if (ok && valid && wg == 0) p.lse_part[cta * 128 + h] = (m + __log2f(l)) * kLn2;
      done = ok;
    } while (false);
    // A wait that gave up leaves this split's partial O unfinished: mark the
    // slot NaN, so that the merge writes NaN for these heads rather than mix
    // in what an earlier call left in the workspace.
    if (!done && wg == 0) p.lse_part[cta * 128 + h] = __int_as_float(0x7fc00000);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

// Merge: one CTA per (sequence, 8 heads); thread (head hh, column group pair
// gp) merges the 8-column groups gp and gp + 32 of its head, reading 16 bytes
// of each per split, so that a warp's reads of one group of one split are
// four runs of 128 contiguous bytes, and all of a thread's loads are in
// flight at once.  Two groups per thread keep every CTA of the 32-sequence
// workload resident in one wave (512 threads per CTA at one group each did
// not fit in the register file and ran a second wave).  Launched as a
// programmatic dependent of the split kernel; it waits for the split
// kernel's results before reading.  Splits whose LSE is -inf are empty and
// contribute nothing (their partial O is never read into the sum); a NaN LSE
// marks a split that gave up on a wait, and makes the head's O and LSE NaN.
constexpr int kMergeHeads = 8;
constexpr int kMergeGroups = 2;  // 8-column groups per thread
constexpr int kMergeThreads = (kDecodeDv / 8 / kMergeGroups) * kMergeHeads;  // 256
constexpr int kMergeBatch = 4;

// four CTAs per SM: 148 x 4 slots hold the 512 CTAs of the 32-sequence workload.
// PLAN: the partials of the long-window kernel (a unit's slots from its plan)
// instead of the split kernel's n_split per (row, head group).
template <bool PLAN>
__global__ void __launch_bounds__(kMergeThreads, 4)
    ssa_decode_merge_kernel(const DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int heads = (p.H_q + kMergeHeads - 1) / kMergeHeads;
  const int b = blockIdx.x / heads;
  const int hh = threadIdx.x % kMergeHeads, gp = threadIdx.x / kMergeHeads;
  const int h = (blockIdx.x % heads) * kMergeHeads + hh;
  if (h >= p.H_q) return;
  const int hg = h >> 7, hr = h & 127;
  constexpr int kGroupStride = kDecodeDv / 8 / kMergeGroups;  // 32: groups gp, gp + 32
  size_t cta0 = ((size_t)b * p.HG + hg) * p.n_split;
  int n = p.n_split;
  if constexpr (PLAN) {
    const int* us = p.plan + p.B * p.HG + 1 + 2 * (b * p.HG + hg);
    cta0 = (size_t)us[0];
    n = us[1];
  }
  const float* lsep = p.lse_part + cta0 * 128 + hr;  // split stride 128
  const uint4* op = reinterpret_cast<const uint4*>(p.o_part) + (cta0 * 64 + gp) * 128 + hr;
  constexpr size_t kSplitStride = 64 * 128;  // uint4 per split
  // One pass, kMergeBatch splits at a time: a batch's LSEs and partial O are
  // loaded together (one round trip to L2 for the usual four splits), and
  // the running max only rescales what earlier batches summed.
  float lmax = -INFINITY;
  float acc[kMergeGroups][8];
#pragma unroll
  for (int q = 0; q < kMergeGroups; ++q)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[q][e] = 0.f;
  float denom = 0.f;
  bool poisoned = false;  // a split gave up (its LSE slot is NaN)
  for (int s0 = 0; s0 < n; s0 += kMergeBatch) {
    float ls[kMergeBatch];
    uint4 raw[kMergeBatch][kMergeGroups];
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      ls[j] = -INFINITY;
      if (s0 + j < n) {
        ls[j] = __ldg(lsep + (size_t)(s0 + j) * 128);
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q)
          raw[j][q] = __ldg(op + (size_t)(s0 + j) * kSplitStride + q * kGroupStride * 128);
      }
    }
    float bmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      poisoned |= ls[j] != ls[j];
      bmax = fmaxf(bmax, ls[j]);  // fmaxf skips a NaN operand
    }
    if (bmax == -INFINITY) continue;  // only empty splits in this batch
    if (bmax > lmax) {
      const float r = __expf(lmax - bmax);  // 0 while nothing is summed yet
      denom *= r;
#pragma unroll
      for (int q = 0; q < kMergeGroups; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[q][e] *= r;
      lmax = bmax;
    }
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      // empty split (its partial O was never written) or one that gave up
      if (ls[j] == -INFINITY || ls[j] != ls[j]) continue;
      const float wgt = __expf(ls[j] - lmax);
      denom += wgt;
#pragma unroll
      for (int q = 0; q < kMergeGroups; ++q) {
        const __half2* hv = reinterpret_cast<const __half2*>(&raw[j][q]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          acc[q][2 * e] += wgt * f.x;
          acc[q][2 * e + 1] += wgt * f.y;
        }
      }
    }
  }
  const float inv = poisoned ? __int_as_float(0x7fc00000) : (denom > 0.f ? 1.f / denom : 0.f);
  uint4* orow = reinterpret_cast<uint4*>(p.o + ((size_t)b * p.H_q + h) * kDecodeDv);
#pragma unroll
  for (int q = 0; q < kMergeGroups; ++q) {
    uint4 pk;
    pk.x = pack_bf16x2(acc[q][0] * inv, acc[q][1] * inv);
    pk.y = pack_bf16x2(acc[q][2] * inv, acc[q][3] * inv);
    pk.z = pack_bf16x2(acc[q][4] * inv, acc[q][5] * inv);
    pk.w = pack_bf16x2(acc[q][6] * inv, acc[q][7] * inv);
    orow[gp + q * kGroupStride] = pk;
  }
  if (gp == 0)
    p.lse[(size_t)b * p.H_q + h] = poisoned ? __int_as_float(0x7fc00000)
                                   : denom > 0.f ? lmax + __logf(denom) : -INFINITY;
}

}  // namespace loza
