/*
 * ssa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU reference for the streaming sparse
 * attention (SSA) that LoZA puts into half of a model's attention layers.
 * It exists to check the CUDA library, and nothing in the product path may
 * load it: only the tests, the smoke check and the benchmark's CPU-baseline
 * / reference arm do.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes, in double precision, with no tiling, no online softmax
 * and no reordering beyond the plain definition:
 *
 *   Masked softmax attention ("LoZA：ZigZag稀疏注意力机制", §2.1 问题形式化,
 *   the second formula: numerator and denominator both summed over the j
 *   with M_ij = 1), with the SSA mask of the QbitAI LoZA article (the
 *   paragraph on the 1024-token sparse window: one global block that keeps
 *   the overall context plus seven local blocks, 128 tokens per block):
 *
 *     J(i) = { j <= i : floor(j/blk) in W(floor(i/blk)) }
 *     W(b) = {0 .. n_sink-1}  U  {max(n_sink, b-n_local+1) .. b}
 *
 *   The global block is block 0, the tokens at the start of the sequence
 *   (LongCat LSA article, 机制 1 流感知索引: sink tokens are the fixed
 *   tokens at the head of the sequence).
 *
 *     s_ij  = scale * sum_c q_ic k_jc                 (j in J(i))
 *     m_i   = max_j s_ij
 *     l_i   = sum_j exp(s_ij - m_i)                   (row max subtracted,
 *                                CSA/HCA tutorial §7.1 数值不稳定问题)
 *     O_i   = sum_j exp(s_ij - m_i) v_j / l_i
 *     LSE_i = m_i + ln l_i      (natural log of sum_j exp(s_ij), scale included)
 *
 *   Decode is the same definition for the single query at position
 *   t = seq_len - 1 of each sequence, with key row j read from the paged cache
 *   at physical row page_table[j / page_size] * page_size + j % page_size,
 *   v_j = the first dv entries of that row, and every query head attending the
 *   same (latent) key/value rows.
 *
 * Inputs are either float64 or bfloat16 bit patterns (uint16, widened exactly
 * to double).  Outputs are float64.
 *
 * Parity status of every function here: pinned by the tests (closed-form mask
 * counts, reduction to textbook causal attention, q = 0 => LSE = ln|J(i)|,
 * constant-V and identical-key invariants, a materialised-mask brute force on
 * tiny inputs, page-permutation invariance and decode == prefill row t).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ELT_F64 0
#define ELT_BF16 1

static double widen(const void* base, int64_t idx, int elt) {
  if (elt == ELT_F64) return ((const double*)base)[idx];
  uint32_t bits = ((uint32_t)((const uint16_t*)base)[idx]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Block kb is in the window W(qb) of query block qb (causality is applied per token). */
int oracle_ssa_block_in_window(int64_t qb, int64_t kb, int64_t n_sink, int64_t n_local) {
  if (kb < 0 || kb > qb) return 0;
  if (kb < n_sink) return 1;
  int64_t lo = qb - n_local + 1;
  if (lo < n_sink) lo = n_sink;
  return kb >= lo;
}

/* M_ij of the SSA mask. */
int oracle_ssa_mask(int64_t i, int64_t j, int64_t blk, int64_t n_sink, int64_t n_local) {
  if (j < 0 || j > i) return 0;
  return oracle_ssa_block_in_window(i / blk, j / blk, n_sink, n_local);
}

/* |J(i)|, counted token by token from the mask. */
int64_t oracle_ssa_row_count(int64_t i, int64_t blk, int64_t n_sink, int64_t n_local) {
  int64_t n = 0;
  for (int64_t j = 0; j <= i; ++j) n += oracle_ssa_mask(i, j, blk, n_sink, n_local);
  return n;
}

/*
 * Key blocks that query block qb touches: kb is listed iff some query i of
 * block qb (i < seq_len) and some key j of block kb have M_ij = 1.  Derived
 * by scanning the mask, not from the window formula.  Ascending order.
 * Returns the count (or -1 if more than cap).
 */
int64_t oracle_ssa_key_blocks(int64_t qb, int64_t blk, int64_t seq_len, int64_t n_sink,
                              int64_t n_local, int64_t* out, int64_t cap) {
  int64_t n = 0;
  int64_t i_hi = (qb + 1) * blk - 1;
  if (i_hi > seq_len - 1) i_hi = seq_len - 1;
  for (int64_t kb = 0; kb <= qb; ++kb) {
    int hit = 0;
    for (int64_t i = qb * blk; i <= i_hi && !hit; ++i)
      for (int64_t j = kb * blk; j < (kb + 1) * blk && j < seq_len && !hit; ++j)
        hit = oracle_ssa_mask(i, j, blk, n_sink, n_local);
    if (hit) {
      if (n >= cap) return -1;
      out[n++] = kb;
    }
  }
  return n;
}

/*
 * One query row i against the keys of its own sequence.
 *   q_row: dqk elements.  Key j lives at row key_row(j) of k_base / v_base,
 *   with row strides k_ld / v_ld (elements).  If page_table is non-NULL the
 *   key row is page_table[j / blk] * blk + j % blk (paged cache), else j.
 */
static int attend_row(const void* q, int64_t q_off, int q_elt, const void* k, const void* v,
                      int kv_elt, int64_t kv_off_k, int64_t kv_off_v, int64_t k_ld, int64_t v_ld,
                      const int32_t* page_table, int64_t n_pages, int64_t i, int64_t blk,
                      int64_t n_sink, int64_t n_local, const int32_t* extra, int64_t n_extra,
                      int dqk, int dv, double scale, double* s_buf, int64_t* j_buf, double* qd,
                      double* o_out, double* lse_out) {
  for (int c = 0; c < dqk; ++c) qd[c] = widen(q, q_off + c, q_elt);

  /* pass 1: every score over J(i), and the row max */
  int64_t n = 0;
  double m = -INFINITY;
  int64_t qb = i / blk;
  for (int64_t kb = 0; kb <= qb; ++kb) {
    /* block kb is attended if it is in the SSA window or in the extra list */
    int in = oracle_ssa_block_in_window(qb, kb, n_sink, n_local);
    for (int64_t e = 0; e < n_extra && !in; ++e) in = (extra[e] == kb);
    if (!in) continue;
    int64_t j_end = (kb + 1) * blk - 1;
    if (j_end > i) j_end = i;
    for (int64_t j = kb * blk; j <= j_end; ++j) {
      int64_t row = j;
      if (page_table) {
        int64_t phys = page_table[j / blk];
        if (phys < 0 || phys >= n_pages) return -1;
        row = phys * blk + j % blk;
      }
      double dot = 0.0;
      for (int c = 0; c < dqk; ++c) dot += qd[c] * widen(k, kv_off_k + row * k_ld + c, kv_elt);
      double s = scale * dot;
      s_buf[n] = s;
      j_buf[n] = row;
      ++n;
      if (s > m) m = s;
    }
  }

  /* pass 2: l_i and the weighted sum of values */
  double l = 0.0;
  for (int c = 0; c < dv; ++c) o_out[c] = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    double p = exp(s_buf[t] - m);
    l += p;
    int64_t row = j_buf[t];
    for (int c = 0; c < dv; ++c) o_out[c] += p * widen(v, kv_off_v + row * v_ld + c, kv_elt);
  }
  for (int c = 0; c < dv; ++c) o_out[c] /= l;
  *lse_out = m + log(l);
  return 0;
}

static int64_t max_keys(int64_t longest_row, int64_t blk, int64_t n_sink, int64_t n_local) {
  int64_t cap = (n_sink + n_local) * blk;
  if (cap > longest_row || cap <= 0) cap = longest_row;
  return cap;
}

/*
 * Dense prefill, rows selected by flat index r = (b*H + h)*L + i.
 * q, k: [B,H,L,dqk]; v: [B,H,L,dv]; o: [n_rows, dv]; lse: [n_rows].
 */
int oracle_ssa_prefill_rows(const void* q, const void* k, const void* v, int elt, int64_t B,
                            int64_t H, int64_t L, int dqk, int dv, int64_t blk, int64_t n_sink,
                            int64_t n_local, double scale, const int64_t* rows, int64_t n_rows,
                            double* o, double* lse) {
  int64_t cap = max_keys(L, blk, n_sink, n_local);
  int err = 0;
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * cap);
    int64_t* j_buf = (int64_t*)malloc(sizeof(int64_t) * cap);
    double* qd = (double*)malloc(sizeof(double) * dqk);
#pragma omp for schedule(dynamic, 16)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t flat = rows[r];
      if (flat < 0 || flat >= B * H * L) {
#pragma omp atomic write
        err = -2;
        continue;
      }
      int64_t bh = flat / L, i = flat % L;
      int rc = attend_row(q, flat * dqk, elt, k, v, elt, bh * L * dqk, bh * L * dv, dqk, dv, NULL,
                          0, i, blk, n_sink, n_local, NULL, 0, dqk, dv, scale, s_buf, j_buf, qd,
                          o + r * dv, lse + r);
      if (rc) {
#pragma omp atomic write
        err = rc;
      }
    }
    free(s_buf);
    free(j_buf);
    free(qd);
  }
  return err;
}

/*
 * Packed variable-length prefill.  q, k: [H,total,dqk]; v: [H,total,dv];
 * cu_seqlens: [n_seqs+1] prefix offsets; rows are flat r = h*total + token.
 * Block indices count from each sequence's own first token.
 */
int oracle_ssa_prefill_varlen_rows(const void* q, const void* k, const void* v, int elt,
                                   const int32_t* cu_seqlens, int64_t n_seqs, int64_t total,
                                   int64_t H, int dqk, int dv, int64_t blk, int64_t n_sink,
                                   int64_t n_local, double scale, const int64_t* rows,
                                   int64_t n_rows, double* o, double* lse) {
  int64_t longest = 1;
  for (int64_t s = 0; s < n_seqs; ++s) {
    int64_t len = cu_seqlens[s + 1] - cu_seqlens[s];
    if (len < 0) return -3;
    if (len > longest) longest = len;
  }
  if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != total) return -3;
  int64_t cap = max_keys(longest, blk, n_sink, n_local);
  int err = 0;
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * cap);
    int64_t* j_buf = (int64_t*)malloc(sizeof(int64_t) * cap);
    double* qd = (double*)malloc(sizeof(double) * dqk);
#pragma omp for schedule(dynamic, 16)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t flat = rows[r];
      if (flat < 0 || flat >= H * total) {
#pragma omp atomic write
        err = -2;
        continue;
      }
      int64_t h = flat / total, tok = flat % total;
      int64_t s = 0;
      while (!(cu_seqlens[s] <= tok && tok < cu_seqlens[s + 1])) ++s;
      int64_t start = cu_seqlens[s];
      int64_t i = tok - start;
      int rc = attend_row(q, flat * dqk, elt, k, v, elt, (h * total + start) * dqk,
                          (h * total + start) * dv, dqk, dv, NULL, 0, i, blk, n_sink, n_local,
                          NULL, 0, dqk, dv, scale, s_buf, j_buf, qd, o + r * dv, lse + r);
      if (rc) {
#pragma omp atomic write
        err = rc;
      }
    }
    free(s_buf);
    free(j_buf);
    free(qd);
  }
  return err;
}

/*
 * Paged decode, one query token per sequence.  q: [B,Hq,dqk]; kv:
 * [n_pages, page_size, dqk] (value = first dv entries of each row);
 * page_table: [B, max_pages]; seq_lens: [B] (including the new token).
 * rows are flat r = b*Hq + h; o: [n_rows, dv]; lse: [n_rows].
 * Returns -1 for a page id outside [0, n_pages), -4 for a bad seq_len.
 */
static int decode_rows(const void* q, const void* kv, int elt, const int32_t* page_table,
                       const int32_t* seq_lens, const int32_t* extra_pages, int64_t max_extra,
                       int64_t q_len, int64_t B, int64_t Hq, int dqk, int dv, int64_t page_size,
                       int64_t max_pages, int64_t n_pages, int64_t n_sink, int64_t n_local,
                       double scale, const int64_t* rows, int64_t n_rows, double* o,
                       double* lse) {
  int64_t longest = 1;
  if (q_len < 1) return -4;
  for (int64_t b = 0; b < B; ++b) {
    if (seq_lens[b] < q_len || seq_lens[b] > max_pages * page_size) return -4;
    if (seq_lens[b] > longest) longest = seq_lens[b];
  }
  int64_t cap = max_keys(longest, page_size, n_sink + max_extra, n_local);
  int err = 0;
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * cap);
    int64_t* j_buf = (int64_t*)malloc(sizeof(int64_t) * cap);
    double* qd = (double*)malloc(sizeof(double) * dqk);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t flat = rows[r];
      if (flat < 0 || flat >= B * q_len * Hq) {
#pragma omp atomic write
        err = -2;
        continue;
      }
      /* row flat = (b * q_len + token) * Hq + h; token k of sequence b sits at
         position seq_len - q_len + k */
      int64_t b = flat / (q_len * Hq);
      int64_t token = (flat / Hq) % q_len;
      int64_t t = (int64_t)seq_lens[b] - q_len + token;
      int rc = attend_row(q, flat * dqk, elt, kv, kv, elt, 0, 0, dqk, dqk,
                          page_table + b * max_pages, n_pages, t, page_size, n_sink, n_local,
                          extra_pages ? extra_pages + b * max_extra : NULL, max_extra, dqk, dv,
                          scale, s_buf, j_buf, qd, o + r * dv, lse + r);
      if (rc) {
#pragma omp atomic write
        err = rc;
      }
    }
    free(s_buf);
    free(j_buf);
    free(qd);
  }
  return err;
}

int oracle_ssa_decode_rows(const void* q, const void* kv, int elt, const int32_t* page_table,
                           const int32_t* seq_lens, int64_t B, int64_t Hq, int dqk, int dv,
                           int64_t page_size, int64_t max_pages, int64_t n_pages, int64_t n_sink,
                           int64_t n_local, double scale, const int64_t* rows, int64_t n_rows,
                           double* o, double* lse) {
  return decode_rows(q, kv, elt, page_table, seq_lens, NULL, 0, 1, B, Hq, dqk, dv, page_size,
                     max_pages, n_pages, n_sink, n_local, scale, rows, n_rows, o, lse);
}

/*
 * Paged decode with q_len query tokens per sequence (a speculative or
 * multi-token step): token k of sequence b is the query at position
 * t = seq_len - q_len + k, attending J(t) as defined at the top of this file
 * -- the same mask applied to each query position, so the new tokens see
 * each other causally.  q: [B, q_len, Hq, dqk]; rows are flat
 * r = (b*q_len + k)*Hq + h; seq_lens[b] >= q_len.  Other arguments as
 * oracle_ssa_decode_rows.
 */
int oracle_ssa_decode_mtp_rows(const void* q, const void* kv, int elt, const int32_t* page_table,
                               const int32_t* seq_lens, int64_t q_len, int64_t B, int64_t Hq,
                               int dqk, int dv, int64_t page_size, int64_t max_pages,
                               int64_t n_pages, int64_t n_sink, int64_t n_local, double scale,
                               const int64_t* rows, int64_t n_rows, double* o, double* lse) {
  return decode_rows(q, kv, elt, page_table, seq_lens, NULL, 0, q_len, B, Hq, dqk, dv, page_size,
                     max_pages, n_pages, n_sink, n_local, scale, rows, n_rows, o, lse);
}

/*
 * Decode over the SSA window plus selected pages: the fixed sink + sliding
 * window budget plus pages chosen per sequence by a page-level indexer
 * (LongCat sparse-attention article, 机制 1 流感知索引 and 机制 3 分层索引,
 * pages of P = 128 tokens).  extra_pages: [B, max_extra] logical page ids
 * of each sequence; any entry that is negative, past the query's page, or
 * already in the window adds nothing, and a page listed twice counts once:
 * the keys are J(t) = { j <= t : page(j) in W(page(t)) or page(j) listed }.
 */
int oracle_ssa_decode_sel_rows(const void* q, const void* kv, int elt, const int32_t* page_table,
                               const int32_t* seq_lens, const int32_t* extra_pages,
                               int64_t max_extra, int64_t B, int64_t Hq, int dqk, int dv,
                               int64_t page_size, int64_t max_pages, int64_t n_pages,
                               int64_t n_sink, int64_t n_local, double scale, const int64_t* rows,
                               int64_t n_rows, double* o, double* lse) {
  return decode_rows(q, kv, elt, page_table, seq_lens, extra_pages, max_extra, 1, B, Hq, dqk, dv,
                     page_size, max_pages, n_pages, n_sink, n_local, scale, rows, n_rows, o, lse);
}

/*
 * Backward pass of the dense SSA prefill: the gradients of a loss whose
 * gradient with respect to O is dO.  Written from the definition of the
 * forward pass above (softmax over J(i) of the scaled scores, "LoZA：ZigZag
 * 稀疏注意力机制" §2.1), differentiated by the chain rule:
 *
 *   P_ij  = exp(s_ij - m_i) / l_i                      (j in J(i))
 *   dP_ij = sum_c dO_ic v_jc                           (dL/dP_ij)
 *   D_i   = sum_j P_ij dP_ij                           (= dO_i . O_i)
 *   dS_ij = P_ij (dP_ij - D_i)                         (dL/ds_ij, softmax Jacobian)
 *   dQ_i  = scale sum_j dS_ij k_j
 *   dK_j  = scale sum_i dS_ij q_i                      (over the i with j in J(i))
 *   dV_j  = sum_i P_ij dO_i
 *
 * q, k, dout: [B,H,L,dqk] / [B,H,L,dv] as for the forward; outputs float64
 * dq [B,H,L,dqk], dk [B,H,L,dqk], dv [B,H,L,dv].  Planes (b, h) run in
 * parallel; inside a plane rows are visited in order and dK, dV accumulate
 * in that order.
 */
int oracle_ssa_prefill_bwd(const void* q, const void* k, const void* v, const void* dout, int elt,
                           int64_t B, int64_t H, int64_t L, int dqk, int dv, int64_t blk,
                           int64_t n_sink, int64_t n_local, double scale, double* dq, double* dk,
                           double* dvv) {
  int64_t cap = max_keys(L, blk, n_sink, n_local);
  int err = 0;
  memset(dk, 0, sizeof(double) * B * H * L * dqk);
  memset(dvv, 0, sizeof(double) * B * H * L * dv);
#pragma omp parallel
  {
    double* s_buf = (double*)malloc(sizeof(double) * cap);
    double* dp_buf = (double*)malloc(sizeof(double) * cap);
    int64_t* j_buf = (int64_t*)malloc(sizeof(int64_t) * cap);
    double* qd = (double*)malloc(sizeof(double) * dqk);
    double* gd = (double*)malloc(sizeof(double) * dv);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
      for (int64_t i = 0; i < L; ++i) {
        const int64_t qrow = bh * L + i;
        for (int c = 0; c < dqk; ++c) qd[c] = widen(q, qrow * dqk + c, elt);
        for (int c = 0; c < dv; ++c) gd[c] = widen(dout, qrow * dv + c, elt);
        /* scores over J(i) and the row max */
        int64_t n = 0;
        double m = -INFINITY;
        const int64_t qb = i / blk;
        for (int64_t j = 0; j <= i; ++j) {
          if (!oracle_ssa_block_in_window(qb, j / blk, n_sink, n_local)) continue;
          const int64_t krow = bh * L + j;
          double dot = 0.0;
          for (int c = 0; c < dqk; ++c) dot += qd[c] * widen(k, krow * dqk + c, elt);
          s_buf[n] = scale * dot;
          j_buf[n] = krow;
          if (s_buf[n] > m) m = s_buf[n];
          ++n;
        }
        if (n > cap) {
#pragma omp atomic write
          err = -3;
          break;
        }
        /* P_ij, dP_ij and D_i */
        double l = 0.0;
        for (int64_t t = 0; t < n; ++t) l += exp(s_buf[t] - m);
        double D = 0.0;
        for (int64_t t = 0; t < n; ++t) {
          s_buf[t] = exp(s_buf[t] - m) / l; /* now P_ij */
          double dot = 0.0;
          for (int c = 0; c < dv; ++c) dot += gd[c] * widen(v, j_buf[t] * dv + c, elt);
          dp_buf[t] = dot;
          D += s_buf[t] * dot;
        }
        /* dS_ij, then the three gradients */
        for (int c = 0; c < dqk; ++c) dq[qrow * dqk + c] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
          const double p = s_buf[t];
          const double ds = p * (dp_buf[t] - D);
          const int64_t krow = j_buf[t];
          for (int c = 0; c < dqk; ++c) {
            dq[qrow * dqk + c] += scale * ds * widen(k, krow * dqk + c, elt);
            dk[krow * dqk + c] += scale * ds * qd[c];
          }
          for (int c = 0; c < dv; ++c) dvv[krow * dv + c] += p * gd[c];
        }
      }
    }
    free(s_buf);
    free(dp_buf);
    free(j_buf);
    free(qd);
    free(gd);
  }
  return err;
}

/* Threads the oracle's parallel regions use (for reporting the CPU baseline). */
int oracle_ssa_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    n = omp_get_num_threads();
  }
  return n;
}
