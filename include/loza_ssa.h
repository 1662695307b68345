/*
 * loza_ssa.h -- C ABI of libloza_ssa.so: streaming sparse attention (SSA) for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (all entry points): masked softmax attention
 *
 *     O_i = sum_{j : M_ij = 1} exp(scale * q_i.k_j) v_j / sum_{j : M_ij = 1} exp(scale * q_i.k_j)
 *
 * ("LoZA：ZigZag稀疏注意力机制", §2.1 问题形式化, second formula) with the SSA
 * mask of LongCat's LoZA (QbitAI article on LoZA, paragraph on the 1024-token
 * sparse window: one global block plus seven local blocks, 128 tokens each):
 *
 *     M_ij = 1  iff  j <= i  and  floor(j/block) in W(floor(i/block))
 *     W(b) = {0 .. n_sink-1}  U  {max(n_sink, b-n_local+1) .. b}
 *
 * The defaults n_sink = 1, n_local = 7, block = 128 give the paper's window:
 * the global block 0 plus the query's own block and the six before it.  The
 * global block sits at the start of the sequence (LongCat LSA article,
 * 机制 1 流感知索引: sink tokens are the first tokens of the sequence).
 * Alongside O every call writes LSE_i = ln sum_{j : M_ij = 1} exp(scale * q_i.k_j)
 * (natural log, scale included) in fp32.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, caller-owned, row-major and
 *     contiguous.  bf16 tensors hold IEEE bfloat16; lse is fp32.
 *   - bf16 tensor pointers must be 16-byte aligned, lse 4-byte aligned; the
 *     outputs the prefill and the backward write with 32-byte stores (o of
 *     loza_ssa_prefill and loza_ssa_prefill_varlen, dq / dk / dv of the
 *     backward calls) 32-byte aligned.
 *   - Work is enqueued on `stream` and is asynchronous; no call synchronises
 *     the device, and no call allocates device memory (loza_ssa_prefill_host
 *     creates its two copy streams once per device, and CUDA events per call).  Inputs are never
 *     modified.  Calls on different streams may run concurrently.
 *   - On any non-zero status nothing has been launched, except where an entry
 *     point says otherwise (loza_ssa_decode_layers, loza_ssa_prefill_host).
 *   - Errors found by the kernels themselves (a page id outside the pool, a
 *     sequence length outside the page table, bad cu_seqlens, a pipeline wait
 *     that timed out) are recorded in a per-device status word instead of
 *     faulting; read it with loza_ssa_get_last_device_status().
 *
 * Status codes (return values) are the LOZA_SSA_* values below.
 */
#ifndef LOZA_SSA_H
#define LOZA_SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* loza_ssa_stream_t;

enum {
  LOZA_SSA_OK = 0,
  LOZA_SSA_ERR_NULL = -1,           /* a required pointer is NULL                              */
  LOZA_SSA_ERR_SHAPE = -2,          /* a size is out of range (<= 0, too large), scale not finite */
  LOZA_SSA_ERR_HEAD_DIM = -3,       /* (d_qk, d_v) not supported by the kernels                 */
  LOZA_SSA_ERR_BLOCK = -4,          /* block / page_size other than 128                         */
  LOZA_SSA_ERR_WINDOW = -5,         /* n_sink < 0, n_local < 1, or too many window blocks      */
  LOZA_SSA_ERR_ALIGN = -6,          /* a pointer is not aligned as required                     */
  LOZA_SSA_ERR_WORKSPACE = -7,      /* workspace missing or smaller than the size query says    */
  LOZA_SSA_ERR_CUDA = -8,           /* a CUDA runtime call failed (see loza_ssa_last_error_string) */
  LOZA_SSA_ERR_SCRATCH_LIMIT = -9,  /* the call needs more than the built-in decode scratch holds */
};

/* Bits of the device status word (loza_ssa_get_last_device_status). */
enum {
  LOZA_SSA_DEV_WAIT_TIMEOUT = 1,    /* a pipeline wait gave up; that CTA skipped its work      */
  LOZA_SSA_DEV_BAD_PAGE = 2,        /* page_table entry outside [0, n_pages); split skipped    */
  LOZA_SSA_DEV_BAD_SEQLEN = 4,      /* decode seq_len < q_len (1) or > max_pages * page_size   */
  LOZA_SSA_DEV_BAD_CU_SEQLENS = 8,  /* cu_seqlens not starting at 0, decreasing, or != total   */
};

/*
 * Dense SSA prefill (causal self-attention of every token of every sequence).
 *   q, k : bf16 [B, H, L, d_qk]        v, o : bf16 [B, H, L, d_v]      lse : fp32 [B, H, L]
 *   (d_qk, d_v) in {(64,64), (128,128), (192,128)}; block must be 128;
 *   n_sink >= 0, n_local >= 1; scale finite (e.g. 1/sqrt(d_qk), the sqrt(d)
 *   of "LoZA：ZigZag稀疏注意力机制" §2.1).  L need not be a multiple of 128.
 * Returns LOZA_SSA_OK or a negative status; o and lse are written on success.
 */
int loza_ssa_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int L, int d_qk, int d_v, int block, int n_sink, int n_local,
                     float scale, loza_ssa_stream_t stream);

/*
 * Dense SSA prefill from HOST buffers: the same result as loza_ssa_prefill,
 * with the copies inside the call.  The B*H (batch, head) planes are cut into
 * n_chunks runs of whole planes; each run is uploaded on a copy stream of the
 * library's, computed on `stream` once it has landed, and downloaded on a
 * second copy stream, so uploads, kernels and downloads of different runs
 * overlap (the two copy directions run at once).
 *   q, k, v     : HOST bf16 [B, H, L, d] as loza_ssa_prefill; page-locked
 *                 (cudaHostAlloc / cudaHostRegister) for the copies to overlap.
 *   o, lse      : HOST outputs, page-locked likewise; complete once `stream`
 *                 reaches the end of the call (synchronise it before reading).
 *   n_chunks    : >= 1 (more than B*H acts as B*H); 8 suits large inputs.
 *   workspace   : DEVICE, 256-byte aligned, at least
 *                 loza_ssa_prefill_host_workspace_size(...) bytes: device
 *                 copies of q, k, v, o, lse, owned by the caller and reusable
 *                 once `stream` has passed the call.
 * Statuses as loza_ssa_prefill, plus LOZA_SSA_ERR_WORKSPACE.  Arguments are
 * checked before anything is enqueued; a CUDA error part-way (LOZA_SSA_ERR_CUDA)
 * can leave the earlier runs' copies and kernels enqueued.  The host buffers
 * must stay valid until `stream` has passed the call.
 */
int loza_ssa_prefill_host(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int L, int d_qk, int d_v, int block, int n_sink,
                          int n_local, float scale, int n_chunks, void* workspace,
                          size_t workspace_bytes, loza_ssa_stream_t stream);

/* Bytes of device workspace loza_ssa_prefill_host needs (0 on invalid sizes). */
size_t loza_ssa_prefill_host_workspace_size(int B, int H, int L, int d_qk, int d_v);

/*
 * Packed variable-length SSA prefill.  Sequence s occupies tokens
 * [cu_seqlens[s], cu_seqlens[s+1]) of the packed axis; block indices count from
 * each sequence's own first token, and no key crosses a sequence boundary.
 *   q, k : bf16 [H, total_tokens, d_qk]   v, o : bf16 [H, total_tokens, d_v]
 *   lse  : fp32 [H, total_tokens]         cu_seqlens : DEVICE int32 [n_seqs + 1]
 *   1 <= n_seqs <= 4000 (<= 3000 when d_qk = 192: the kernel keeps one prefix
 *   per sequence in shared memory).  max_seqlen is the caller's bound on any sequence
 *   length (used to size the launch; a longer sequence is still computed).
 * Other arguments as for loza_ssa_prefill.
 */
int loza_ssa_prefill_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens, int n_seqs, int total_tokens, int max_seqlen,
                            int H, int d_qk, int d_v, int block, int n_sink, int n_local,
                            float scale, loza_ssa_stream_t stream);

/*
 * Backward pass of the dense SSA prefill (loza_ssa_prefill's gradients):
 * given the upstream gradient dout = dL/dO, computes
 *   D_i = dO_i . O_i,  dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dO_i,
 * over the same SSA key sets J(i) as the forward pass, with
 * P_ij = exp(scale q_i.k_j - lse_i) -- the chain rule applied to the masked
 * softmax attention of "LoZA：ZigZag稀疏注意力机制" §2.1.
 *   q, k, dq, dk : bf16 [B, H, L, d_qk]  v, o, dout, dv : bf16 [B, H, L, d_v]
 *   lse          : fp32 [B, H, L] as written by loza_ssa_prefill
 *   (d_qk, d_v) in {(64,64), (128,128), (192,128)} (the last: the MLA head
 *   dims of the layers LoZA converts); block must be 128.
 *   workspace    : DEVICE scratch of at least
 *                  loza_ssa_prefill_bwd_workspace_size(...) bytes, 256-byte
 *                  aligned, owned by the caller, contents irrelevant on entry.
 * dq, dk, dv are overwritten (not accumulated into).  Statuses as for
 * loza_ssa_prefill; LOZA_SSA_ERR_HEAD_DIM for other head dims.
 */
int loza_ssa_prefill_bwd(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int H, int L, int d_qk, int d_v, int block, int n_sink, int n_local,
                         float scale, void* workspace, size_t workspace_bytes,
                         loza_ssa_stream_t stream);

/* Bytes of workspace loza_ssa_prefill_bwd needs (0 on invalid arguments):
 * fp32 D per row plus fp32 partial dK / dV of the sink blocks' chunks. */
size_t loza_ssa_prefill_bwd_workspace_size(int B, int H, int L, int d_qk, int d_v, int n_sink,
                                           int n_local);

/*
 * Backward of the packed varlen prefill (loza_ssa_prefill_varlen's
 * gradients).  Every sequence is its own attention problem: its gradients are
 * those of the dense backward over its slice, and no key of one sequence
 * reaches another's.
 *   q, k, dq, dk : bf16 [H, total_tokens, d_qk]  v, o, dout, dv : bf16 [H, total_tokens, d_v]
 *   lse          : fp32 [H, total_tokens]         cu_seqlens     : DEVICE int32 [n_seqs + 1]
 *   1 <= n_seqs <= 4000; (d_qk, d_v) as for loza_ssa_prefill_bwd; max_seqlen
 *   only has to be >= 1.
 *   workspace    : DEVICE scratch of at least
 *                  loza_ssa_prefill_varlen_bwd_workspace_size(...) bytes,
 *                  256-byte aligned, owned by the caller.
 * Invalid cu_seqlens (not 0 .. total_tokens, or decreasing) compute nothing
 * and set LOZA_SSA_DEV_BAD_CU_SEQLENS in the device status word.  Other
 * statuses as for loza_ssa_prefill_bwd.
 */
int loza_ssa_prefill_varlen_bwd(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                const int* cu_seqlens, int n_seqs, int total_tokens,
                                int max_seqlen, int H, int d_qk, int d_v, int block, int n_sink,
                                int n_local, float scale, void* workspace, size_t workspace_bytes,
                                loza_ssa_stream_t stream);

/* Bytes of workspace loza_ssa_prefill_varlen_bwd needs (0 on invalid
 * arguments): an upper bound that holds for any lengths summing to
 * total_tokens. */
size_t loza_ssa_prefill_varlen_bwd_workspace_size(int n_seqs, int total_tokens, int max_seqlen,
                                                  int H, int d_qk, int d_v, int n_sink,
                                                  int n_local);

/*
 * Paged SSA decode, absorbed-MLA layout: one new query token per sequence,
 * H_q query heads all attending one shared latent key/value row per token.
 *   q          : bf16 [B, H_q, d_qk]
 *   paged_kv   : bf16 [n_pages, page_size, d_qk]; the value of a token is the
 *                first d_v entries of its row
 *   page_table : DEVICE int32 [B, max_pages]; logical page p of sequence b is
 *                physical page page_table[b*max_pages + p]
 *   seq_lens   : DEVICE int32 [B]; the length INCLUDING the new token, whose
 *                position t = seq_len - 1 is the query position
 *   o          : bf16 [B, H_q, d_v]          lse : fp32 [B, H_q]
 *   (d_qk, d_v) must be (576, 512); page_size must be 128; the window reads
 *   logical pages {0..n_sink-1} and the n_local pages ending at t's page.
 *   workspace  : DEVICE scratch of at least
 *                loza_ssa_decode_workspace_size(B, H_q, d_v, n_sink, n_local)
 *                bytes, 256-byte aligned, owned by the caller, contents
 *                irrelevant on entry and overwritten.
 * Kernels: windows of up to 16 listed pages (the window's, plus any chosen
 * ones for loza_ssa_decode_selected) run as split CTAs of two pages each,
 * merged by LSE in the same launch (or a second one); wider windows (a
 * full-attention layer is the widest) run as three launches -- a one-CTA
 * plan of each sequence's pages, CTA pairs that stream an equal share of all
 * pages with an online softmax, and the LSE merge of their partials.  The
 * results agree with each other to rounding (same tolerance against the
 * float64 definition), not bit for bit.
 */
int loza_ssa_decode(const void* q, const void* paged_kv, const int* page_table,
                    const int* seq_lens, void* o, float* lse, int B, int H_q, int d_qk, int d_v,
                    int page_size, int max_pages, int n_pages, int n_sink, int n_local,
                    float scale, void* workspace, size_t workspace_bytes,
                    loza_ssa_stream_t stream);

/* Bytes of workspace loza_ssa_decode needs (0 on invalid arguments). */
size_t loza_ssa_decode_workspace_size(int B, int H_q, int d_v, int n_sink, int n_local);

/*
 * Paged decode over the SSA window plus pages chosen per sequence: the fixed
 * sink + sliding-window budget plus pages selected by a page-level indexer
 * (LongCat sparse-attention article, 机制 1 流感知索引 and 机制 3 分层索引, pages
 * of P = 128 tokens; the indexer itself is the caller's).
 *   extra_pages : DEVICE int32 [B, max_extra]; row b lists logical pages of
 *                 sequence b.  An entry that is negative, at or after the first
 *                 local page of the window, or below n_sink (i.e. not strictly
 *                 between the sink pages and the local run) adds nothing, and
 *                 a page listed twice counts once.  Every listed page lies
 *                 before the query's page, so all 128 of its keys are visible.
 *   max_extra   : >= 0; n_sink + n_local + max_extra <= 4096.
 * The keys of sequence b are { j <= t : page(j) in W(page(t)) or page(j) listed }.
 * workspace: at least loza_ssa_decode_selected_workspace_size(B, H_q, d_v,
 * n_sink, n_local, max_extra) bytes.  Other arguments, layouts, ownership and
 * statuses as for loza_ssa_decode (max_extra = 0 gives the same result).
 */
int loza_ssa_decode_selected(const void* q, const void* paged_kv, const int* page_table,
                             const int* seq_lens, const int* extra_pages, int max_extra, void* o,
                             float* lse, int B, int H_q, int d_qk, int d_v, int page_size,
                             int max_pages, int n_pages, int n_sink, int n_local, float scale,
                             void* workspace, size_t workspace_bytes,
                             loza_ssa_stream_t stream);

/* Bytes of workspace loza_ssa_decode_selected needs (0 on invalid arguments). */
size_t loza_ssa_decode_selected_workspace_size(int B, int H_q, int d_v, int n_sink, int n_local,
                                               int max_extra);

/*
 * Paged SSA decode over an FP8 latent cache.  Token j's cached row is 576
 * e4m3 codes k8_j (OCP FP8 E4M3: 1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, subnormals; 0x7f / 0xff are NaN and must not occur) and one
 * fp32 scale s_j, standing for K_j = s_j * k8_j (V_j = its first 512 entries).
 * The result is loza_ssa_decode's over those K_j: the SSA window of the QbitAI
 * LoZA article, softmax in fp32.  (An FP8 cache is one of the variants of the
 * decode workload; the pages' only FP8 remark -- the CSA/HCA tutorial's
 * section 5.1, item 3, on mixed-precision training -- is about compressed
 * matrices and fixes no cache format, so the per-token scale is this
 * library's choice: it keeps the scale out of the tensor-core products.)
 *   paged_kv_fp8 : DEVICE uint8 [n_pages, page_size, 576] e4m3 codes, 16-byte aligned.
 *   kv_scale     : DEVICE fp32 [n_pages, page_size], finite; 4-byte aligned.
 * workspace: at least loza_ssa_decode_workspace_size(B, H_q, d_v, n_sink,
 * n_local) bytes.  Other arguments, layouts, ownership and statuses as for
 * loza_ssa_decode; kv_scale == NULL is LOZA_SSA_ERR_NULL.
 */
int loza_ssa_decode_fp8(const void* q, const void* paged_kv_fp8, const float* kv_scale,
                        const int* page_table, const int* seq_lens, void* o, float* lse, int B,
                        int H_q, int d_qk, int d_v, int page_size, int max_pages, int n_pages,
                        int n_sink, int n_local, float scale, void* workspace,
                        size_t workspace_bytes, loza_ssa_stream_t stream);

/*
 * Paged SSA decode with q_len query tokens per sequence (speculative or
 * multi-token-prediction steps): the tokens of sequence b sit at positions
 * t = seq_len[b] - q_len .. seq_len[b] - 1, and token t attends the keys
 * J(t) = { j <= t : page(j) in W(page(t)) } -- the SSA mask of the QbitAI
 * LoZA article's 1024-token window paragraph (one global block plus seven
 * local blocks of 128 tokens) applied to each query position, so the tokens
 * see each other causally and each has its own window.
 *   q     : bf16 [B, q_len, H_q, d_qk]     o : bf16 [B, q_len, H_q, d_v]
 *   lse   : fp32 [B, q_len, H_q]
 *   q_len : >= 1, B * q_len <= 65535; every seq_len must be >= q_len (a
 *           shorter one sets LOZA_SSA_DEV_BAD_SEQLEN in the device status
 *           word and its rows come out as O = 0, LSE = -inf).
 * workspace: at least loza_ssa_decode_mtp_workspace_size(B, q_len, H_q, d_v,
 * n_sink, n_local) bytes.  Other arguments, layouts, ownership and statuses as
 * for loza_ssa_decode (q_len = 1 gives the same result).
 */
int loza_ssa_decode_mtp(const void* q, const void* paged_kv, const int* page_table,
                        const int* seq_lens, int q_len, void* o, float* lse, int B, int H_q,
                        int d_qk, int d_v, int page_size, int max_pages, int n_pages, int n_sink,
                        int n_local, float scale, void* workspace, size_t workspace_bytes,
                        loza_ssa_stream_t stream);

/* Bytes of workspace loza_ssa_decode_mtp needs (0 on invalid arguments). */
size_t loza_ssa_decode_mtp_workspace_size(int B, int q_len, int H_q, int d_v, int n_sink,
                                          int n_local);

/*
 * One attention layer of a LoZA decode step (the ZigZag layer stack of the
 * QbitAI LoZA article: half of LongCat-Flash's MLA layers keep full attention,
 * half become SSA).  All layers share one page table and one seq_lens array;
 * each has its own query, cache pool and outputs.
 */
typedef struct loza_ssa_decode_layer {
  const void* q;        /* bf16 [B, H_q, d_qk]                              */
  const void* paged_kv; /* bf16 [n_pages, page_size, d_qk]: this layer's pool */
  void* o;              /* bf16 [B, H_q, d_v]                               */
  float* lse;           /* fp32 [B, H_q]                                    */
  int full_attention;   /* nonzero: every key up to the query (an MLA layer);
                           0: the SSA window n_sink + n_local                */
} loza_ssa_decode_layer;

/*
 * Decode step over a stack of layers, in order, on one stream: each layer is
 * loza_ssa_decode with its own window -- {n_sink, n_local} for SSA layers,
 * all pages 0 .. page(t) for full-attention layers (computed as a window of
 * max_pages local pages, so max_pages <= 4096, i.e. contexts up to 512K
 * tokens, when any layer is full).
 *   layers   : HOST array of n_layers descriptors (read during the call only).
 *   workspace: at least loza_ssa_decode_layers_workspace_size(...) bytes; the
 *              layers run one after another and reuse it.
 * Other arguments as for loza_ssa_decode.  Returns the first failing layer's
 * status; the layers before it have been launched.
 */
int loza_ssa_decode_layers(const loza_ssa_decode_layer* layers, int n_layers,
                           const int* page_table, const int* seq_lens, int B, int H_q, int d_qk,
                           int d_v, int page_size, int max_pages, int n_pages, int n_sink,
                           int n_local, float scale, void* workspace, size_t workspace_bytes,
                           loza_ssa_stream_t stream);

/* Bytes of workspace loza_ssa_decode_layers needs for a stack that holds at
 * least one full-attention layer (any_full != 0) or only SSA layers. */
size_t loza_ssa_decode_layers_workspace_size(int B, int H_q, int d_v, int max_pages, int n_sink,
                                             int n_local, int any_full);

/* Static description of a status code (never NULL). */
const char* loza_ssa_status_string(int status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* loza_ssa_last_error_string(void);

/*
 * Waits for `stream`, then returns and clears the current device's status
 * word: 0 if no kernel reported a problem since the last read, else an OR of
 * LOZA_SSA_DEV_* bits.  Returns LOZA_SSA_ERR_CUDA if the wait or read failed.
 */
int loza_ssa_get_last_device_status(loza_ssa_stream_t stream);

/*
 * Debug: run the kernels' own tile scheduler on the device.  For every query
 * block qb in [0, n_qblocks) writes the key blocks it visits, ascending, to
 * tiles[qb*max_tiles ...] and their number to counts[qb] (DEVICE int32 buffers
 * of n_qblocks*max_tiles and n_qblocks entries).  A count above max_tiles is
 * reported but only max_tiles ids are written.
 */
int loza_ssa_debug_enumerate_tiles(int n_qblocks, int n_sink, int n_local, int* tiles,
                                   int* counts, int max_tiles, loza_ssa_stream_t stream);

/*
 * Debug: exercise the kernels' bounded pipeline wait.  One warp is launched;
 * thread 0 waits on an mbarrier that nothing ever arrives on, through the same
 * wait routine every pipeline of the library uses, but with a limit of
 * timeout_us microseconds (1 .. 100000) instead of the library's 2 s.  When
 * the limit passes it sets the CTA's abort flag and LOZA_SSA_DEV_WAIT_TIMEOUT
 * in the device status word and returns; the other 31 threads then wait on
 * the same barrier with ten times the limit and must give up on the abort
 * flag.  result (device int[2]): result[0] = 1 if thread 0's wait gave up,
 * result[1] = how many of the other threads' waits gave up (31 expected).
 * The limit is wall-clock time (the GPU's global timer), so time the GPU
 * spends on other contexts counts against it: under heavy time-slicing the
 * library's 2 s limit could in principle be reached by a wait that would
 * have completed, which is reported the same way.
 */
int loza_ssa_debug_wait_timeout(int timeout_us, int* result, loza_ssa_stream_t stream);

/*
 * Debug, HOST arithmetic only (no device work): how the long-window decode
 * shares the listed pages of n_units (row, head group) units over CTA pairs,
 * computed with the inline functions its kernels use.  unit_pages: HOST int32
 * [n_units], pages each unit lists (>= 0).  Outputs (HOST): pair_start int64
 * [pairs_launched + 1], the first page of pair k in the flattened list (pairs
 * past the ones used start at the total); slot_first / slot_count int32
 * [n_units], the unit's partial slots.  Returns LOZA_SSA_OK, or
 * LOZA_SSA_ERR_NULL / LOZA_SSA_ERR_SHAPE.
 */
int loza_ssa_debug_long_partition(const int* unit_pages, int n_units, int pairs_launched,
                                  long long* pair_start, int* slot_first, int* slot_count);

/*
 * Debug: run the decode kernel's page selection on the device.  For every
 * sequence b writes the PHYSICAL pages the decode window reads (logical order)
 * to pages[b*max_tiles ...] and their number to counts[b]; entries it would
 * reject are written as -1 and flagged in the device status word.
 */
int loza_ssa_debug_decode_pages(const int* page_table, const int* seq_lens, int B, int max_pages,
                                int n_pages, int page_size, int n_sink, int n_local, int* pages,
                                int* counts, int max_tiles, loza_ssa_stream_t stream);

/*
 * Paged SSA decode that allocates nothing and takes no workspace.
 *
 * The pages have no counterpart for this entry point; it exists for callers
 * that cannot hand the library device memory at the point of the call: a
 * plugin's enqueue step inside a framework that owns every allocation, or
 * latency-critical code that must not call cudaMalloc (which can synchronise
 * the device and take milliseconds) just to obtain scratch space.
 *
 * Arguments, layouts and results are those of loza_ssa_decode without the
 * workspace: the split partials live instead in one scratch array compiled
 * into the library, LOZA_SSA_STATIC_SCRATCH_BYTES long, which every GPU that
 * loads the library holds until the process exits.  It holds
 * LOZA_SSA_STATIC_SCRATCH_SLOTS split slots (one per split of the decode:
 * two window pages of one sequence and head group of up to 128 heads); a call
 * needs B * ceil(H_q/128) * ceil((n_sink + n_local)/2) of them (e.g. 32
 * sequences with the default 8-page window and up to 128 heads) and is rejected with
 * LOZA_SSA_ERR_SCRATCH_LIMIT, before anything is launched, if it needs more.
 *
 * The first call on a device looks up that device's address of the array
 * (with the device current); make that first call before any stream
 * capture on the device.  All calls on a device share the one array: calls
 * whose kernels overlap on the GPU (for example on two streams at once) race
 * and corrupt each other's results, so order them on one stream.  The array
 * keeps the last call's contents; nothing in it needs to start at zero,
 * because every slot a call reads is first written by the same call: a split
 * whose pipeline wait gave up writes NaN to its slot's LSE (and sets
 * LOZA_SSA_DEV_WAIT_TIMEOUT), so that the heads it covers come out NaN rather
 * than mixed with an earlier call's partials.
 * The array's device address is looked up once per device and kept for the
 * life of the process; it does not survive cudaDeviceReset() or a release and
 * re-creation of the device's primary context, after which this entry point
 * must not be called again in the same process.
 * Argument errors are reported as by loza_ssa_decode (the same codes, checked
 * first); LOZA_SSA_ERR_SCRATCH_LIMIT only for an otherwise valid call.
 * The library calls no allocation routine for this entry point.
 */
#define LOZA_SSA_STATIC_SCRATCH_SLOTS 128
#define LOZA_SSA_STATIC_SCRATCH_BYTES (LOZA_SSA_STATIC_SCRATCH_SLOTS * 128 * (512 * 2 + 4))
int loza_ssa_decode_static_scratch(const void* q, const void* paged_kv, const int* page_table,
                                   const int* seq_lens, void* o, float* lse, int B, int H_q,
                                   int d_qk, int d_v, int page_size, int max_pages, int n_pages,
                                   int n_sink, int n_local, float scale,
                                   loza_ssa_stream_t stream);

/* Library version, major*10000 + minor*100 + patch. */
int loza_ssa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOZA_SSA_H */
