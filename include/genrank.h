/*
 * genrank.h — C ABI of the GenRank hot-path library (libgenrank.so, sm_100a).
 *
 * The operations follow the GenRank pages ("Towards Large-scale Generative
 * Ranking"):
 *   - huaxiaozhuan.com chapter notes "GenRank [2025]", §1.4.1 Item-Action
 *     Organization (token = item embedding + action embedding, candidates carry
 *     the mask action, candidate mask) and §1.4.2 Position & Time Biases (the
 *     position, request-index and pre-request time embeddings, the five-way
 *     input sum, ALiBi fused into the attention score, slopes 2^(-8(h+1)/H));
 *   - wln20.github.io "生成式排序 —— 小红书 GenRank 精读笔记" (the candidate mask
 *     makes batched scoring equal to appending each candidate alone);
 *   - fun-rec mdbook "The Overall Generative Ranking Paradigm", §7.2.1 and
 *     §7.2.2 (history causal, candidates see all history and not each other;
 *     ALiBi over position and time).
 *
 * Conventions shared by every entry point:
 *   - Every array argument is a DEVICE pointer owned by the caller, unless it is
 *     documented as a host pointer.  The library allocates no memory and keeps
 *     no state between calls; scratch space is the caller's workspace.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  Nothing inside synchronises except genrank_check_error.
 *   - The return value is GENRANK_OK or a host-detected GENRANK_ERR_* code; on
 *     such an error nothing was launched.  Errors found in the data on the device
 *     (ids out of range, unsorted timestamps, ...) are OR-ed as GENRANK_DERR_*
 *     bits into *dev_err (one caller-zeroed device int32); the kernels clamp the
 *     offending index and keep going, so no call traps or hangs the GPU.  Every
 *     wait inside a kernel is bounded and reports GENRANK_DERR_TIMEOUT.
 *   - Token layout ("jagged"): users are contiguous; user u owns tokens
 *     [seq_offsets[u], seq_offsets[u+1]), history first (hist_len[u] tokens,
 *     oldest first), then its candidates.  Every call also takes T, a HOST
 *     value: the row count of every per-token array (normally seq_offsets[B]).
 *     Kernels never touch rows at or beyond T; offsets that point past it raise
 *     GENRANK_DERR_LAYOUT.
 *   - dtype is GENRANK_F32 or GENRANK_BF16 and applies to every floating-point
 *     tensor of the call unless stated otherwise; accumulation is fp32.
 */
#ifndef GENRANK_H_
#define GENRANK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *genrank_stream_t; /* the same handle as cudaStream_t */

enum { GENRANK_F32 = 0, GENRANK_BF16 = 1 };

/* host-detected status codes (return values) */
enum {
  GENRANK_OK = 0,
  GENRANK_ERR_INVALID_ARG = 1,  /* null pointer, bad size or stride */
  GENRANK_ERR_UNSUPPORTED = 2,  /* a valid but unsupported shape or dtype */
  GENRANK_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
  GENRANK_ERR_LAUNCH = 4,       /* a kernel launch failed (cudaGetLastError) */
  GENRANK_ERR_CUDA = 5          /* another CUDA runtime/driver call failed */
};

/* device-detected data errors (bits of *dev_err) */
enum {
  GENRANK_DERR_LAYOUT = 1 << 0,     /* bad seq_offsets / hist_len, or offsets beyond T */
  GENRANK_DERR_ITEM_ID = 1 << 1,    /* item id outside [0, n_item) (clamped) */
  GENRANK_DERR_ACTION_ID = 1 << 2,  /* history action id outside [0, n_action) (clamped) */
  GENRANK_DERR_TS_ORDER = 1 << 3,   /* history timestamps decrease, candidate times differ,
                                       or the request time precedes the last history time */
  GENRANK_DERR_POS_RANGE = 1 << 4,  /* position >= n_pos (clamped) */
  GENRANK_DERR_INDEX = 1 << 5,      /* a metadata index outside its table (backward) */
  GENRANK_DERR_TIMEOUT = 1 << 6     /* a bounded in-kernel wait gave up */
};

/* Human-readable name of a GENRANK_OK / GENRANK_ERR_* return code. */
const char *genrank_status_string(int code);

/* Human-readable name of one GENRANK_DERR_* bit (or "clean" for 0). */
const char *genrank_device_error_string(int bit);

/* Synchronises `stream`, reads *dev_err and returns it (0 when clean); returns
 * -GENRANK_ERR_CUDA if the copy or the synchronisation failed. */
int genrank_check_error(const int32_t *dev_err, genrank_stream_t stream);

/* ALiBi slopes, written to HOST arrays of H floats:
 *   slope_pos[h]  = 2^(-8(h+1)/H)                (per unit of position)
 *   slope_time[h] = slope_pos[h] / 3600          (per second of |t_i - t_j|)
 * huaxiaozhuan "GenRank [2025]" §1.4.2 gives the slope formula and the H = 8
 * example (1/2 ... 1/256); the per-second time slope is the linear time bias of
 * the workloads this library serves.  Returns GENRANK_ERR_INVALID_ARG for H < 1. */
int genrank_alibi_slopes(int H, float *slope_pos, float *slope_time);

/* ---------------------------------------------------------------------------
 * Step a1 + a2: per-token metadata and the five-way embedding sum.
 *   E_i = item[x_i] + action[a_i, or M for candidates] + pos_tab[pos_i]
 *         + ri_tab[req_idx_i] + rt_tab[rt_bucket_i]
 * (huaxiaozhuan "GenRank [2025]" §1.4.1 token sum, §1.4.2 input
 * representation), summed in fp32 and rounded once to dtype.
 *   pos_i       = 1-based index for history tokens; n_u + 1 for every candidate
 *                 (§1.4.2 Position Embeddings: candidates of one request share it)
 *   req_idx_i   = |{t_1..t_i}|, distinct timestamps so far, clamped to n_ri - 1
 *                 (§1.4.2 Request Index Embeddings)
 *   rt_bucket_i = 0 if no earlier request, else 1 + min(n_rt - 2,
 *                 floor(4 log2(gap + 1))), gap = t_i - max{t_j : t_j < t_i}
 *                 (§1.4.2 Pre-Request Time Embeddings; the bucket form is this
 *                 library's reading); a candidate's values are those of the
 *                 token made by appending it alone at time t_req.
 * Arguments:
 *   B            number of users (>= 1); seq_offsets [B+1] int32, hist_len [B] int32
 *   item_ids     [T] int32, rows of item_tab
 *   action_ids   [T] int32 in [0, n_action); ignored at candidate slots
 *   ts           [T] int64 seconds; history non-decreasing; every candidate slot
 *                holds the request time t_req >= the last history time
 *   item_tab     [n_item, d]; action_tab [n_action + 1, d] whose LAST row is the
 *                mask action M; pos_tab [n_pos, d] (row 0 unused); ri_tab [n_ri, d];
 *                rt_tab [n_rt, d] with 2 <= n_rt <= 65.  Row-major, dtype, 16-byte
 *                aligned rows (d * sizeof(dtype) a multiple of 16).
 *   E            [T, d] output (dtype); pos, req_idx, rt_bucket: [T] int32 outputs
 * Two kernels on `stream`: the per-user metadata scan, then the row gather-sum. */
int genrank_embed_assemble(int B, int64_t T, const int32_t *seq_offsets, const int32_t *hist_len,
                           const int32_t *item_ids, const int32_t *action_ids, const int64_t *ts,
                           const void *item_tab, int64_t n_item, const void *action_tab,
                           int n_action, const void *pos_tab, int n_pos, const void *ri_tab,
                           int n_ri, const void *rt_tab, int n_rt, int d, int dtype,
                           void *E, int32_t *pos, int32_t *req_idx, int32_t *rt_bucket,
                           int32_t *dev_err, genrank_stream_t stream);

/* Step a2 with the first block's pre-norm fused in: the same metadata and gather-sum
 * as genrank_embed_assemble, but instead of E each token's row is written as
 *   x_out [T, d] fp32  = E_i as genrank_embed_assemble rounds it (bf16), upcast
 *   a_out [T, d] bf16  = bf16(x_out_i / sqrt(mean_j x_out_ij^2 + eps))
 * which is bit for bit what genrank_rmsnorm(E, ..., x_out) gives after
 * genrank_embed_assemble (the same lanes, summation order and rounding): the fp32
 * residual stream and the normalised input of a pre-RMSNorm block, without E's
 * round trip through memory.  bf16 tables and d = 512 only (GENRANK_ERR_UNSUPPORTED
 * otherwise); x_out and a_out 16-byte aligned with row stride d; eps >= 0.  Other
 * arguments and errors as genrank_embed_assemble. */
int genrank_embed_assemble_rmsnorm(int B, int64_t T, const int32_t *seq_offsets,
                                   const int32_t *hist_len, const int32_t *item_ids,
                                   const int32_t *action_ids, const int64_t *ts,
                                   const void *item_tab, int64_t n_item, const void *action_tab,
                                   int n_action, const void *pos_tab, int n_pos,
                                   const void *ri_tab, int n_ri, const void *rt_tab, int n_rt,
                                   int d, float *x_out, void *a_out, float eps, int32_t *pos,
                                   int32_t *req_idx, int32_t *rt_bucket, int32_t *dev_err,
                                   genrank_stream_t stream);

/* Step a5: table gradients of the embedding sum (training).  Each token's dE_i
 * is added to the five rows it read: d_item[x_i], d_action[a_i or M],
 * d_pos[pos_i], d_ri[req_idx_i], d_rt[rt_bucket_i].  pos/req_idx/rt_bucket are
 * the metadata written by genrank_embed_assemble.  dE is [T, d] in dtype; the
 * five gradient tables are fp32, caller-zeroed (the call accumulates into them),
 * with the row counts of the forward tables (d_action has n_action + 1 rows).
 * Float atomics make the summation order, and so the last bits, vary from run
 * to run. */
int genrank_embed_assemble_bwd(int B, int64_t T, const int32_t *seq_offsets, const int32_t *hist_len,
                               const int32_t *item_ids, const int32_t *action_ids,
                               const int32_t *pos, const int32_t *req_idx,
                               const int32_t *rt_bucket, const void *dE, int d, int dtype,
                               float *d_item, int64_t n_item, float *d_action, int n_action,
                               float *d_pos, int n_pos, float *d_ri, int n_ri, float *d_rt,
                               int n_rt, int32_t *dev_err, genrank_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step a3: masked multi-head attention with on-the-fly ALiBi position and time
 * biases (huaxiaozhuan "GenRank [2025]" §1.4.2 score formula; §1.4.1 candidate
 * mask; fun-rec §7.2.2 bias over position and time).  For user u, head h, local
 * rows i and keys j:
 *   s_ij = scale * q_i.k_j - slope_pos[h] |p_i - p_j| - slope_time[h] |t_i - t_j|
 *   visible(i, j) = j <= i                 for history rows (i < n_u)
 *                 = j < n_u  or  j == i    for candidate rows
 *   O_i = sum_j softmax_j(s_ij) v_j over visible j;  LSE_i = log sum_j exp(s_ij)
 * p = pos from genrank_embed_assemble, t = ts.  No N x N bias is ever stored.
 * Arguments:
 *   max_seqlen   an upper bound of seq_offsets[u+1] - seq_offsets[u] (host value)
 *   q, k, v      [T] rows of H * dh values; head h of token t starts at
 *                ptr + t * tok_stride + h * dh (elements).  A fused [T, 3, H, dh]
 *                projection output passes q = base, k = base + H*dh, v = base + 2*H*dh,
 *                tok_stride = 3*H*dh.  tok_stride * sizeof(dtype) % 16 == 0 and
 *                16-byte aligned bases are required.
 *   pos [T] int32, ts [T] int64 (device); slope_pos, slope_time: HOST arrays [H]
 *   scale        > 0, normally 1/sqrt(dh)
 *   o            [T, H * dh] output, row stride o_stride elements (dtype)
 *   lse          [H, T] fp32 natural-log LSE output, or NULL to skip
 *   ws, ws_bytes caller scratch of at least genrank_attn_workspace_size(..., 0) bytes;
 *                its contents on entry do not matter (nothing needs zeroing)
 * Supported: bf16 with dh = 64 runs the tcgen05/TMEM/TMA kernel; fp32 (any
 * dtype) with dh in {32, 64, 128} runs the CUDA-core kernel.  H <= 64. */
int genrank_attn_fwd(int B, int64_t T, const int32_t *seq_offsets, const int32_t *hist_len, int max_seqlen,
                     const void *q, const void *k, const void *v, int64_t tok_stride, int H,
                     int dh, const int32_t *pos, const int64_t *ts, const float *slope_pos,
                     const float *slope_time, float scale, int dtype, void *o, int64_t o_stride,
                     float *lse, void *ws, size_t ws_bytes, int32_t *dev_err,
                     genrank_stream_t stream);

/* Step a4: gradients of step a3 (training).  Given dO [T, H*dh] (row stride
 * o_stride, like o), the forward's o and lse, writes dq, dk, dv with the layout
 * of q, k, v (tok_stride).  The biases have no parameters, so there is no bias
 * gradient.  With P = softmax(S): dV = P^T dO, dP = dO V^T,
 * dS = P * (dP - rowsum(dO * O)), dQ = scale dS K, dK = scale dS^T Q.
 * Every token row of dq/dk/dv is written (no accumulation into them).
 * bf16 with dh = 64 runs on tcgen05 tensor cores (fp32 dQ accumulated in the
 * workspace); fp32, or dh = 32, runs the CUDA-core kernels.  The workspace
 * (genrank_attn_workspace_size(..., 1) bytes) needs no initialisation: the call
 * zeroes what it accumulates into. */
int genrank_attn_bwd(int B, int64_t T, const int32_t *seq_offsets, const int32_t *hist_len, int max_seqlen,
                     const void *q, const void *k, const void *v, int64_t tok_stride, int H,
                     int dh, const int32_t *pos, const int64_t *ts, const float *slope_pos,
                     const float *slope_time, float scale, int dtype, const void *o,
                     const void *dO, int64_t o_stride, const float *lse, void *dq, void *dk,
                     void *dv, void *ws, size_t ws_bytes, int32_t *dev_err,
                     genrank_stream_t stream);

/* ---------------------------------------------------------------------------
 * Bucketed time bias.  fun-rec "The Overall Generative Ranking Paradigm" §7.2.2 (and
 * its zh twin) writes the ALiBi bias as
 *   -m_p (p_i - p_j) - m_t bucket(t_i - t_j)
 * without defining bucket().  This library's reading: the quarter-octave grid of the
 * pre-request time embedding, bucket(D) = min(62, floor(4 log2(D + 1))) for a gap of D
 * seconds (two items of one request share bucket 0; gaps from about 12.9 h on share
 * bucket 62).  Same arguments, layouts, workspace sizes and error behaviour as
 * genrank_attn_fwd / genrank_attn_bwd, except that slope_tb[h] is the slope per
 * bucket (the plainest reading takes slope_tb = slope_pos).  Unlike the linear time
 * bias this term does not split into a row part and a column part, so the kernels
 * evaluate the bucket for every visible pair (exactly, in fp32: the binary exponent
 * of (D + 1)^4 for D + 1 <= 46341).  Per-user time spans are clamped to 2^29 s.
 * bf16 with dh = 64 only; anything else returns GENRANK_ERR_UNSUPPORTED. */
int genrank_attn_fwd_bucketed(int B, int64_t T, const int32_t *seq_offsets,
                              const int32_t *hist_len, int max_seqlen, const void *q,
                              const void *k, const void *v, int64_t tok_stride, int H, int dh,
                              const int32_t *pos, const int64_t *ts, const float *slope_pos,
                              const float *slope_tb, float scale, int dtype, void *o,
                              int64_t o_stride, float *lse, void *ws, size_t ws_bytes,
                              int32_t *dev_err, genrank_stream_t stream);

/* Gradients of genrank_attn_fwd_bucketed (the bucketed bias has no parameters either):
 * dV = P^T dO, dS = P * (dP - rowsum(dO * O)), dQ = scale dS K, dK = scale dS^T Q. */
int genrank_attn_bwd_bucketed(int B, int64_t T, const int32_t *seq_offsets,
                              const int32_t *hist_len, int max_seqlen, const void *q,
                              const void *k, const void *v, int64_t tok_stride, int H, int dh,
                              const int32_t *pos, const int64_t *ts, const float *slope_pos,
                              const float *slope_tb, float scale, int dtype, const void *o,
                              const void *dO, int64_t o_stride, const float *lse, void *dq,
                              void *dk, void *dv, void *ws, size_t ws_bytes, int32_t *dev_err,
                              genrank_stream_t stream);

/* ---------------------------------------------------------------------------
 * Comparison path: attention with a dense per-user N x N bias read from memory, the
 * relative attention bias of the interleaved organisation that GenRank replaces
 * (fun-rec "The Overall Generative Ranking Paradigm" §7.2.2: score_ij = q_i.k_j/sqrt(d)
 * + rab(i, j), an N x N matrix whose I/O grows with the square of the length; §7.2.0:
 * the interleaved sequence spends two tokens per interaction, 2 n_c + m in all;
 * huaxiaozhuan "GenRank [2025]" §1.4.2).  It runs the forward kernel with the ALiBi
 * terms replaced by one bf16 bias value per visible pair:
 *   s_ij = scale q_i.k_j + bias[u][i][j]      (i, j local to user u)
 * with the mask of genrank_attn_fwd (history causal; a candidate sees the history and
 * itself), so the two layouts and the two biases can be timed on the same kernels.
 * Arguments as genrank_attn_fwd (same workspace size), minus pos/ts/slopes, plus:
 *   bias   [B][Lpad][Lpad] bf16, shared by the heads, row-major, 16-byte aligned
 *   Lpad   a multiple of 128 and >= max_seqlen (every tile read stays in the block)
 * bf16 with dh = 64 only; anything else returns GENRANK_ERR_UNSUPPORTED.  The row
 * offset starts at 0 (no sign bound holds for a learned bias); a tile whose row sum
 * leaves [2^-100, 2^100] is redone with its exact maximum. */
int genrank_attn_fwd_dense_bias(int B, int64_t T, const int32_t *seq_offsets,
                                const int32_t *hist_len, int max_seqlen, const void *q,
                                const void *k, const void *v, int64_t tok_stride, int H, int dh,
                                const void *bias, int64_t Lpad, float scale, int dtype, void *o,
                                int64_t o_stride, float *lse, void *ws, size_t ws_bytes,
                                int32_t *dev_err, genrank_stream_t stream);

/* ---------------------------------------------------------------------------
 * Candidate scoring from cached history keys and values (KV-cached serving).
 * huaxiaozhuan "GenRank [2025]" §1.3.2 (feature-engineering paragraph) credits the
 * KV cache with keeping generative ranking efficient as the candidate set grows,
 * and fun-rec "The Overall Generative Ranking Paradigm" §7.2.1 counts the halved KV
 * cache among the action-oriented layout's gains.  A user's history keys and values
 * do not depend on the candidates (history rows are causal, §1.3.1), so a server
 * keeps them and scores each request's candidates against them.  For user u with
 * n_u = hist_offsets[u+1] - hist_offsets[u] cached rows and candidate rows
 * [cand_offsets[u], cand_offsets[u+1]), every candidate c (position n_u + 1, time
 * ts_cand[c]) sees the whole history and itself (§1.4.1):
 *   s_cj = scale q_c.k_j - slope_pos[h] |p_c - p_j| - slope_time[h] |t_c - t_j|
 *   s_cc = scale q_c.k_c
 *   O_c = sum softmax(s) v over {history of u} + {c};  LSE_c = log sum exp(s)
 * which equals the candidate rows of genrank_attn_fwd over history + candidates.
 * Arguments:
 *   B, cand_offsets [B+1]   users and their candidate rows (C = cand_offsets[B] rows)
 *   max_cand                an upper bound of cand_offsets[u+1] - cand_offsets[u]
 *   q_c, k_c, v_c           candidate projections, [C] rows of H * dh with row
 *                           stride cand_stride (as genrank_attn_fwd's q, k, v)
 *   Th, hist_offsets [B+1]  the cache: user u owns rows [hist_offsets[u],
 *                           hist_offsets[u+1]) of k_hist, v_hist ([Th] rows of H*dh,
 *                           stride hist_stride), pos_hist [Th] int32 (the 1-based
 *                           positions, <= n_u + 1) and ts_hist [Th] int64 seconds,
 *                           non-decreasing per user
 *   ts_cand [C] int64       each candidate's request time, >= its user's last history time
 *   o [C, H*dh] (o_stride), lse [H, C] fp32 (or NULL): outputs for the candidate rows
 *   ws, ws_bytes            at least genrank_attn_cached_workspace_size(...) bytes;
 *                           contents on entry do not matter
 * bf16 with dh = 64 only (tcgen05/TMEM/TMA kernel); anything else returns
 * GENRANK_ERR_UNSUPPORTED.  Device-detected: GENRANK_DERR_LAYOUT (offsets beyond C
 * or Th, more than max_cand candidates), GENRANK_DERR_TS_ORDER, GENRANK_DERR_POS_RANGE. */
int genrank_attn_fwd_cached(int B, int64_t C, const int32_t *cand_offsets, int max_cand,
                            const void *q_c, const void *k_c, const void *v_c,
                            int64_t cand_stride, int64_t Th, const int32_t *hist_offsets,
                            const void *k_hist, const void *v_hist, int64_t hist_stride,
                            const int32_t *pos_hist, const int64_t *ts_hist,
                            const int64_t *ts_cand, int H, int dh, const float *slope_pos,
                            const float *slope_time, float scale, int dtype, void *o,
                            int64_t o_stride, float *lse, void *ws, size_t ws_bytes,
                            int32_t *dev_err, genrank_stream_t stream);

/* Bytes of workspace genrank_attn_fwd_cached needs for these sizes (0 if invalid). */
size_t genrank_attn_cached_workspace_size(int B, int64_t C, int64_t Th, int H, int dh,
                                          int max_cand);

/* The candidate rows of genrank_attn_fwd only, on its own jagged layout: for every user
 * u the rows [seq_offsets[u] + hist_len[u], seq_offsets[u+1]) of o (and those columns
 * of lse) are written exactly as genrank_attn_fwd defines them; history rows of o and
 * lse are left untouched.  This is candidate scoring with the history keys and values
 * read in place from k and v (the cached kernel in the layout the full attention
 * uses): a model whose next step reads only candidate rows (the last block before the
 * head: only candidates reach the logits, huaxiaozhuan "GenRank [2025]" §1.3.1) skips
 * the history rows' attention.  Arguments, layouts and errors as genrank_attn_fwd;
 * bf16 with dh = 64 only (GENRANK_ERR_UNSUPPORTED otherwise); ws of at least
 * genrank_attn_candidates_workspace_size(...) bytes, contents on entry do not matter. */
int genrank_attn_fwd_candidates(int B, int64_t T, const int32_t *seq_offsets,
                                const int32_t *hist_len, int max_seqlen, const void *q,
                                const void *k, const void *v, int64_t tok_stride, int H, int dh,
                                const int32_t *pos, const int64_t *ts, const float *slope_pos,
                                const float *slope_time, float scale, int dtype, void *o,
                                int64_t o_stride, float *lse, void *ws, size_t ws_bytes,
                                int32_t *dev_err, genrank_stream_t stream);

/* Bytes of workspace genrank_attn_fwd_candidates needs (0 if invalid). */
size_t genrank_attn_candidates_workspace_size(int B, int64_t T, int H, int dh, int max_seqlen);

/* genrank_attn_fwd for callers that cannot allocate device memory.
 * The paper has no counterpart of this call; it exists for deployment.  Some
 * callers cannot call cudaMalloc (or any allocator, torch's included) where they
 * run attention: serving loops that forbid device allocations after start-up,
 * or hosts that own all device memory and hand out no scratch.  This call takes
 * the same arguments as genrank_attn_fwd minus the workspace: its scratch is a
 * 16 MiB array compiled into the library, which every GPU that loads the library
 * holds until the process exits.  Inputs and outputs are still the caller's.
 *   - Only the tensor-core kernel (bf16, dh = 64) uses the array.  For it, sizes
 *     whose workspace (genrank_attn_workspace_size(..., 0)) exceeds 16 MiB are
 *     rejected with GENRANK_ERR_WORKSPACE before any launch; the CUDA-core kernel
 *     (fp32, or dh = 32) needs no scratch and takes any size.
 *   - The first call on each device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; nothing in it needs to start at zero.  Calls that overlap on the
 *     GPU (other streams, other host threads) race on it: serialise them.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
int genrank_attn_fwd_static(int B, int64_t T, const int32_t *seq_offsets, const int32_t *hist_len,
                            int max_seqlen, const void *q, const void *k, const void *v,
                            int64_t tok_stride, int H, int dh, const int32_t *pos,
                            const int64_t *ts, const float *slope_pos, const float *slope_time,
                            float scale, int dtype, void *o, int64_t o_stride, float *lse,
                            int32_t *dev_err, genrank_stream_t stream);

/* Candidate logits of a one-block scorer without FFN: the score is read at
 * candidate positions only (huaxiaozhuan "GenRank [2025]" §1.3.1: the loss and
 * the ranking output live at candidate positions), and for
 *   h = x + attn W_o,   z = h . w_head
 * the logit is z = x . w_head + attn . u with u = W_o w_head (a d-vector the
 * caller forms once per weights), so the candidate rows are read once and no
 * [m, d] intermediate is formed:
 *   z[c] = sum_j x[rows[c], j] w[j] + sum_j o[rows[c], j] u[j]   (fp32 accumulation)
 * Arguments:
 *   M            number of candidates (>= 0); rows [M] int64 token rows in [0, T)
 *   x, o         [T, d] row-major in dtype with row strides x_stride, o_stride
 *                (elements); 16-byte aligned rows (d, strides: multiples of 16 bytes)
 *   w, u         [d] fp32, 16-byte aligned; z [M] fp32 output
 * A row outside [0, T) sets GENRANK_DERR_INDEX and gives z[c] = 0. */
int genrank_candidate_logits(int M, const int64_t *rows, int64_t T, int d, const void *x,
                             int64_t x_stride, const void *o, int64_t o_stride, int dtype,
                             const float *w, const float *u, float *z, int32_t *dev_err,
                             genrank_stream_t stream);

/* The candidate rows of a token matrix, gathered into a dense one: only candidate rows
 * reach the ranking output (huaxiaozhuan "GenRank [2025]" §1.3.1), so the last block's
 * output projection, residual and FFN run on them alone.
 *   dst [M] rows: dst row k = src row rows[k], row_bytes bytes each (a byte copy, so
 *   any element type), src rows src_stride bytes apart, dst rows dst_stride apart.
 * Arguments: M >= 0; rows [M] int64 in [0, T) (device); row_bytes > 0 and the strides
 * multiples of 16, strides >= row_bytes; src, dst 16-byte aligned device pointers that
 * do not overlap.  The caller owns every buffer.  A row outside [0, T) sets
 * GENRANK_DERR_INDEX and zeroes its destination row.  Returns GENRANK_ERR_INVALID_ARG
 * for invalid sizes or alignment, before any launch. */
int genrank_gather_rows(int64_t M, const int64_t *rows, int64_t T, int64_t row_bytes,
                        const void *src, int64_t src_stride, void *dst, int64_t dst_stride,
                        int32_t *dev_err, genrank_stream_t stream);

/* ---------------------------------------------------------------------------
 * The blocks around the attention, on tensor cores with fused epilogues.
 * huaxiaozhuan "GenRank [2025]" §1.4.1 and fun-rec §7.2.1: the action-oriented layout
 * halves the tokens and so the linear-projection cost; the four-layer workloads'
 * block is pre-RMSNorm (unit gain) attention and a 4d SiLU FFN, each added to an fp32
 * residual stream, with a final RMSNorm and the candidate head.  Matrices are
 * row-major; A and the weights are bf16, and a weight W [K][N] is passed TRANSPOSED,
 * Wt [N][K] (each output column's weights contiguous), so both tensor-core operands
 * are K-major.  Accumulation is fp32 in tensor memory.  Pointers 16-byte aligned,
 * row strides (elements) multiples of 16 bytes. */
enum { GENRANK_EPI_STORE = 0, GENRANK_EPI_SILU = 1 };

/* C [M][N] = bf16(A W) (GENRANK_EPI_STORE) or bf16(SiLU(A W)) (GENRANK_EPI_SILU),
 * A [M][K], Wt [N][K].  N a multiple of 256, K a multiple of 64, else
 * GENRANK_ERR_UNSUPPORTED. */
int genrank_linear(int M, int N, int K, const void *A, int64_t lda, const void *Wt, int64_t ldw,
                   int epilogue, void *C, int64_t ldc, int32_t *dev_err,
                   genrank_stream_t stream);

/* The residual update and the next RMSNorm in one pass over each row:
 *   x_out = x_in + A W                      (fp32 [M][d]; x_out may equal x_in)
 *   a_out = bf16(x_out / sqrt(mean_j x_out_j^2 + eps))     (or NULL)
 *   z     = (x_out / sqrt(mean_j x_out_j^2 + eps)) . w_head (when w_head != NULL; z [M])
 * A [M][K] bf16, Wt [d][K] bf16.  d must be 512 (one 128 x 512 fp32 tile fills tensor
 * memory), K a multiple of 64; else GENRANK_ERR_UNSUPPORTED.  At least one of a_out
 * and w_head must be given. */
int genrank_linear_residual_rmsnorm(int M, int d, int K, const void *A, int64_t lda,
                                    const void *Wt, int64_t ldw, const float *x_in,
                                    float *x_out, int64_t ldx, void *a_out, int64_t lda_out,
                                    const float *w_head, float *z, float eps, int32_t *dev_err,
                                    genrank_stream_t stream);

/* a_out [M][d] = bf16(x / sqrt(mean_j x_j^2 + eps)) for x [M][d] in dtype, and x_out =
 * fp32 copy of x when x_out != NULL (the residual stream of the first block).  d a
 * multiple of 8 with d * sizeof(dtype) a multiple of 16. */
int genrank_rmsnorm(int64_t M, int d, const void *x, int64_t ldx, int dtype, float *x_out,
                    int64_t ldxo, void *a_out, int64_t lda_out, float eps, int32_t *dev_err,
                    genrank_stream_t stream);

/* Bytes of workspace genrank_attn_fwd (is_bwd = 0) or genrank_attn_bwd
 * (is_bwd = 1) need for these sizes.  Returns 0 for invalid sizes. */
size_t genrank_attn_workspace_size(int B, int64_t T, int H, int dh, int max_seqlen, int is_bwd);

#ifdef __cplusplus
}
#endif

#endif /* GENRANK_H_ */
