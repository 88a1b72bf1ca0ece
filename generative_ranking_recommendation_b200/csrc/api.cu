// C ABI of libgenrank: host-side argument checks and dispatch to the kernels.
// Declarations and argument documentation live in include/genrank.h.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace gr;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int elem_size(int dtype) { return dtype == GENRANK_BF16 ? 2 : (dtype == GENRANK_F32 ? 4 : 0); }

bool fill_attn(AttnArgs& a, int B, int64_t T, const int32_t* off, const int32_t* hl,
               int max_seqlen, const void* q, const void* k, const void* v, int64_t tok_stride,
               int H, int dh, const int32_t* pos, const int64_t* ts, const float* sp,
               const float* st, float scale, int dtype, int64_t o_stride, int32_t* err) {
  memset(&a, 0, sizeof(a));
  a.B = B;
  a.T = T;
  a.off = off;
  a.hist_len = hl;
  a.max_seqlen = max_seqlen;
  a.q = q;
  a.k = k;
  a.v = v;
  a.tok_stride = tok_stride;
  a.H = H;
  a.dh = dh;
  a.pos = pos;
  a.ts = ts;
  for (int h = 0; h < H; ++h) {
    a.slope_pos[h] = sp[h];
    a.slope_time[h] = st[h];
  }
  a.scale = scale;
  a.dtype = dtype;
  a.o_stride = o_stride;
  a.err = err;
  return true;
}

int check_attn_common(int B, int64_t T, const int32_t* off, const int32_t* hl, int max_seqlen,
                      const void* q, const void* k, const void* v, int64_t tok_stride, int H,
                      int dh, const int32_t* pos, const int64_t* ts, const float* sp,
                      const float* st, float scale, int dtype, int64_t o_stride,
                      int32_t* err) {
  if (B < 1 || T < 0 || max_seqlen < 0 || H < 1 || dh < 1 || !off || !hl || !pos || !ts ||
      !sp || !st || !err || !(scale > 0.f) || !isfinite(scale))
    return GENRANK_ERR_INVALID_ARG;
  if (T > 0 && (!q || !k || !v)) return GENRANK_ERR_INVALID_ARG;
  if (H > kMaxHeads) return GENRANK_ERR_UNSUPPORTED;
  const int es = elem_size(dtype);
  if (!es) return GENRANK_ERR_INVALID_ARG;
  if (tok_stride < (int64_t)H * dh || o_stride < (int64_t)H * dh) return GENRANK_ERR_INVALID_ARG;
  if ((tok_stride * es) % 16 || (o_stride * es) % 16 || (dh * es) % 16)
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return GENRANK_ERR_INVALID_ARG;
  for (int h = 0; h < H; ++h)
    if (!isfinite(sp[h]) || !isfinite(st[h]) || sp[h] < 0.f || st[h] < 0.f)
      return GENRANK_ERR_INVALID_ARG;
  return GENRANK_OK;
}

bool use_tc(int dtype, int dh) { return dtype == GENRANK_BF16 && dh == 64; }

// genrank_attn_fwd with the linear or the bucketed time bias
int attn_fwd_impl(int time_bias, int B, int64_t T, const int32_t* seq_offsets,
                  const int32_t* hist_len, int max_seqlen, const void* q, const void* k,
                  const void* v, int64_t tok_stride, int H, int dh, const int32_t* pos,
                  const int64_t* ts, const float* slope_pos, const float* slope_time, float scale,
                  int dtype, void* o, int64_t o_stride, float* lse, void* ws, size_t ws_bytes,
                  int32_t* dev_err, genrank_stream_t stream) {
  int rc = check_attn_common(B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh,
                             pos, ts, slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  if (rc) return rc;
  if (T > 0 && (!o || !aligned16(o))) return GENRANK_ERR_INVALID_ARG;
  if (!use_tc(dtype, dh) && dh != 32 && dh != 64) return GENRANK_ERR_UNSUPPORTED;
  const size_t need = genrank_attn_workspace_size(B, T, H, dh, max_seqlen, 0);
  if (use_tc(dtype, dh) && (!ws || ws_bytes < need || !aligned16(ws))) return GENRANK_ERR_WORKSPACE;
  if (T == 0) return GENRANK_OK;
  AttnArgs a;
  fill_attn(a, B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts,
            slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  a.time_bias = time_bias;
  a.o = o;
  a.lse = lse;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return use_tc(dtype, dh) ? launch_attn_fwd_tc(a, s) : launch_attn_fwd_simt(a, s);
}

// genrank_attn_bwd with the linear or the bucketed time bias
int attn_bwd_impl(int time_bias, int B, int64_t T, const int32_t* seq_offsets,
                  const int32_t* hist_len, int max_seqlen, const void* q, const void* k,
                  const void* v, int64_t tok_stride, int H, int dh, const int32_t* pos,
                  const int64_t* ts, const float* slope_pos, const float* slope_time, float scale,
                  int dtype, const void* o, const void* dO, int64_t o_stride, const float* lse,
                  void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, int32_t* dev_err,
                  genrank_stream_t stream) {
  int rc = check_attn_common(B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh,
                             pos, ts, slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  if (rc) return rc;
  if (T > 0 && (!o || !dO || !lse || !dq || !dk || !dv)) return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(o) || !aligned16(dO))
    return GENRANK_ERR_INVALID_ARG;
  if (dh != 32 && dh != 64) return GENRANK_ERR_UNSUPPORTED;
  const size_t need = genrank_attn_workspace_size(B, T, H, dh, max_seqlen, 1);
  if (!ws || ws_bytes < need || !aligned16(ws)) return GENRANK_ERR_WORKSPACE;
  if (T == 0) return GENRANK_OK;
  AttnArgs a;
  fill_attn(a, B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts,
            slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  a.time_bias = time_bias;
  a.o = const_cast<void*>(o);
  a.dO = dO;
  a.lse_in = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return use_tc(dtype, dh) ? launch_attn_bwd_tc(a, s) : launch_attn_bwd_simt(a, s);
}

}  // namespace

extern "C" {

const char* genrank_status_string(int code) {
  switch (code) {
    case GENRANK_OK: return "ok";
    case GENRANK_ERR_INVALID_ARG: return "invalid argument";
    case GENRANK_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case GENRANK_ERR_WORKSPACE: return "workspace missing or too small";
    case GENRANK_ERR_LAUNCH: return "kernel launch failed";
    case GENRANK_ERR_CUDA: return "CUDA call failed";
    default: return "unknown status";
  }
}

const char* genrank_device_error_string(int bit) {
  switch (bit) {
    case 0: return "clean";
    case GENRANK_DERR_LAYOUT: return "device: bad seq_offsets/hist_len layout";
    case GENRANK_DERR_ITEM_ID: return "device: item id out of range";
    case GENRANK_DERR_ACTION_ID: return "device: action id out of range";
    case GENRANK_DERR_TS_ORDER: return "device: timestamps out of order";
    case GENRANK_DERR_POS_RANGE: return "device: position beyond the position table";
    case GENRANK_DERR_INDEX: return "device: metadata index out of range";
    case GENRANK_DERR_TIMEOUT: return "device: bounded wait timed out";
    default: return "several or unknown device error bits";
  }
}

int genrank_check_error(const int32_t* dev_err, genrank_stream_t stream) {
  if (!dev_err) return -GENRANK_ERR_INVALID_ARG;
  int32_t h = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, dev_err, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return -GENRANK_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return -GENRANK_ERR_CUDA;
  return h;
}

int genrank_alibi_slopes(int H, float* slope_pos, float* slope_time) {
  if (H < 1 || !slope_pos || !slope_time) return GENRANK_ERR_INVALID_ARG;
  for (int h = 0; h < H; ++h) {
    const double m = exp2(-8.0 * (h + 1) / (double)H);
    slope_pos[h] = (float)m;
    slope_time[h] = (float)(m / 3600.0);
  }
  return GENRANK_OK;
}

int genrank_embed_assemble(int B, int64_t T, const int32_t* seq_offsets, const int32_t* hist_len,
                           const int32_t* item_ids, const int32_t* action_ids, const int64_t* ts,
                           const void* item_tab, int64_t n_item, const void* action_tab,
                           int n_action, const void* pos_tab, int n_pos, const void* ri_tab,
                           int n_ri, const void* rt_tab, int n_rt, int d, int dtype, void* E,
                           int32_t* pos, int32_t* req_idx, int32_t* rt_bucket, int32_t* dev_err,
                           genrank_stream_t stream) {
  const int es = elem_size(dtype);
  if (B < 1 || T < 0 || !seq_offsets || !hist_len || !dev_err || !es || d < 1)
    return GENRANK_ERR_INVALID_ARG;
  if (n_item < 1 || n_action < 1 || n_pos < 2 || n_ri < 2 || n_rt < 2)
    return GENRANK_ERR_INVALID_ARG;
  if (n_rt > 65) return GENRANK_ERR_UNSUPPORTED;
  if (((int64_t)d * es) % 16) return GENRANK_ERR_INVALID_ARG;
  if (T > 0 && (!item_ids || !action_ids || !ts || !item_tab || !action_tab || !pos_tab ||
                !ri_tab || !rt_tab || !E || !pos || !req_idx || !rt_bucket))
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(item_tab) || !aligned16(action_tab) || !aligned16(pos_tab) ||
      !aligned16(ri_tab) || !aligned16(rt_tab) || !aligned16(E))
    return GENRANK_ERR_INVALID_ARG;
  EmbedFwdArgs a{B, T, seq_offsets, hist_len, item_ids, action_ids, ts, item_tab, n_item,
                 action_tab, n_action, pos_tab, n_pos, ri_tab, n_ri, rt_tab, n_rt, d, dtype,
                 E, pos, req_idx, rt_bucket, dev_err};
  return launch_embed_fwd(a, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_embed_assemble_rmsnorm(int B, int64_t T, const int32_t* seq_offsets,
                                   const int32_t* hist_len, const int32_t* item_ids,
                                   const int32_t* action_ids, const int64_t* ts,
                                   const void* item_tab, int64_t n_item, const void* action_tab,
                                   int n_action, const void* pos_tab, int n_pos,
                                   const void* ri_tab, int n_ri, const void* rt_tab, int n_rt,
                                   int d, float* x_out, void* a_out, float eps, int32_t* pos,
                                   int32_t* req_idx, int32_t* rt_bucket, int32_t* dev_err,
                                   genrank_stream_t stream) {
  if (B < 1 || T < 0 || !seq_offsets || !hist_len || !dev_err || d < 1 || !(eps >= 0.f))
    return GENRANK_ERR_INVALID_ARG;
  if (n_item < 1 || n_action < 1 || n_pos < 2 || n_ri < 2 || n_rt < 2)
    return GENRANK_ERR_INVALID_ARG;
  if (n_rt > 65 || d != 512) return GENRANK_ERR_UNSUPPORTED;
  if (T > 0 && (!item_ids || !action_ids || !ts || !item_tab || !action_tab || !pos_tab ||
                !ri_tab || !rt_tab || !x_out || !a_out || !pos || !req_idx || !rt_bucket))
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(item_tab) || !aligned16(action_tab) || !aligned16(pos_tab) ||
      !aligned16(ri_tab) || !aligned16(rt_tab) || !aligned16(x_out) || !aligned16(a_out))
    return GENRANK_ERR_INVALID_ARG;
  EmbedFwdArgs a{B, T, seq_offsets, hist_len, item_ids, action_ids, ts, item_tab, n_item,
                 action_tab, n_action, pos_tab, n_pos, ri_tab, n_ri, rt_tab, n_rt, d, GENRANK_BF16,
                 nullptr, pos, req_idx, rt_bucket, dev_err, x_out, a_out, eps};
  return launch_embed_fwd(a, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_embed_assemble_bwd(int B, int64_t T, const int32_t* seq_offsets,
                               const int32_t* hist_len, const int32_t* item_ids,
                               const int32_t* action_ids, const int32_t* pos,
                               const int32_t* req_idx, const int32_t* rt_bucket, const void* dE,
                               int d, int dtype, float* d_item, int64_t n_item, float* d_action,
                               int n_action, float* d_pos, int n_pos, float* d_ri, int n_ri,
                               float* d_rt, int n_rt, int32_t* dev_err, genrank_stream_t stream) {
  const int es = elem_size(dtype);
  if (B < 1 || T < 0 || !seq_offsets || !hist_len || !dev_err || !es || d < 2 || (d & 1))
    return GENRANK_ERR_INVALID_ARG;
  if (n_item < 1 || n_action < 1 || n_pos < 1 || n_ri < 1 || n_rt < 1)
    return GENRANK_ERR_INVALID_ARG;
  if (T > 0 && (!item_ids || !action_ids || !pos || !req_idx || !rt_bucket || !dE || !d_item ||
                !d_action || !d_pos || !d_ri || !d_rt))
    return GENRANK_ERR_INVALID_ARG;
  EmbedBwdArgs a{B, T, seq_offsets, hist_len, item_ids, action_ids, pos, req_idx, rt_bucket, dE,
                 d, dtype, d_item, n_item, d_action, n_action, d_pos, n_pos, d_ri, n_ri, d_rt,
                 n_rt, dev_err};
  return launch_embed_bwd(a, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_candidate_logits(int M, const int64_t* rows, int64_t T, int d, const void* x,
                             int64_t x_stride, const void* o, int64_t o_stride, int dtype,
                             const float* w, const float* u, float* z, int32_t* dev_err,
                             genrank_stream_t stream) {
  const int es = elem_size(dtype);
  if (M < 0 || T < 0 || d < 1 || !es || !dev_err) return GENRANK_ERR_INVALID_ARG;
  if (M == 0) return GENRANK_OK;
  if (!rows || !x || !o || !w || !u || !z) return GENRANK_ERR_INVALID_ARG;
  if (x_stride < d || o_stride < d || (d * es) % 16 || (x_stride * es) % 16 ||
      (o_stride * es) % 16)
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(o) || !aligned16(w) || !aligned16(u))
    return GENRANK_ERR_INVALID_ARG;
  CandLogitsArgs a;
  a.M = M;
  a.rows = rows;
  a.T = T;
  a.d = d;
  a.x = x;
  a.x_stride = x_stride;
  a.o = o;
  a.o_stride = o_stride;
  a.dtype = dtype;
  a.w = w;
  a.u = u;
  a.z = z;
  a.err = dev_err;
  return launch_cand_logits(a, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_gather_rows(int64_t M, const int64_t* rows, int64_t T, int64_t row_bytes,
                        const void* src, int64_t src_stride, void* dst, int64_t dst_stride,
                        int32_t* dev_err, genrank_stream_t stream) {
  if (M < 0 || T < 0 || row_bytes <= 0 || row_bytes % 16 || !dev_err)
    return GENRANK_ERR_INVALID_ARG;
  if (M == 0) return GENRANK_OK;
  if (!rows || !src || !dst || src_stride < row_bytes || dst_stride < row_bytes ||
      src_stride % 16 || dst_stride % 16 || !aligned16(src) || !aligned16(dst))
    return GENRANK_ERR_INVALID_ARG;
  GatherRowsArgs a;
  a.M = M;
  a.rows = rows;
  a.T = T;
  a.row_bytes = row_bytes;
  a.src = src;
  a.src_stride = src_stride;
  a.dst = dst;
  a.dst_stride = dst_stride;
  a.err = dev_err;
  return launch_gather_rows(a, reinterpret_cast<cudaStream_t>(stream));
}

size_t genrank_attn_workspace_size(int B, int64_t T, int H, int dh, int max_seqlen, int is_bwd) {
  if (B < 1 || T < 0 || H < 1 || dh < 1 || max_seqlen < 0) return 0;
  if (is_bwd) {
    const size_t simt = attn_bwd_simt_workspace(B, T, H, dh, max_seqlen);
    if (dh != 64) return simt;
    const size_t tc = attn_bwd_tc_workspace(B, T, H, max_seqlen);
    return tc > simt ? tc : simt;
  }
  return attn_fwd_tc_workspace(B, T, H, max_seqlen);
}

int genrank_attn_fwd(int B, int64_t T, const int32_t* seq_offsets, const int32_t* hist_len,
                     int max_seqlen, const void* q, const void* k, const void* v,
                     int64_t tok_stride, int H, int dh, const int32_t* pos, const int64_t* ts,
                     const float* slope_pos, const float* slope_time, float scale, int dtype,
                     void* o, int64_t o_stride, float* lse, void* ws, size_t ws_bytes,
                     int32_t* dev_err, genrank_stream_t stream) {
  return attn_fwd_impl(kTimeBiasLinear, B, T, seq_offsets, hist_len, max_seqlen, q, k, v,
                       tok_stride, H, dh, pos, ts, slope_pos, slope_time, scale, dtype, o,
                       o_stride, lse, ws, ws_bytes, dev_err, stream);
}

int genrank_attn_fwd_bucketed(int B, int64_t T, const int32_t* seq_offsets,
                              const int32_t* hist_len, int max_seqlen, const void* q,
                              const void* k, const void* v, int64_t tok_stride, int H, int dh,
                              const int32_t* pos, const int64_t* ts, const float* slope_pos,
                              const float* slope_tb, float scale, int dtype, void* o,
                              int64_t o_stride, float* lse, void* ws, size_t ws_bytes,
                              int32_t* dev_err, genrank_stream_t stream) {
  if (!use_tc(dtype, dh)) return GENRANK_ERR_UNSUPPORTED;
  return attn_fwd_impl(kTimeBiasBucketed, B, T, seq_offsets, hist_len, max_seqlen, q, k, v,
                       tok_stride, H, dh, pos, ts, slope_pos, slope_tb, scale, dtype, o,
                       o_stride, lse, ws, ws_bytes, dev_err, stream);
}

int genrank_attn_fwd_dense_bias(int B, int64_t T, const int32_t* seq_offsets,
                                const int32_t* hist_len, int max_seqlen, const void* q,
                                const void* k, const void* v, int64_t tok_stride, int H, int dh,
                                const void* bias, int64_t Lpad, float scale, int dtype, void* o,
                                int64_t o_stride, float* lse, void* ws, size_t ws_bytes,
                                int32_t* dev_err, genrank_stream_t stream) {
  if (B < 1 || T < 0 || max_seqlen < 0 || H < 1 || dh < 1 || !seq_offsets || !hist_len ||
      !dev_err || !(scale > 0.f) || !isfinite(scale))
    return GENRANK_ERR_INVALID_ARG;
  if (H > kMaxHeads) return GENRANK_ERR_UNSUPPORTED;
  if (!use_tc(dtype, dh)) return GENRANK_ERR_UNSUPPORTED;
  if (T > 0 && (!q || !k || !v || !o || !bias)) return GENRANK_ERR_INVALID_ARG;
  if (tok_stride < (int64_t)H * dh || o_stride < (int64_t)H * dh || (tok_stride * 2) % 16 ||
      (o_stride * 2) % 16)
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(bias))
    return GENRANK_ERR_INVALID_ARG;
  // every tile a work item reads lies in the user's Lpad x Lpad block
  if (Lpad < 128 || Lpad % 128 || Lpad < max_seqlen) return GENRANK_ERR_INVALID_ARG;
  const size_t need = genrank_attn_workspace_size(B, T, H, dh, max_seqlen, 0);
  if (!ws || ws_bytes < need || !aligned16(ws)) return GENRANK_ERR_WORKSPACE;
  if (T == 0) return GENRANK_OK;
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B;
  a.T = T;
  a.off = seq_offsets;
  a.hist_len = hist_len;
  a.max_seqlen = max_seqlen;
  a.q = q;
  a.k = k;
  a.v = v;
  a.tok_stride = tok_stride;
  a.H = H;
  a.dh = dh;
  a.scale = scale;
  a.dtype = dtype;
  a.o = o;
  a.o_stride = o_stride;
  a.lse = lse;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.err = dev_err;
  return launch_attn_fwd_dense(a, bias, Lpad, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_linear(int M, int N, int K, const void* A, int64_t lda, const void* Wt, int64_t ldw,
                   int epilogue, void* C, int64_t ldc, int32_t* dev_err,
                   genrank_stream_t stream) {
  if (M < 0 || N < 1 || K < 1 || !dev_err) return GENRANK_ERR_INVALID_ARG;
  if (epilogue != GENRANK_EPI_STORE && epilogue != GENRANK_EPI_SILU) return GENRANK_ERR_INVALID_ARG;
  if (N % 256 || K % 64) return GENRANK_ERR_UNSUPPORTED;
  if (M == 0) return GENRANK_OK;
  if (!A || !Wt || !C || !aligned16(A) || !aligned16(Wt) || !aligned16(C))
    return GENRANK_ERR_INVALID_ARG;
  if (lda < K || ldw < K || ldc < N || (lda * 2) % 16 || (ldw * 2) % 16 || (ldc * 2) % 16)
    return GENRANK_ERR_INVALID_ARG;
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.M = M;
  g.N = N;
  g.K = K;
  g.a = A;
  g.lda = lda;
  g.w = Wt;
  g.ldw = ldw;
  g.epilogue = epilogue == GENRANK_EPI_SILU ? kEpiSilu : kEpiStore;
  g.c = C;
  g.ldc = ldc;
  g.err = dev_err;
  return launch_gemm_tc(g, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_linear_residual_rmsnorm(int M, int d, int K, const void* A, int64_t lda,
                                    const void* Wt, int64_t ldw, const float* x_in,
                                    float* x_out, int64_t ldx, void* a_out, int64_t lda_out,
                                    const float* w_head, float* z, float eps, int32_t* dev_err,
                                    genrank_stream_t stream) {
  if (M < 0 || d < 1 || K < 1 || !dev_err || !(eps >= 0.f)) return GENRANK_ERR_INVALID_ARG;
  if (d != 512 || K % 64) return GENRANK_ERR_UNSUPPORTED;
  if (M == 0) return GENRANK_OK;
  if (!A || !Wt || !x_in || !x_out || (!a_out && !w_head) || (w_head && !z))
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(Wt) || !aligned16(x_in) || !aligned16(x_out) ||
      (a_out && !aligned16(a_out)) || (w_head && !aligned16(w_head)))
    return GENRANK_ERR_INVALID_ARG;
  if (lda < K || ldw < K || ldx < d || (a_out && lda_out < d) || (lda * 2) % 16 ||
      (ldw * 2) % 16 || (ldx * 4) % 16 || (a_out && (lda_out * 2) % 16))
    return GENRANK_ERR_INVALID_ARG;
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.M = M;
  g.N = d;
  g.K = K;
  g.a = A;
  g.lda = lda;
  g.w = Wt;
  g.ldw = ldw;
  g.epilogue = kEpiResRms;
  g.x_in = x_in;
  g.x_out = x_out;
  g.ldx = ldx;
  g.a_out = a_out;
  g.lda_out = lda_out;
  g.w_head = w_head;
  g.z = z;
  g.eps = eps;
  g.err = dev_err;
  return launch_gemm_tc(g, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_rmsnorm(int64_t M, int d, const void* x, int64_t ldx, int dtype, float* x_out,
                    int64_t ldxo, void* a_out, int64_t lda_out, float eps, int32_t* dev_err,
                    genrank_stream_t stream) {
  const int es = elem_size(dtype);
  if (M < 0 || d < 1 || !es || !dev_err || !(eps >= 0.f)) return GENRANK_ERR_INVALID_ARG;
  if ((d * es) % 16 || d % 8) return GENRANK_ERR_UNSUPPORTED;
  if (M == 0) return GENRANK_OK;
  if (!x || !a_out || !aligned16(x) || !aligned16(a_out) || (x_out && !aligned16(x_out)))
    return GENRANK_ERR_INVALID_ARG;
  if (ldx < d || lda_out < d || (x_out && ldxo < d) || (ldx * es) % 16 || (lda_out * 2) % 16 ||
      (x_out && (ldxo * 4) % 16))
    return GENRANK_ERR_INVALID_ARG;
  return launch_rmsnorm(M, d, x, ldx, dtype, x_out, ldxo, a_out, lda_out, eps,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t genrank_attn_cached_workspace_size(int B, int64_t C, int64_t Th, int H, int dh,
                                          int max_cand) {
  if (B < 1 || C < 0 || Th < 0 || H < 1 || dh < 1 || max_cand < 0) return 0;
  return attn_fwd_cached_workspace(B, C, Th, H, max_cand);
}

int genrank_attn_fwd_cached(int B, int64_t C, const int32_t* cand_offsets, int max_cand,
                            const void* q_c, const void* k_c, const void* v_c,
                            int64_t cand_stride, int64_t Th, const int32_t* hist_offsets,
                            const void* k_hist, const void* v_hist, int64_t hist_stride,
                            const int32_t* pos_hist, const int64_t* ts_hist,
                            const int64_t* ts_cand, int H, int dh, const float* slope_pos,
                            const float* slope_time, float scale, int dtype, void* o,
                            int64_t o_stride, float* lse, void* ws, size_t ws_bytes,
                            int32_t* dev_err, genrank_stream_t stream) {
  if (B < 1 || C < 0 || Th < 0 || max_cand < 0 || H < 1 || dh < 1 || !cand_offsets ||
      !hist_offsets || !ts_cand || !slope_pos || !slope_time || !dev_err || !(scale > 0.f) ||
      !isfinite(scale))
    return GENRANK_ERR_INVALID_ARG;
  if (H > kMaxHeads) return GENRANK_ERR_UNSUPPORTED;
  const int es = elem_size(dtype);
  if (!es) return GENRANK_ERR_INVALID_ARG;
  if (C > 0 && (!q_c || !k_c || !v_c)) return GENRANK_ERR_INVALID_ARG;
  if (cand_stride < (int64_t)H * dh || o_stride < (int64_t)H * dh ||
      (cand_stride * es) % 16 || (o_stride * es) % 16 || (dh * es) % 16)
    return GENRANK_ERR_INVALID_ARG;
  if (!aligned16(q_c) || !aligned16(k_c) || !aligned16(v_c)) return GENRANK_ERR_INVALID_ARG;
  for (int h = 0; h < H; ++h)
    if (!isfinite(slope_pos[h]) || !isfinite(slope_time[h]) || slope_pos[h] < 0.f ||
        slope_time[h] < 0.f)
      return GENRANK_ERR_INVALID_ARG;
  if (Th > 0 && (!k_hist || !v_hist || !pos_hist || !ts_hist)) return GENRANK_ERR_INVALID_ARG;
  if (Th > 0 && (hist_stride < (int64_t)H * dh || !aligned16(k_hist) || !aligned16(v_hist) ||
                 (hist_stride * es) % 16))
    return GENRANK_ERR_INVALID_ARG;
  if (C > 0 && (!o || !aligned16(o))) return GENRANK_ERR_INVALID_ARG;
  if (!use_tc(dtype, dh)) return GENRANK_ERR_UNSUPPORTED;
  const size_t need = genrank_attn_cached_workspace_size(B, C, Th, H, dh, max_cand);
  if (!ws || ws_bytes < need || !aligned16(ws)) return GENRANK_ERR_WORKSPACE;
  if (C == 0) return GENRANK_OK;
  CachedAttnArgs c;
  memset(&c, 0, sizeof(c));
  fill_attn(c.a, B, C, cand_offsets, nullptr, max_cand, q_c, k_c, v_c, cand_stride, H, dh,
            nullptr, ts_cand, slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  c.a.o = o;
  c.a.lse = lse;
  c.a.ws = ws;
  c.a.ws_bytes = ws_bytes;
  c.hist_off = hist_offsets;
  c.k_hist = k_hist;
  c.v_hist = v_hist;
  c.hist_stride = hist_stride;
  c.Th = Th;
  c.pos_hist = pos_hist;
  c.ts_hist = ts_hist;
  c.max_cand = max_cand;
  return launch_attn_fwd_cached(c, reinterpret_cast<cudaStream_t>(stream));
}

size_t genrank_attn_candidates_workspace_size(int B, int64_t T, int H, int dh, int max_seqlen) {
  if (B < 1 || T < 0 || H < 1 || dh < 1 || max_seqlen < 0) return 0;
  return attn_fwd_cached_workspace(B, T, T, H, max_seqlen);
}

int genrank_attn_fwd_candidates(int B, int64_t T, const int32_t* seq_offsets,
                                const int32_t* hist_len, int max_seqlen, const void* q,
                                const void* k, const void* v, int64_t tok_stride, int H, int dh,
                                const int32_t* pos, const int64_t* ts, const float* slope_pos,
                                const float* slope_time, float scale, int dtype, void* o,
                                int64_t o_stride, float* lse, void* ws, size_t ws_bytes,
                                int32_t* dev_err, genrank_stream_t stream) {
  int rc = check_attn_common(B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh,
                             pos, ts, slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  if (rc) return rc;
  if (T > 0 && (!o || !aligned16(o))) return GENRANK_ERR_INVALID_ARG;
  if (!use_tc(dtype, dh)) return GENRANK_ERR_UNSUPPORTED;
  const size_t need = genrank_attn_candidates_workspace_size(B, T, H, dh, max_seqlen);
  if (!ws || ws_bytes < need || !aligned16(ws)) return GENRANK_ERR_WORKSPACE;
  if (T == 0) return GENRANK_OK;
  CachedAttnArgs c;
  memset(&c, 0, sizeof(c));
  fill_attn(c.a, B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh, pos, ts,
            slope_pos, slope_time, scale, dtype, o_stride, dev_err);
  c.a.o = o;
  c.a.lse = lse;
  c.a.ws = ws;
  c.a.ws_bytes = ws_bytes;
  c.hist_off = nullptr;  // the jagged array: history keys are the users' own history rows
  c.k_hist = k;
  c.v_hist = v;
  c.hist_stride = tok_stride;
  c.Th = T;
  c.pos_hist = pos;
  c.ts_hist = ts;
  c.max_cand = max_seqlen;
  return launch_attn_fwd_cached(c, reinterpret_cast<cudaStream_t>(stream));
}

int genrank_attn_bwd(int B, int64_t T, const int32_t* seq_offsets, const int32_t* hist_len,
                     int max_seqlen, const void* q, const void* k, const void* v,
                     int64_t tok_stride, int H, int dh, const int32_t* pos, const int64_t* ts,
                     const float* slope_pos, const float* slope_time, float scale, int dtype,
                     const void* o, const void* dO, int64_t o_stride, const float* lse, void* dq,
                     void* dk, void* dv, void* ws, size_t ws_bytes, int32_t* dev_err,
                     genrank_stream_t stream) {
  return attn_bwd_impl(kTimeBiasLinear, B, T, seq_offsets, hist_len, max_seqlen, q, k, v,
                       tok_stride, H, dh, pos, ts, slope_pos, slope_time, scale, dtype, o, dO,
                       o_stride, lse, dq, dk, dv, ws, ws_bytes, dev_err, stream);
}

int genrank_attn_bwd_bucketed(int B, int64_t T, const int32_t* seq_offsets,
                              const int32_t* hist_len, int max_seqlen, const void* q,
                              const void* k, const void* v, int64_t tok_stride, int H, int dh,
                              const int32_t* pos, const int64_t* ts, const float* slope_pos,
                              const float* slope_tb, float scale, int dtype, const void* o,
                              const void* dO, int64_t o_stride, const float* lse, void* dq,
                              void* dk, void* dv, void* ws, size_t ws_bytes, int32_t* dev_err,
                              genrank_stream_t stream) {
  if (!use_tc(dtype, dh)) return GENRANK_ERR_UNSUPPORTED;
  return attn_bwd_impl(kTimeBiasBucketed, B, T, seq_offsets, hist_len, max_seqlen, q, k, v,
                       tok_stride, H, dh, pos, ts, slope_pos, slope_tb, scale, dtype, o, dO,
                       o_stride, lse, dq, dk, dv, ws, ws_bytes, dev_err, stream);
}

}  // extern "C"
