// Internal launch interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gr {

struct EmbedFwdArgs {
  int B;
  long long T;
  const int32_t* off;
  const int32_t* hist_len;
  const int32_t* item_ids;
  const int32_t* action_ids;
  const int64_t* ts;
  const void* item_tab;
  long long n_item;
  const void* action_tab;
  int n_action;
  const void* pos_tab;
  int n_pos;
  const void* ri_tab;
  int n_ri;
  const void* rt_tab;
  int n_rt;
  int d;
  int dtype;
  void* E;
  int32_t* pos;
  int32_t* req_idx;
  int32_t* rt_bucket;
  int32_t* err;
  // with x_out: instead of E, the fp32 copy of E's rows (x_out) and their RMSNorm in
  // bf16 (a_out), the first block's input (bf16 tables, d = 512)
  float* x_out = nullptr;
  void* a_out = nullptr;
  float eps = 0.f;
};

struct EmbedBwdArgs {
  int B;
  long long T;
  const int32_t* off;
  const int32_t* hist_len;
  const int32_t* item_ids;
  const int32_t* action_ids;
  const int32_t* pos;
  const int32_t* req_idx;
  const int32_t* rt_bucket;
  const void* dE;
  int d;
  int dtype;
  float* g_item;
  long long n_item;
  float* g_action;
  int n_action;
  float* g_pos;
  int n_pos;
  float* g_ri;
  int n_ri;
  float* g_rt;
  int n_rt;
  int32_t* err;
};

constexpr int kMaxHeads = 64;

// time term of the ALiBi bias: linear in seconds, slope_time[h] per second, or bucketed,
// slope_time[h] per bucket of min(62, floor(4 log2(|t_i - t_j| + 1)))
constexpr int kTimeBiasLinear = 0;
constexpr int kTimeBiasBucketed = 1;

// Everything an attention launch needs; slopes are copied by value.
struct AttnArgs {
  int B;
  long long T;
  const int32_t* off;
  const int32_t* hist_len;
  int max_seqlen;
  const void* q;
  const void* k;
  const void* v;
  long long tok_stride;  // elements
  int H;
  int dh;
  const int32_t* pos;
  const int64_t* ts;
  float slope_pos[kMaxHeads];
  float slope_time[kMaxHeads];
  float scale;
  int dtype;
  int time_bias;  // kTimeBiasLinear or kTimeBiasBucketed
  void* o;
  long long o_stride;  // elements
  float* lse;          // [H, T] or null
  // backward only
  const void* dO;
  void* dq;
  void* dk;
  void* dv;
  const float* lse_in;
  void* ws;
  size_t ws_bytes;
  int32_t* err;
};

// Candidates scored against a cache of their users' history keys and values: `a`
// describes the candidate rows (a.off = candidate offsets [B+1], a.q/k/v = candidate
// projections with a.tok_stride, a.T = C candidate rows, a.ts = the candidates' request
// times [C], a.o / a.lse = outputs [C, H*dh] / [H, C]); the cache has Th rows.
struct CachedAttnArgs {
  AttnArgs a;
  // [B+1] rows of user u's history in the cache; null for one jagged token array (the
  // full attention's layout): user u's history rows [off[u], off[u] + hist_len[u]) of
  // the keys and values, its candidates the rest of [off[u], off[u+1])
  const int32_t* hist_off;
  const void* k_hist;
  const void* v_hist;
  long long hist_stride;  // elements
  long long Th;
  const int32_t* pos_hist;  // [Th]
  const int64_t* ts_hist;   // [Th]
  int max_cand;             // bound of the candidates per user
};

// C = A Wt^T on tensor cores with a fused epilogue (bf16 A [M][K], Wt [N][K], K-major)
constexpr int kEpiStore = 0;   // C = bf16(A W)
constexpr int kEpiSilu = 1;    // C = bf16(SiLU(A W))
constexpr int kEpiResRms = 2;  // x_out = x_in + A W; a_out = bf16(rms(x_out)); z = rms . w
struct GemmArgs {
  int M, N, K;
  const void* a;
  long long lda;
  const void* w;  // Wt [N][K]
  long long ldw;
  int epilogue;
  void* c;  // store / silu: [M][N] bf16
  long long ldc;
  const float* x_in;  // res+rms: [M][N] fp32 residual stream in and out (may alias)
  float* x_out;
  long long ldx;
  void* a_out;  // res+rms: [M][N] bf16 normalised rows, or null
  long long lda_out;
  const float* w_head;  // res+rms: [N] fp32 head vector, or null
  float* z;             // res+rms: [M] fp32 head output
  float eps;
  int32_t* err;
};
int launch_gemm_tc(const GemmArgs& g, cudaStream_t st);
int launch_rmsnorm(long long M, int d, const void* x, long long ldx, int x_dtype, float* x_out,
                   long long ldxo, void* a_out, long long lda, float eps, cudaStream_t st);

struct CandLogitsArgs {
  long long M;
  const int64_t* rows;
  long long T;
  int d;
  const void* x;
  long long x_stride;  // elements
  const void* o;
  long long o_stride;  // elements
  int dtype;
  const float* w;
  const float* u;
  float* z;
  int32_t* err;
};

int launch_cand_logits(const CandLogitsArgs& a, cudaStream_t st);

struct GatherRowsArgs {
  long long M;
  const int64_t* rows;
  long long T;
  long long row_bytes;   // a multiple of 16
  const void* src;
  long long src_stride;  // bytes
  void* dst;
  long long dst_stride;  // bytes
  int32_t* err;
};
int launch_gather_rows(const GatherRowsArgs& a, cudaStream_t st);

int launch_embed_fwd(const EmbedFwdArgs& a, cudaStream_t st);
int launch_embed_bwd(const EmbedBwdArgs& a, cudaStream_t st);

// CUDA-core attention (fp32 storage, or bf16 with dh != 64)
int launch_attn_fwd_simt(const AttnArgs& a, cudaStream_t st);
int launch_attn_bwd_simt(const AttnArgs& a, cudaStream_t st);
size_t attn_bwd_simt_workspace(int B, long long T, int H, int dh, int max_seqlen);

// tcgen05 / TMEM / TMA attention forward and backward (bf16, dh = 64)
int launch_attn_fwd_tc(const AttnArgs& a, cudaStream_t st);
size_t attn_fwd_tc_workspace(int B, long long T, int H, int max_seqlen);
int launch_attn_fwd_cached(const CachedAttnArgs& c, cudaStream_t st);
// forward with a dense per-user bias [B][Lpad][Lpad] (bf16) in place of the ALiBi terms
int launch_attn_fwd_dense(const AttnArgs& a, const void* bias, long long Lpad, cudaStream_t st);
size_t attn_fwd_cached_workspace(int B, long long C, long long Th, int H, int max_cand);
int launch_attn_bwd_tc(const AttnArgs& a, cudaStream_t st);
size_t attn_bwd_tc_workspace(int B, long long T, int H, int max_seqlen);

}  // namespace gr
