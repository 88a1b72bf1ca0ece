// Action-oriented input assembly: per-token metadata and the five-way embedding
// gather-sum (forward), and its scatter-add backward.
//
// "GenRank [2025]" chapter notes (huaxiaozhuan.com), §1.4.1 and §1.4.2: a token
// is psi(x_i) + phi(a_i) (candidates: psi(x_j) + m, the mask action), plus the
// position embedding (candidates of one request share position n + 1), the
// request-index embedding |{t_1..t_i}| and the pre-request time embedding
// bucket(t_i - max_{t_j < t_i} t_j).
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {

// ------------------------------------------------------------------------------------------
// block scans (inclusive) over blockDim.x <= 1024 threads
// ------------------------------------------------------------------------------------------
template <bool kMax>
__device__ int block_scan(int v, int* sh /* >= 32 ints */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int x = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = kMax ? max(v, x) : v + x;
  }
  if (lane == 31) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? sh[lane] : (kMax ? -2147483647 : 0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int x = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w = kMax ? max(w, x) : w + x;
    }
    sh[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v = kMax ? max(v, sh[warp - 1]) : v + sh[warp - 1];
  __syncthreads();
  return v;
}

// One block per user.  History tokens are scanned in chunks of blockDim.x with
// the request count and the current group start carried across chunks.
__global__ void __launch_bounds__(256) k_token_meta(
    int B, long long T, const int32_t* __restrict__ off, const int32_t* __restrict__ hist_len,
    const int64_t* __restrict__ ts, int n_pos, int n_ri, int n_rt, int32_t* __restrict__ pos,
    int32_t* __restrict__ req_idx, int32_t* __restrict__ rt_bucket, int32_t* err) {
  __shared__ int sh[32];
  __shared__ int carry_cnt, carry_gs;
  const int u = blockIdx.x;
  long long s = off[u], e = off[u + 1];
  int n = hist_len[u];
  if (s < 0 || e < s || e > T) {
    if (threadIdx.x == 0) flag(err, GENRANK_DERR_LAYOUT);
    return;
  }
  const int L = (int)(e - s);
  if (n < 0 || n > L) {
    if (threadIdx.x == 0) flag(err, GENRANK_DERR_LAYOUT);
    n = max(0, min(n, L));
  }
  if (threadIdx.x == 0) {
    carry_cnt = 0;
    carry_gs = 0;
  }
  __syncthreads();
  for (int c0 = 0; c0 < n; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const bool valid = i < n;
    long long t = valid ? ts[s + i] : 0;
    long long tp = (valid && i > 0) ? ts[s + i - 1] : t;
    int is_new = valid && (i == 0 || t != tp);
    if (valid && i > 0 && t < tp) flag(err, GENRANK_DERR_TS_ORDER);
    const int cc = carry_cnt, cg = carry_gs;
    int cnt = block_scan<false>(is_new, sh) + cc;
    int gs = max(block_scan<true>(is_new ? i : 0, sh), cg);
    if (valid) {
      int p = i + 1;
      if (p >= n_pos) {
        flag(err, GENRANK_DERR_POS_RANGE);
        p = n_pos - 1;
      }
      pos[s + i] = p;
      req_idx[s + i] = min(cnt, n_ri - 1);
      rt_bucket[s + i] = gs > 0 ? time_bucket(t - ts[s + gs - 1], n_rt) : 0;
    }
    const int last = min(c0 + (int)blockDim.x, n) - 1;
    if (i == last) {
      carry_cnt = cnt;
      carry_gs = gs;
    }
    __syncthreads();
  }
  if (L > n) {
    const long long t_req = ts[s + n];
    const long long tl = n > 0 ? ts[s + n - 1] : t_req;
    if (threadIdx.x == 0 && n > 0 && t_req < tl) flag(err, GENRANK_DERR_TS_ORDER);
    const bool new_req = (n == 0) || (t_req > tl);
    const int cnt = carry_cnt + (new_req ? 1 : 0);
    const int gs = new_req ? n : carry_gs;
    const int b = gs > 0 ? time_bucket(t_req - ts[s + gs - 1], n_rt) : 0;
    int p = n + 1;
    if (p >= n_pos) {
      if (threadIdx.x == 0) flag(err, GENRANK_DERR_POS_RANGE);
      p = n_pos - 1;
    }
    for (int i = n + threadIdx.x; i < L; i += blockDim.x) {
      if (ts[s + i] != t_req) flag(err, GENRANK_DERR_TS_ORDER);
      pos[s + i] = p;
      req_idx[s + i] = min(cnt, n_ri - 1);
      rt_bucket[s + i] = b;
    }
  }
}

// Gather-sum, one warp per group of 32 tokens: the warp finds the user of its first
// token with a 32-way search of seq_offsets, each lane loads one token's ids
// (coalesced) and walks to that token's user, then the warp gathers the tokens' five
// rows with 16-byte vector loads, the row indices broadcast from their lanes by
// shuffles, two tokens' loads in flight together.  The rows are summed in fp32 and
// rounded once.  At most 64 registers per thread keep four blocks resident per SM.
// kNorm (bf16, d = 512): instead of E, each row is written as its fp32 value and its
// RMSNorm in bf16 (the first pre-norm block's input), one token at a time.
template <typename T, bool kNorm>
__global__ void __launch_bounds__(256, 4) k_embed_fwd(
    int B, long long Ttok, const int32_t* __restrict__ off, const int32_t* __restrict__ hist_len,
    const int32_t* __restrict__ item_ids, const int32_t* __restrict__ action_ids,
    const T* __restrict__ item_tab, long long n_item, const T* __restrict__ action_tab,
    int n_action, const T* __restrict__ pos_tab, const T* __restrict__ ri_tab,
    const T* __restrict__ rt_tab, int d, int n_pos, int n_ri, int n_rt,
    const int32_t* __restrict__ pos, const int32_t* __restrict__ req_idx,
    const int32_t* __restrict__ rt_bucket, T* __restrict__ E, int tokens_per_warp, int32_t* err,
    float* __restrict__ x_out = nullptr, T* __restrict__ a_out = nullptr, float eps = 0.f) {
  constexpr int V = Elem<T>::kPerVec;
  constexpr int U = 2;  // tokens whose row gathers are in flight together
  const int lane = threadIdx.x & 31;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long tend = min(Ttok, (long long)off[B]);
  const int nv = d / V;
  for (long long t0 = warp * tokens_per_warp; t0 < min(tend, (warp + 1) * tokens_per_warp);
       t0 += 32) {
    // one token per lane: its owner, and its five row indices (coalesced id loads)
    const long long t = t0 + lane;
    const bool live = t < tend;
    int u = warp_find_user(off, B, t0);
    long long it = 0;
    int a = 0, p = 0, r = 0, b = 0;
    if (live) {
      while (u < B - 1 && t >= off[u + 1]) ++u;
      const bool cand = (t - off[u]) >= hist_len[u];
      it = item_ids[t];
      if (it < 0 || it >= n_item) {
        flag(err, GENRANK_DERR_ITEM_ID);
        it = it < 0 ? 0 : n_item - 1;
      }
      a = n_action;  // the mask-action row M
      if (!cand) {
        a = action_ids[t];
        if (a < 0 || a >= n_action) {
          flag(err, GENRANK_DERR_ACTION_ID);
          a = a < 0 ? 0 : n_action - 1;
        }
      }
      p = pos[t];
      r = req_idx[t];
      b = rt_bucket[t];
      if (p < 0 || p >= n_pos || r < 0 || r >= n_ri || b < 0 || b >= n_rt) {
        // only reachable when the metadata pass rejected this user's layout
        flag(err, GENRANK_DERR_INDEX);
        p = min(max(p, 0), n_pos - 1);
        r = min(max(r, 0), n_ri - 1);
        b = min(max(b, 0), n_rt - 1);
      }
    }
    const int nt = (int)min(32LL, tend - t0);
    if constexpr (kNorm) {
      // one token at a time: the lane's two 8-column vectors of the row (d = 512) are
      // summed, rounded to the table type (E's value), written as the fp32 x row, and
      // normalised with the row's sum of squares (the same lanes, order and
      // reduction as the RMSNorm pass over E, so the result is the same bit for bit)
      for (int k = 0; k < nt; ++k) {
        const uint4* rw[5];
        rw[0] = reinterpret_cast<const uint4*>(item_tab + __shfl_sync(0xffffffffu, it, k) * d);
        rw[1] = reinterpret_cast<const uint4*>(action_tab +
                                               (long long)__shfl_sync(0xffffffffu, a, k) * d);
        rw[2] = reinterpret_cast<const uint4*>(pos_tab +
                                               (long long)__shfl_sync(0xffffffffu, p, k) * d);
        rw[3] = reinterpret_cast<const uint4*>(ri_tab +
                                               (long long)__shfl_sync(0xffffffffu, r, k) * d);
        rw[4] = reinterpret_cast<const uint4*>(rt_tab +
                                               (long long)__shfl_sync(0xffffffffu, b, k) * d);
        uint4 xv[2][5];
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
          for (int c = 0; c < 5; ++c) xv[w][c] = __ldg(rw[c] + lane + 32 * w);
        float f[2][V];
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          float g[V];
          Elem<T>::unpack(xv[w][0], f[w]);
#pragma unroll
          for (int c = 1; c < 5; ++c) {
            Elem<T>::unpack(xv[w][c], g);
#pragma unroll
            for (int e = 0; e < V; ++e) f[w][e] += g[e];
          }
          Elem<T>::unpack(Elem<T>::pack(f[w]), f[w]);  // E's rounded value
#pragma unroll
          for (int e = 0; e < V; ++e) ss = fmaf(f[w][e], f[w][e], ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rn = rsqrtf(ss / (float)d + eps);
        const long long row = t0 + k;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int c0 = (lane + 32 * w) * V;
          float4* xo = reinterpret_cast<float4*>(x_out + row * d + c0);
#pragma unroll
          for (int e = 0; e < V; e += 4)
            xo[e / 4] = make_float4(f[w][e], f[w][e + 1], f[w][e + 2], f[w][e + 3]);
          float h[V];
#pragma unroll
          for (int e = 0; e < V; ++e) h[e] = f[w][e] * rn;
          *reinterpret_cast<uint4*>(a_out + row * d + c0) = Elem<T>::pack(h);
        }
      }
    } else {
    // the warp gathers the tokens' rows U at a time, indices broadcast from their lanes
    for (int k = 0; k < nt; k += U) {
      const uint4* rows[U][5];
#pragma unroll
      for (int q = 0; q < U; ++q) {
        const int src = min(k + q, nt - 1);
        const long long itq = __shfl_sync(0xffffffffu, it, src);
        rows[q][0] = reinterpret_cast<const uint4*>(item_tab + itq * d);
        rows[q][1] = reinterpret_cast<const uint4*>(
            action_tab + (long long)__shfl_sync(0xffffffffu, a, src) * d);
        rows[q][2] = reinterpret_cast<const uint4*>(
            pos_tab + (long long)__shfl_sync(0xffffffffu, p, src) * d);
        rows[q][3] = reinterpret_cast<const uint4*>(
            ri_tab + (long long)__shfl_sync(0xffffffffu, r, src) * d);
        rows[q][4] = reinterpret_cast<const uint4*>(
            rt_tab + (long long)__shfl_sync(0xffffffffu, b, src) * d);
      }
      for (int v = lane; v < nv; v += 32) {
        uint4 x[U][5];
#pragma unroll
        for (int q = 0; q < U; ++q)
#pragma unroll
          for (int c = 0; c < 5; ++c) x[q][c] = __ldg(rows[q][c] + v);
#pragma unroll
        for (int q = 0; q < U; ++q) {
          float f[V], g[V];
          Elem<T>::unpack(x[q][0], f);
#pragma unroll
          for (int c = 1; c < 5; ++c) {
            Elem<T>::unpack(x[q][c], g);
#pragma unroll
            for (int e = 0; e < V; ++e) f[e] += g[e];
          }
          if (k + q < nt) reinterpret_cast<uint4*>(E + (t0 + k + q) * d)[v] = Elem<T>::pack(f);
        }
      }
    }
    }
  }
}

// ------------------------------------------------------------------------------------------
// backward: scatter-add dE into the five fp32 gradient tables
// ------------------------------------------------------------------------------------------
// Grid (token chunks, column slices of kCols).  The small tables (action, pos,
// ri, rt) are accumulated for the CTA's column slice in shared memory and added
// to global memory once at the end; item rows go straight to global memory with
// vector reductions.  Without room in shared memory every table goes straight
// to global memory.
constexpr int kBwdCols = 64;

GR_DEVICE void red_add_v2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

template <typename T, bool kSmem>
__global__ void __launch_bounds__(1024) k_embed_bwd(
    int B, long long Ttok, const int32_t* __restrict__ off, const int32_t* __restrict__ hist_len,
    const int32_t* __restrict__ item_ids, const int32_t* __restrict__ action_ids,
    const int32_t* __restrict__ pos, const int32_t* __restrict__ req_idx,
    const int32_t* __restrict__ rt_bucket, const T* __restrict__ dE, int d,
    float* __restrict__ g_item, long long n_item, float* __restrict__ g_action, int n_action,
    float* __restrict__ g_pos, int n_pos, float* __restrict__ g_ri, int n_ri,
    float* __restrict__ g_rt, int n_rt, int tokens_per_warp, int32_t* err) {
  extern __shared__ float acc[];  // [rows_small][kBwdCols] when kSmem
  const int n_act_rows = n_action + 1;
  const int rows_small = n_act_rows + n_pos + n_ri + n_rt;
  float* s_action = acc;
  float* s_pos = s_action + n_act_rows * kBwdCols;
  float* s_ri = s_pos + n_pos * kBwdCols;
  float* s_rt = s_ri + n_ri * kBwdCols;
  if (kSmem) {
    for (int i = threadIdx.x; i < rows_small * kBwdCols; i += blockDim.x) acc[i] = 0.f;
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int c0 = blockIdx.y * kBwdCols;
  const int col = c0 + 2 * lane;  // each lane owns two adjacent columns
  const bool col_ok = col < d;
  const long long tend = min(Ttok, (long long)off[B]);
  const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  for (long long t0 = warp * tokens_per_warp; t0 < min(tend, (warp + 1) * tokens_per_warp);
       t0 += 32) {
    // one token per lane: its owner and its five row indices (coalesced id loads)
    const long long t = t0 + lane;
    int u = warp_find_user(off, B, t0);
    long long it = -1;
    int a = 0, p = 0, r = 0, b = 0;
    if (t < tend) {
      while (u < B - 1 && t >= off[u + 1]) ++u;
      const bool cand = (t - off[u]) >= hist_len[u];
      it = item_ids[t];
      a = cand ? n_action : action_ids[t];
      p = pos[t];
      r = req_idx[t];
      b = rt_bucket[t];
      const bool bad = it < 0 || it >= n_item || a < 0 || a > n_action || p < 0 ||
                       p >= n_pos || r < 0 || r >= n_ri || b < 0 || b >= n_rt;
      if (bad) {
        flag(err, GENRANK_DERR_INDEX);
        it = -1;  // skipped below
      }
    }
    const int nt = (int)min(32LL, tend - t0);
    // the warp adds the tokens' gradient slices, two tokens' dE loads in flight
    for (int k = 0; k < nt; k += 2) {
      long long itq[2];
      int aq[2], pq[2], rq[2], bq[2];
      float g0[2], g1[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int src = min(k + q, nt - 1);
        itq[q] = __shfl_sync(0xffffffffu, it, src);
        aq[q] = __shfl_sync(0xffffffffu, a, src);
        pq[q] = __shfl_sync(0xffffffffu, p, src);
        rq[q] = __shfl_sync(0xffffffffu, r, src);
        bq[q] = __shfl_sync(0xffffffffu, b, src);
        g0[q] = g1[q] = 0.f;
        if (col_ok && itq[q] >= 0 && k + q < nt) {
          if (sizeof(T) == 2) {
            const uint32_t w =
                *reinterpret_cast<const uint32_t*>(dE + (t0 + k + q) * d + col);
            g0[q] = bf16_lo(w);
            g1[q] = bf16_hi(w);
          } else {
            const float2 w = *reinterpret_cast<const float2*>(dE + (t0 + k + q) * d + col);
            g0[q] = w.x;
            g1[q] = w.y;
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (!col_ok || itq[q] < 0 || k + q >= nt) continue;
        red_add_v2(g_item + itq[q] * d + col, g0[q], g1[q]);
        if (kSmem) {
          // a slice row holds column 2l + k at k * 32 + l, so each of these adds covers
          // 32 consecutive words (one per bank)
          atomicAdd(s_action + aq[q] * kBwdCols + lane, g0[q]);
          atomicAdd(s_action + aq[q] * kBwdCols + 32 + lane, g1[q]);
          atomicAdd(s_pos + pq[q] * kBwdCols + lane, g0[q]);
          atomicAdd(s_pos + pq[q] * kBwdCols + 32 + lane, g1[q]);
          atomicAdd(s_ri + rq[q] * kBwdCols + lane, g0[q]);
          atomicAdd(s_ri + rq[q] * kBwdCols + 32 + lane, g1[q]);
          atomicAdd(s_rt + bq[q] * kBwdCols + lane, g0[q]);
          atomicAdd(s_rt + bq[q] * kBwdCols + 32 + lane, g1[q]);
        } else {
          red_add_v2(g_action + (long long)aq[q] * d + col, g0[q], g1[q]);
          red_add_v2(g_pos + (long long)pq[q] * d + col, g0[q], g1[q]);
          red_add_v2(g_ri + (long long)rq[q] * d + col, g0[q], g1[q]);
          red_add_v2(g_rt + (long long)bq[q] * d + col, g0[q], g1[q]);
        }
      }
    }
  }
  if (kSmem) {
    __syncthreads();
    for (int i = threadIdx.x; i < rows_small * kBwdCols; i += blockDim.x) {
      const float v = acc[i];
      const int j = i % kBwdCols;  // column 2 (j % 32) + j / 32 of the slice
      const int row = i / kBwdCols, c = c0 + 2 * (j & 31) + (j >> 5);
      if (v == 0.f || c >= d) continue;
      float* dst;
      if (row < n_act_rows) dst = g_action + (long long)row * d;
      else if (row < n_act_rows + n_pos) dst = g_pos + (long long)(row - n_act_rows) * d;
      else if (row < n_act_rows + n_pos + n_ri) dst = g_ri + (long long)(row - n_act_rows - n_pos) * d;
      else dst = g_rt + (long long)(row - n_act_rows - n_pos - n_ri) * d;
      atomicAdd(dst + c, v);
    }
  }
}

// ------------------------------------------------------------------------------------------
// host launchers
// ------------------------------------------------------------------------------------------
static int sm_count() {
  const int n = sm_count_current();
  return n > 0 ? n : 148;  // only sizes the grid
}

int launch_embed_fwd(const EmbedFwdArgs& a, cudaStream_t st) {
  k_token_meta<<<a.B, 256, 0, st>>>(a.B, a.T, a.off, a.hist_len, a.ts, a.n_pos, a.n_ri, a.n_rt,
                                    a.pos, a.req_idx, a.rt_bucket, a.err);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  if (a.T == 0) return GENRANK_OK;
  // one 32-token group per warp (more when the batch is large), so that ~16 blocks of
  // 256 threads stay resident per SM
  const long long warps_target = (long long)sm_count() * 64 * 4;
  int tpw = 32 * (int)max(1LL, (a.T + 32 * warps_target - 1) / (32 * warps_target));
  long long warps = (a.T + tpw - 1) / tpw;
  long long blocks = (warps + 7) / 8;
  if (a.x_out) {  // bf16 tables, d = 512 (checked by the caller)
    using T = __nv_bfloat16;
    k_embed_fwd<T, true><<<(unsigned)blocks, 256, 0, st>>>(
        a.B, a.T, a.off, a.hist_len, a.item_ids, a.action_ids, (const T*)a.item_tab, a.n_item,
        (const T*)a.action_tab, a.n_action, (const T*)a.pos_tab, (const T*)a.ri_tab,
        (const T*)a.rt_tab, a.d, a.n_pos, a.n_ri, a.n_rt, a.pos, a.req_idx, a.rt_bucket, nullptr,
        tpw, a.err, a.x_out, (T*)a.a_out, a.eps);
  } else if (a.dtype == GENRANK_BF16) {
    using T = __nv_bfloat16;
    k_embed_fwd<T, false><<<(unsigned)blocks, 256, 0, st>>>(
        a.B, a.T, a.off, a.hist_len, a.item_ids, a.action_ids, (const T*)a.item_tab, a.n_item,
        (const T*)a.action_tab, a.n_action, (const T*)a.pos_tab, (const T*)a.ri_tab,
        (const T*)a.rt_tab, a.d, a.n_pos, a.n_ri, a.n_rt, a.pos, a.req_idx, a.rt_bucket, (T*)a.E,
        tpw, a.err);
  } else {
    using T = float;
    k_embed_fwd<T, false><<<(unsigned)blocks, 256, 0, st>>>(
        a.B, a.T, a.off, a.hist_len, a.item_ids, a.action_ids, (const T*)a.item_tab, a.n_item,
        (const T*)a.action_tab, a.n_action, (const T*)a.pos_tab, (const T*)a.ri_tab,
        (const T*)a.rt_tab, a.d, a.n_pos, a.n_ri, a.n_rt, a.pos, a.req_idx, a.rt_bucket, (T*)a.E,
        tpw, a.err);
  }
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

template <typename T, bool kSmem>
static int launch_bwd_t(const EmbedBwdArgs& a, cudaStream_t st) {
  const int rows_small = a.n_action + 1 + a.n_pos + a.n_ri + a.n_rt;
  const size_t smem = kSmem ? (size_t)rows_small * kBwdCols * sizeof(float) : 0;
  if (kSmem) {
    if (cudaFuncSetAttribute(k_embed_bwd<T, kSmem>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return GENRANK_ERR_CUDA;
  }
  const int slices = (a.d + kBwdCols - 1) / kBwdCols;
  // about two waves of one 1024-thread CTA per SM over all slices
  const long long ctas_per_slice = max(1LL, (long long)(2 * sm_count() + slices - 1) / slices);
  const long long warps = ctas_per_slice * 32;
  // tokens per warp: whole groups of 32 (one token's ids per lane)
  const int tpw = 32 * (int)max(1LL, (a.T + 32 * warps - 1) / (32 * warps));
  const long long chunks = max(1LL, ((a.T + tpw - 1) / tpw + 31) / 32);
  dim3 grid((unsigned)chunks, (unsigned)slices);
  k_embed_bwd<T, kSmem><<<grid, 1024, smem, st>>>(
      a.B, a.T, a.off, a.hist_len, a.item_ids, a.action_ids, a.pos, a.req_idx, a.rt_bucket,
      (const T*)a.dE, a.d, a.g_item, a.n_item, a.g_action, a.n_action, a.g_pos, a.n_pos, a.g_ri,
      a.n_ri, a.g_rt, a.n_rt, tpw, a.err);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

int launch_embed_bwd(const EmbedBwdArgs& a, cudaStream_t st) {
  if (a.T == 0) return GENRANK_OK;
  const size_t rows_small = (size_t)a.n_action + 1 + a.n_pos + a.n_ri + a.n_rt;
  const bool smem_ok = rows_small * kBwdCols * sizeof(float) <= 224 * 1024;
  if (a.dtype == GENRANK_BF16)
    return smem_ok ? launch_bwd_t<__nv_bfloat16, true>(a, st)
                   : launch_bwd_t<__nv_bfloat16, false>(a, st);
  return smem_ok ? launch_bwd_t<float, true>(a, st) : launch_bwd_t<float, false>(a, st);
}

}  // namespace gr
