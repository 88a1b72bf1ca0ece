// CUDA-core masked ALiBi attention, forward and backward.
//
// Used for fp32 storage (and bf16 with head dim 32), where tensor-core tiles do
// not apply.  Semantics as in the ALiBi score of "GenRank [2025]" chapter notes
// §1.4.2 and the candidate mask of §1.4.1: history rows are causal, candidate
// rows see all history and themselves.  The bias is evaluated literally,
// -m|p_i - p_j| - m_t|t_i - t_j|, with exact integer distances.
//
// Each query (or key) row is handled by G = DH/32 adjacent threads, each owning
// 32 of the DH columns; keys (or queries) are staged through shared memory in
// chunks of 32 rows.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace gr {

constexpr int kChunk = 32;

template <typename T>
GR_DEVICE void load32(const T* p, float* f) {
#pragma unroll
  for (int c = 0; c < 32; ++c) f[c] = Elem<T>::load(p + c);
}

template <int G>
GR_DEVICE float pair_sum(float x) {
  if (G == 2) {
    const unsigned lane = threadIdx.x & 31;
    const unsigned m = 3u << (lane & ~1u);
    x += __shfl_xor_sync(m, x, 1);
  }
  return x;
}

struct UserSpan {
  long long s;
  int L, n;
  bool ok;
};

GR_DEVICE UserSpan user_span(const AttnArgs& a, int u) {
  UserSpan r;
  r.s = a.off[u];
  long long e = a.off[u + 1];
  r.n = a.hist_len[u];
  r.ok = !(r.s < 0 || e < r.s || e > a.T);
  r.L = r.ok ? (int)(e - r.s) : 0;
  if (r.ok && (r.n < 0 || r.n > r.L)) r.n = max(0, min(r.n, r.L));
  return r;
}

// ------------------------------------------------------------------------------------------
// forward
// ------------------------------------------------------------------------------------------
template <typename T, int DH>
__global__ void __launch_bounds__(128) k_attn_fwd_simt(const __grid_constant__ AttnArgs a) {
  constexpr int G = DH / 32, R = 128 / G;
  __shared__ float sK[kChunk][DH + 1], sV[kChunk][DH + 1];
  __shared__ int sP[kChunk];
  __shared__ long long sT[kChunk];
  const int u = blockIdx.x, h = blockIdx.y;
  const UserSpan us = user_span(a, u);
  if (!us.ok) {
    if (threadIdx.x == 0 && blockIdx.z == 0 && h == 0) flag(a.err, GENRANK_DERR_LAYOUT);
    return;
  }
  const int q0 = blockIdx.z * R;
  if (q0 >= us.L) return;
  const int r = threadIdx.x / G, g = threadIdx.x % G;
  const int i = q0 + r;
  const bool row = i < us.L;
  const int n = us.n;
  const int lim = min(i, n - 1);
  const T* Q = (const T*)a.q;
  const T* K = (const T*)a.k;
  const T* Vv = (const T*)a.v;
  float q[32], o[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) o[c] = 0.f;
  if (row) load32(Q + (us.s + i) * a.tok_stride + h * DH + g * 32, q);
  else {
#pragma unroll
    for (int c = 0; c < 32; ++c) q[c] = 0.f;
  }
  const float sp = a.slope_pos[h], st = a.slope_time[h];
  const int p_i = row ? a.pos[us.s + i] : 0;
  const long long t_i = row ? a.ts[us.s + i] : 0;
  float m = -INFINITY, l = 0.f;
  const int kend = min(q0 + R, n);
  for (int c0 = 0; c0 < kend; c0 += kChunk) {
    __syncthreads();
    for (int x = threadIdx.x; x < kChunk * DH; x += blockDim.x) {
      const int j = x / DH, c = x % DH;
      if (c0 + j < kend) {
        const long long rowoff = (us.s + c0 + j) * a.tok_stride + h * DH + c;
        sK[j][c] = Elem<T>::load(K + rowoff);
        sV[j][c] = Elem<T>::load(Vv + rowoff);
      }
    }
    for (int j = threadIdx.x; j < kChunk; j += blockDim.x) {
      if (c0 + j < kend) {
        sP[j] = a.pos[us.s + c0 + j];
        sT[j] = a.ts[us.s + c0 + j];
      }
    }
    __syncthreads();
    if (!row) continue;
    const int jn = min(kChunk, lim - c0 + 1);
    if (jn <= 0) continue;
    float sc[kChunk];
    float cmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      if (j < jn) {
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) dot = fmaf(q[c], sK[j][g * 32 + c], dot);
        dot = pair_sum<G>(dot);
        const float bias = -sp * fabsf((float)(p_i - sP[j])) -
                           st * (float)llabs(t_i - sT[j]);
        sc[j] = fmaf(dot, a.scale, bias);
        cmax = fmaxf(cmax, sc[j]);
      }
    }
    const float mn = fmaxf(m, cmax);
    const float corr = expf(m - mn);
    l *= corr;
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] *= corr;
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      if (j < jn) {
        const float p = expf(sc[j] - mn);
        l += p;
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = fmaf(p, sV[j][g * 32 + c], o[c]);
      }
    }
    m = mn;
  }
  if (!row) return;
  if (i >= n) {  // a candidate also sees itself; its bias to itself is zero
    float kk[32], vv[32];
    load32(K + (us.s + i) * a.tok_stride + h * DH + g * 32, kk);
    load32(Vv + (us.s + i) * a.tok_stride + h * DH + g * 32, vv);
    float dot = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) dot = fmaf(q[c], kk[c], dot);
    dot = pair_sum<G>(dot);
    const float sc = dot * a.scale;
    const float mn = fmaxf(m, sc);
    const float corr = expf(m - mn), p = expf(sc - mn);
    l = l * corr + p;
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = fmaf(p, vv[c], o[c] * corr);
    m = mn;
  }
  const float inv = 1.f / l;
  T* O = (T*)a.o + (us.s + i) * a.o_stride + h * DH + g * 32;
#pragma unroll
  for (int c = 0; c < 32; ++c) Elem<T>::store(O + c, o[c] * inv);
  if (a.lse && g == 0) a.lse[(long long)h * a.T + us.s + i] = m + logf(l);
}

// ------------------------------------------------------------------------------------------
// backward
// ------------------------------------------------------------------------------------------
// D_i = rowsum(dO_i * O_i) per head, into the workspace [H, T].
template <typename T>
__global__ void k_attn_bwd_dot(const __grid_constant__ AttnArgs a, float* Dw) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= a.T * a.H) return;
  const long long t = idx / a.H;
  const int h = (int)(idx % a.H);
  const T* O = (const T*)a.o + t * a.o_stride + h * a.dh;
  const T* G = (const T*)a.dO + t * a.o_stride + h * a.dh;
  float acc = 0.f;
  for (int c = 0; c < a.dh; ++c) acc = fmaf(Elem<T>::load(O + c), Elem<T>::load(G + c), acc);
  Dw[(long long)h * a.T + t] = acc;
}

// dQ: one query row per G threads; keys staged in shared memory.
template <typename T, int DH>
__global__ void __launch_bounds__(128) k_attn_bwd_dq_simt(const __grid_constant__ AttnArgs a,
                                                         const float* __restrict__ Dw) {
  constexpr int G = DH / 32, R = 128 / G;
  __shared__ float sK[kChunk][DH + 1], sV[kChunk][DH + 1];
  __shared__ int sP[kChunk];
  __shared__ long long sT[kChunk];
  const int u = blockIdx.x, h = blockIdx.y;
  const UserSpan us = user_span(a, u);
  if (!us.ok) {
    if (threadIdx.x == 0 && blockIdx.z == 0 && h == 0) flag(a.err, GENRANK_DERR_LAYOUT);
    return;
  }
  const int q0 = blockIdx.z * R;
  if (q0 >= us.L) return;
  const int r = threadIdx.x / G, g = threadIdx.x % G;
  const int i = q0 + r;
  const bool row = i < us.L;
  const int n = us.n;
  const int lim = min(i, n - 1);
  const T* Q = (const T*)a.q;
  const T* K = (const T*)a.k;
  const T* Vv = (const T*)a.v;
  float q[32], go[32], dq[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) dq[c] = 0.f;
  float lse_i = 0.f, D_i = 0.f;
  int p_i = 0;
  long long t_i = 0;
  if (row) {
    load32(Q + (us.s + i) * a.tok_stride + h * DH + g * 32, q);
    load32((const T*)a.dO + (us.s + i) * a.o_stride + h * DH + g * 32, go);
    lse_i = a.lse_in[(long long)h * a.T + us.s + i];
    D_i = Dw[(long long)h * a.T + us.s + i];
    p_i = a.pos[us.s + i];
    t_i = a.ts[us.s + i];
  }
  const float sp = a.slope_pos[h], st = a.slope_time[h];
  const int kend = min(q0 + R, n);
  for (int c0 = 0; c0 < kend; c0 += kChunk) {
    __syncthreads();
    for (int x = threadIdx.x; x < kChunk * DH; x += blockDim.x) {
      const int j = x / DH, c = x % DH;
      if (c0 + j < kend) {
        const long long rowoff = (us.s + c0 + j) * a.tok_stride + h * DH + c;
        sK[j][c] = Elem<T>::load(K + rowoff);
        sV[j][c] = Elem<T>::load(Vv + rowoff);
      }
    }
    for (int j = threadIdx.x; j < kChunk; j += blockDim.x) {
      if (c0 + j < kend) {
        sP[j] = a.pos[us.s + c0 + j];
        sT[j] = a.ts[us.s + c0 + j];
      }
    }
    __syncthreads();
    if (!row) continue;
    const int jn = min(kChunk, lim - c0 + 1);
    for (int j = 0; j < jn; ++j) {
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        dot = fmaf(q[c], sK[j][g * 32 + c], dot);
        dp = fmaf(go[c], sV[j][g * 32 + c], dp);
      }
      dot = pair_sum<G>(dot);
      dp = pair_sum<G>(dp);
      const float s = fmaf(dot, a.scale,
                           -sp * fabsf((float)(p_i - sP[j])) - st * (float)llabs(t_i - sT[j]));
      const float p = expf(s - lse_i);
      const float ds = p * (dp - D_i);
#pragma unroll
      for (int c = 0; c < 32; ++c) dq[c] = fmaf(ds, sK[j][g * 32 + c], dq[c]);
    }
  }
  if (!row) return;
  if (i >= n) {
    float kk[32], vv[32];
    load32(K + (us.s + i) * a.tok_stride + h * DH + g * 32, kk);
    load32(Vv + (us.s + i) * a.tok_stride + h * DH + g * 32, vv);
    float dot = 0.f, dp = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      dot = fmaf(q[c], kk[c], dot);
      dp = fmaf(go[c], vv[c], dp);
    }
    dot = pair_sum<G>(dot);
    dp = pair_sum<G>(dp);
    const float p = expf(dot * a.scale - lse_i);
    const float ds = p * (dp - D_i);
#pragma unroll
    for (int c = 0; c < 32; ++c) dq[c] = fmaf(ds, kk[c], dq[c]);
  }
  T* out = (T*)a.dq + (us.s + i) * a.tok_stride + h * DH + g * 32;
#pragma unroll
  for (int c = 0; c < 32; ++c) Elem<T>::store(out + c, dq[c] * a.scale);
}

// dK, dV: one key row per G threads; the queries that see the block's keys are
// staged in shared memory.  History key j is seen by every row i >= j of the
// user; a candidate key only by itself.
template <typename T, int DH>
__global__ void __launch_bounds__(128) k_attn_bwd_dkv_simt(const __grid_constant__ AttnArgs a,
                                                          const float* __restrict__ Dw) {
  constexpr int G = DH / 32, R = 128 / G;
  __shared__ float sQ[kChunk][DH + 1], sG[kChunk][DH + 1];
  __shared__ float sL[kChunk], sD[kChunk];
  __shared__ int sP[kChunk];
  __shared__ long long sT[kChunk];
  const int u = blockIdx.x, h = blockIdx.y;
  const UserSpan us = user_span(a, u);
  if (!us.ok) {
    if (threadIdx.x == 0 && blockIdx.z == 0 && h == 0) flag(a.err, GENRANK_DERR_LAYOUT);
    return;
  }
  const int k0 = blockIdx.z * R;
  if (k0 >= us.L) return;
  const int r = threadIdx.x / G, g = threadIdx.x % G;
  const int j = k0 + r;
  const bool row = j < us.L;
  const int n = us.n;
  const T* Q = (const T*)a.q;
  const T* K = (const T*)a.k;
  const T* Vv = (const T*)a.v;
  const T* GO = (const T*)a.dO;
  float kk[32], vv[32], dk[32], dv[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  int p_j = 0;
  long long t_j = 0;
  if (row) {
    load32(K + (us.s + j) * a.tok_stride + h * DH + g * 32, kk);
    load32(Vv + (us.s + j) * a.tok_stride + h * DH + g * 32, vv);
    p_j = a.pos[us.s + j];
    t_j = a.ts[us.s + j];
  }
  const float sp = a.slope_pos[h], st = a.slope_time[h];
  // queries needed by the block's history keys: rows [k0, L)
  const int qbeg = k0 < n ? k0 : us.L;
  for (int c0 = qbeg; c0 < us.L; c0 += kChunk) {
    __syncthreads();
    for (int x = threadIdx.x; x < kChunk * DH; x += blockDim.x) {
      const int ii = x / DH, c = x % DH;
      if (c0 + ii < us.L) {
        sQ[ii][c] = Elem<T>::load(Q + (us.s + c0 + ii) * a.tok_stride + h * DH + c);
        sG[ii][c] = Elem<T>::load(GO + (us.s + c0 + ii) * a.o_stride + h * DH + c);
      }
    }
    for (int ii = threadIdx.x; ii < kChunk; ii += blockDim.x) {
      if (c0 + ii < us.L) {
        sP[ii] = a.pos[us.s + c0 + ii];
        sT[ii] = a.ts[us.s + c0 + ii];
        sL[ii] = a.lse_in[(long long)h * a.T + us.s + c0 + ii];
        sD[ii] = Dw[(long long)h * a.T + us.s + c0 + ii];
      }
    }
    __syncthreads();
    if (!row || j >= n) continue;
    for (int ii = 0; ii < kChunk; ++ii) {
      const int i = c0 + ii;
      if (i < j || i >= us.L) continue;
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        dot = fmaf(sQ[ii][g * 32 + c], kk[c], dot);
        dp = fmaf(sG[ii][g * 32 + c], vv[c], dp);
      }
      dot = pair_sum<G>(dot);
      dp = pair_sum<G>(dp);
      const float s = fmaf(dot, a.scale,
                           -sp * fabsf((float)(sP[ii] - p_j)) - st * (float)llabs(sT[ii] - t_j));
      const float p = expf(s - sL[ii]);
      const float ds = p * (dp - sD[ii]);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        dv[c] = fmaf(p, sG[ii][g * 32 + c], dv[c]);
        dk[c] = fmaf(ds, sQ[ii][g * 32 + c], dk[c]);
      }
    }
  }
  if (!row) return;
  if (j >= n) {  // a candidate key is seen only by its own row
    float qq[32], go[32];
    load32(Q + (us.s + j) * a.tok_stride + h * DH + g * 32, qq);
    load32(GO + (us.s + j) * a.o_stride + h * DH + g * 32, go);
    float dot = 0.f, dp = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      dot = fmaf(qq[c], kk[c], dot);
      dp = fmaf(go[c], vv[c], dp);
    }
    dot = pair_sum<G>(dot);
    dp = pair_sum<G>(dp);
    const float p = expf(dot * a.scale - a.lse_in[(long long)h * a.T + us.s + j]);
    const float ds = p * (dp - Dw[(long long)h * a.T + us.s + j]);
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      dv[c] = p * go[c];
      dk[c] = ds * qq[c];
    }
  }
  T* odk = (T*)a.dk + (us.s + j) * a.tok_stride + h * DH + g * 32;
  T* odv = (T*)a.dv + (us.s + j) * a.tok_stride + h * DH + g * 32;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    Elem<T>::store(odk + c, dk[c] * a.scale);
    Elem<T>::store(odv + c, dv[c]);
  }
}

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
template <typename T, int DH>
static int fwd_t(const AttnArgs& a, cudaStream_t st) {
  constexpr int R = 128 / (DH / 32);
  // users on x (up to 2^31 - 1 of them), heads on y, row blocks on z
  const int rblocks = (a.max_seqlen + R - 1) / R;
  if (rblocks == 0) return GENRANK_OK;
  if (rblocks > 65535) return GENRANK_ERR_UNSUPPORTED;
  dim3 grid(a.B, a.H, rblocks);
  k_attn_fwd_simt<T, DH><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

int launch_attn_fwd_simt(const AttnArgs& a, cudaStream_t st) {
  const bool bf = a.dtype == GENRANK_BF16;
  if (a.dh == 32) return bf ? fwd_t<__nv_bfloat16, 32>(a, st) : fwd_t<float, 32>(a, st);
  if (a.dh == 64) return bf ? fwd_t<__nv_bfloat16, 64>(a, st) : fwd_t<float, 64>(a, st);
  return GENRANK_ERR_UNSUPPORTED;
}

size_t attn_bwd_simt_workspace(int B, long long T, int H, int dh, int max_seqlen) {
  (void)B;
  (void)dh;
  (void)max_seqlen;
  return (size_t)T * H * sizeof(float) + 256;
}

template <typename T, int DH>
static int bwd_t(const AttnArgs& a, cudaStream_t st) {
  constexpr int R = 128 / (DH / 32);
  float* Dw = (float*)a.ws;
  const long long nth = a.T * a.H;
  if (nth == 0) return GENRANK_OK;
  k_attn_bwd_dot<T><<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(a, Dw);
  const int rblocks = (a.max_seqlen + R - 1) / R;
  if (rblocks == 0) return GENRANK_OK;
  if (rblocks > 65535) return GENRANK_ERR_UNSUPPORTED;
  dim3 grid(a.B, a.H, rblocks);
  k_attn_bwd_dq_simt<T, DH><<<grid, 128, 0, st>>>(a, Dw);
  k_attn_bwd_dkv_simt<T, DH><<<grid, 128, 0, st>>>(a, Dw);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

int launch_attn_bwd_simt(const AttnArgs& a, cudaStream_t st) {
  const bool bf = a.dtype == GENRANK_BF16;
  if (a.dh == 32) return bf ? bwd_t<__nv_bfloat16, 32>(a, st) : bwd_t<float, 32>(a, st);
  if (a.dh == 64) return bf ? bwd_t<__nv_bfloat16, 64>(a, st) : bwd_t<float, 64>(a, st);
  return GENRANK_ERR_UNSUPPORTED;
}

}  // namespace gr
