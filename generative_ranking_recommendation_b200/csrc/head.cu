// Candidate-side helpers ("GenRank [2025]" chapter notes §1.3.1: the loss and the
// ranking output live at candidate positions):
//   * the logits of a one-block scorer without FFN, z = x . w + o . u at candidate rows
//     (u = W_o w_head is formed by the caller);
//   * the gather of candidate rows that the last block's projections and FFN run on.
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {

// One warp per candidate: each lane reads 16-byte vectors of the two rows and the
// matching fp32 weights, and the warp reduces the two dot products in fp32.
template <typename T>
__global__ void __launch_bounds__(256) k_cand_logits(const CandLogitsArgs a) {
  constexpr int V = Elem<T>::kPerVec;
  const int lane = threadIdx.x & 31;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long c = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); c < a.M;
       c += nwarps) {
    const long long row = a.rows[c];
    if (row < 0 || row >= a.T) {
      if (lane == 0) {
        flag(a.err, GENRANK_DERR_INDEX);
        a.z[c] = 0.f;
      }
      continue;
    }
    const T* xr = static_cast<const T*>(a.x) + row * a.x_stride;
    const T* orow = static_cast<const T*>(a.o) + row * a.o_stride;
    float acc = 0.f;
    for (int j = lane * V; j < a.d; j += 32 * V) {
      float xf[V], of[V];
      Elem<T>::unpack(*reinterpret_cast<const uint4*>(xr + j), xf);
      Elem<T>::unpack(*reinterpret_cast<const uint4*>(orow + j), of);
#pragma unroll
      for (int e = 0; e < V; e += 4) {
        const float4 w4 = __ldg(reinterpret_cast<const float4*>(a.w + j + e));
        const float4 u4 = __ldg(reinterpret_cast<const float4*>(a.u + j + e));
        acc = fmaf(xf[e], w4.x, acc);
        acc = fmaf(xf[e + 1], w4.y, acc);
        acc = fmaf(xf[e + 2], w4.z, acc);
        acc = fmaf(xf[e + 3], w4.w, acc);
        acc = fmaf(of[e], u4.x, acc);
        acc = fmaf(of[e + 1], u4.y, acc);
        acc = fmaf(of[e + 2], u4.z, acc);
        acc = fmaf(of[e + 3], u4.w, acc);
      }
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) a.z[c] = acc;
  }
}

int launch_cand_logits(const CandLogitsArgs& a, cudaStream_t st) {
  if (a.M == 0) return GENRANK_OK;
  const int n = sm_count_current();
  const int sms = n > 0 ? n : 148;  // only sizes the grid
  const long long blocks = (a.M + 7) / 8;
  const int grid = (int)(blocks < 16LL * sms ? blocks : 16LL * sms);
  if (a.dtype == GENRANK_BF16)
    k_cand_logits<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  else
    k_cand_logits<float><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

// dst row k = src row rows[k], whole rows of row_bytes (a multiple of 16): one warp per
// row, each lane moving 16-byte vectors.  A row index outside [0, T) is flagged and its
// destination row zeroed.
__global__ void __launch_bounds__(256) k_gather_rows(const GatherRowsArgs a) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  const long long vecs = a.row_bytes / 16;
  for (long long k = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < a.M;
       k += nwarps) {
    const long long row = a.rows[k];
    uint4* d = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.dst) + k * a.dst_stride);
    if (row < 0 || row >= a.T) {
      if (lane == 0) flag(a.err, GENRANK_DERR_INDEX);
      for (long long v = lane; v < vecs; v += 32) d[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4* s =
        reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.src) + row * a.src_stride);
    for (long long v = lane; v < vecs; v += 32) d[v] = __ldg(s + v);
  }
}

int launch_gather_rows(const GatherRowsArgs& a, cudaStream_t st) {
  if (a.M == 0) return GENRANK_OK;
  const int n = sm_count_current();
  const int sms = n > 0 ? n : 148;  // only sizes the grid
  const long long blocks = (a.M + 7) / 8;
  const int grid = (int)(blocks < 16LL * sms ? blocks : 16LL * sms);
  k_gather_rows<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace gr
