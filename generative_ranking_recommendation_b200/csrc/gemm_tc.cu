// Linear layers of the GenRank blocks on 5th-generation tensor cores (sm_100a), with
// the elementwise work around them fused into the epilogue.
//
// The blocks around the attention ("GenRank [2025]" chapter notes §1.4.1: the
// action-oriented layout halves the tokens, so the projections cost half of the
// interleaved layout's) are, per layer of the four-layer workloads:
//   a = rmsnorm(x);  qkv = a Wqkv;  o = attention(qkv);  x += o Wo;
//   a2 = rmsnorm(x);  x += SiLU(a2 W1) W2;  (final: z = rmsnorm(x) . w_head)
// C = A W is computed here as A [M][K] times the transposed weight Wt [N][K] (both
// bf16, K-major), fp32 accumulation in tensor memory, with one of three epilogues:
//   store:     C = bf16(A W)
//   silu:      C = bf16(SiLU(A W))
//   res+rms:   x_out = x_in + A W (fp32, the whole row of d <= 512 columns in one
//              tile), a_out = bf16(x_out / sqrt(mean(x_out^2) + eps)) and, when a head
//              vector is given, z = (x_out / sqrt(...)) . w_head
// so the residual stream is read and written once per update and the normalised
// activations never take a separate pass.
//
// Design, one CTA per SM (persistent), 192 threads:
//   * warp 1 issues TMA loads of 128 x 64 A tiles and BN x 64 Wt tiles (128B swizzle,
//     no multicast) into a ring of stages;
//   * warp 0 (one thread) issues tcgen05.mma M = 128, N = 256, K = 16 (four per 64-wide
//     k-step, two side by side for BN = 512) into a TMEM accumulator; the store and SiLU
//     epilogues double-buffer the accumulator (2 x 256 columns) so a tile's epilogue
//     overlaps the next tile's MMAs; res+rms uses all 512 columns for one tile;
//   * warps 2-5 (one accumulator row per thread) run the epilogue from TMEM.
// Tiles are ordered with the N tiles of one M tile adjacent, so CTAs running them at the
// same time share the A tile in L2.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {
namespace tg {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, 256, 0, 0);  // A K-major, Wt K-major

template <int kEpi>
struct Cfg {
  static constexpr int BN = kEpi == kEpiResRms ? 512 : 256;
  static constexpr int kStages = kEpi == kEpiResRms ? 2 : 4;
  static constexpr int kAccBufs = kEpi == kEpiResRms ? 1 : 2;
  static constexpr uint32_t kABytes = BM * BK * 2;  // 16 KB
  static constexpr uint32_t kBBytes = BN * BK * 2;  // 32 or 64 KB
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kOffBar = kStages * kStageBytes;
  // barriers: full[S], empty[S], acc_full[2], acc_empty[2], done
  static constexpr uint32_t kNumBars = 2 * kStages + 5;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmem = kOffMisc + 16 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "1024-byte aligned stages");
};

struct Params {
  CUtensorMap ta, tb;
  GemmArgs g;
};

GR_DEVICE uint32_t par(int x) { return (uint32_t)(x & 1); }

GR_DEVICE bool wait_warp(uint64_t* bar, uint32_t ph, volatile int* abort_flag, int32_t* err) {
  const bool ok = mbar_wait(bar, ph, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

GR_DEVICE float silu(float v) { return v / (1.f + __expf(-v)); }

// 32 fp32 values to 16 bf16 pairs, stored as four 16-byte vectors at dst.
GR_DEVICE void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                       pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                       pack_bf16(v[8 * q + 6], v[8 * q + 7]));
}

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1) k_gemm_tc(const __grid_constant__ Params P) {
  using C = Cfg<kEpi>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemmArgs& g = P.g;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&P.ta);
    tma_prefetch_desc(&P.tb);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m_tiles = (g.M + BM - 1) / BM;
  const int n_tiles = g.N / C::BN;
  const int tiles = m_tiles * n_tiles;
  const int ksteps = g.K / BK;

  if (warp == 1) {
    // ------------------------------------------------------------------ TMA producer
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int mt = t / n_tiles, nt = t - mt * n_tiles;
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const int st = it % C::kStages;
        if (!wait_warp(&empty[st], par(it / C::kStages) ^ 1u, abort_flag, g.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* sa = smem + st * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          mbar_expect_tx(&full[st], C::kStageBytes);
          tma_load_2d(sa, &P.ta, &full[st], ks * BK, mt * BM);
#pragma unroll
          for (int h = 0; h < C::BN / 256; ++h)
            tma_load_2d(sb + h * (256 * BK * 2), &P.tb, &full[st], ks * BK, nt * C::BN + 256 * h);
        }
      }
    }
    // the copies issued last land before the CTA exits
    if (lane == 0)
      for (int x = max(0, it - C::kStages); x < it; ++x)
        mbar_drain(&full[x % C::kStages], par(x / C::kStages));
  } else if (warp == 0) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
        const int buf = tc % C::kAccBufs;
        if (!mbar_wait(&acc_empty[buf], par(tc / C::kAccBufs) ^ 1u, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * 256);
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int st = it % C::kStages;
          if (!mbar_wait(&full[st], par(it / C::kStages), abort_flag, g.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
#pragma unroll
            for (int h = 0; h < C::BN / 256; ++h) {
              const uint64_t bd = smem_desc_sw128(sb + h * (256 * BK * 2) + kk * 32, 16, 1024);
              mma_bf16_ss(acc + h * 256, ad, bd, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&empty[st]);  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
      }
      // every MMA issued has completed before TMEM is freed
      mma_commit(done);
      mbar_drain(done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue warps 2-5
    const int q = warp & 3;  // TMEM lane quadrant
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    int tc = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
      const int mt = t / n_tiles, nt = t - mt * n_tiles;
      const int buf = tc % C::kAccBufs;
      if (!wait_warp(&acc_full[buf], par(tc / C::kAccBufs), abort_flag, g.err)) break;
      tc_fence_after();
      const long long row = (long long)mt * BM + q * 32 + lane;
      const bool valid = row < g.M;
      const uint32_t acc = lane_base + (uint32_t)(buf * 256);
      if (kEpi != kEpiResRms) {
        __nv_bfloat16* crow = (__nv_bfloat16*)g.c + row * g.ldc + (long long)nt * C::BN;
#pragma unroll 1
        for (int c = 0; c < C::BN; c += 32) {
          float v[32];
          tmem_ld32(acc + c, v);
          if (kEpi == kEpiSilu) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = silu(v[e]);
          }
          if (valid) store_bf16x32(crow + c, v);
        }
      } else {
        // x_out = x_in + acc over the whole row (d columns), kept in TMEM for the
        // second pass; then the normalised row and the optional head dot product
        const float* xin = g.x_in + row * g.ldx;
        float* xout = g.x_out + row * g.ldx;
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < g.N; c += 32) {
          float v[32];
          tmem_ld32(acc + c, v);
          if (valid) {
            const float4* x4 = reinterpret_cast<const float4*>(xin + c);
            float4* o4 = reinterpret_cast<float4*>(xout + c);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 xv = x4[e];
              xv.x += v[4 * e];
              xv.y += v[4 * e + 1];
              xv.z += v[4 * e + 2];
              xv.w += v[4 * e + 3];
              v[4 * e] = xv.x;
              v[4 * e + 1] = xv.y;
              v[4 * e + 2] = xv.z;
              v[4 * e + 3] = xv.w;
              o4[e] = xv;
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(v[e], v[e], ss);
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(v[e]);
          tmem_st32(acc + c, w);
        }
        const float r = rsqrtf(ss / (float)g.N + g.eps);
        float z = 0.f;
#pragma unroll 1
        for (int c = 0; c < g.N; c += 32) {
          float v[32];
          tmem_ld32(acc + c, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= r;
          if (valid && g.a_out) store_bf16x32((__nv_bfloat16*)g.a_out + row * g.lda_out + c, v);
          if (g.w_head) {
            const float4* w4 = reinterpret_cast<const float4*>(g.w_head + c);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 wv = w4[e];
              z = fmaf(v[4 * e], wv.x, z);
              z = fmaf(v[4 * e + 1], wv.y, z);
              z = fmaf(v[4 * e + 2], wv.z, z);
              z = fmaf(v[4 * e + 3], wv.w, z);
            }
          }
        }
        if (valid && g.w_head) g.z[row] = z;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------------------------------
// RMSNorm of a row-major [M][d] matrix (bf16 or fp32 in): one warp per row; writes the
// bf16 normalised rows and, optionally, the fp32 copy of the input (the residual stream).
// ------------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256) k_rmsnorm(long long M, int d, const Tin* __restrict__ x,
                                                 long long ldx, float* __restrict__ x_out,
                                                 long long ldxo, __nv_bfloat16* __restrict__ a_out,
                                                 long long lda, float eps) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  constexpr int kVec = Elem<Tin>::kPerVec;  // elements per 16-byte load
  const Tin* xr = x + row * ldx;
  float ss = 0.f;
  for (int c = lane * kVec; c < d; c += 32 * kVec) {
    float f[kVec];
    Elem<Tin>::unpack(*reinterpret_cast<const uint4*>(xr + c), f);
#pragma unroll
    for (int e = 0; e < kVec; ++e) ss = fmaf(f[e], f[e], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)d + eps);
  for (int c = lane * kVec; c < d; c += 32 * kVec) {
    float f[kVec];
    Elem<Tin>::unpack(*reinterpret_cast<const uint4*>(xr + c), f);
    if (x_out) {
#pragma unroll
      for (int e = 0; e < kVec; e += 4)
        *reinterpret_cast<float4*>(x_out + row * ldxo + c + e) =
            make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
    }
#pragma unroll
    for (int e = 0; e < kVec; e += 2)
      *reinterpret_cast<uint32_t*>(a_out + row * lda + c + e) = pack_bf16(f[e] * r, f[e + 1] * r);
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [rows][K] bf16 with row stride ld elements; box 64 x box_rows, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, long long rows, int K, long long ld,
                     int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static DeviceOnce gemm_smem_attr[3];

template <int kEpi>
static int launch_t(const GemmArgs& g, cudaStream_t st) {
  using C = Cfg<kEpi>;
  Params p;
  if (!make_map(&p.ta, g.a, g.M, g.K, g.lda, BM) || !make_map(&p.tb, g.w, g.N, g.K, g.ldw, 256))
    return GENRANK_ERR_CUDA;
  p.g = g;
  if (!set_smem_limit_once(gemm_smem_attr[kEpi], (const void*)k_gemm_tc<kEpi>, (int)C::kSmem))
    return GENRANK_ERR_CUDA;
  const int sms = sm_count_current();
  if (sms <= 0) return GENRANK_ERR_CUDA;
  const long long tiles = (long long)((g.M + BM - 1) / BM) * (g.N / C::BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  k_gemm_tc<kEpi><<<grid, kThreads, C::kSmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace tg

int launch_gemm_tc(const GemmArgs& g, cudaStream_t st) {
  using namespace tg;
  if (g.M == 0) return GENRANK_OK;
  switch (g.epilogue) {
    case kEpiStore: return launch_t<kEpiStore>(g, st);
    case kEpiSilu: return launch_t<kEpiSilu>(g, st);
    case kEpiResRms: return launch_t<kEpiResRms>(g, st);
    default: return GENRANK_ERR_INVALID_ARG;
  }
}

int launch_rmsnorm(long long M, int d, const void* x, long long ldx, int x_dtype, float* x_out,
                   long long ldxo, void* a_out, long long lda, float eps, cudaStream_t st) {
  if (M == 0) return GENRANK_OK;
  const unsigned blocks = (unsigned)((M + 7) / 8);
  if (x_dtype == GENRANK_BF16)
    tg::k_rmsnorm<__nv_bfloat16><<<blocks, 256, 0, st>>>(M, d, (const __nv_bfloat16*)x, ldx,
                                                         x_out, ldxo, (__nv_bfloat16*)a_out,
                                                         lda, eps);
  else
    tg::k_rmsnorm<float><<<blocks, 256, 0, st>>>(M, d, (const float*)x, ldx, x_out, ldxo,
                                                 (__nv_bfloat16*)a_out, lda, eps);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace gr
