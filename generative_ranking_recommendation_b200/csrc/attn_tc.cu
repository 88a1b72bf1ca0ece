// Jagged masked ALiBi attention forward on 5th-generation tensor cores (sm_100a).
//
// Semantics ("GenRank [2025]" chapter notes, §1.4.1 candidate mask and §1.4.2
// ALiBi score; fun-rec "The Overall Generative Ranking Paradigm" §7.2.2):
//   s_ij = scale q_i.k_j - m_h |p_i - p_j| - m_t,h |t_i - t_j|, history rows causal,
//   candidate rows see all history and themselves.
//
// Design (bf16 inputs, head dim 64, fp32 accumulation):
//   * Work items are (user, 128-row query tile, head).  A one-block scheduling
//     kernel lists the (user, tile) pairs sorted by the number of 128-key tiles
//     they visit (longest first); a persistent grid of one CTA per SM walks the
//     list round-robin.  Key tiles a query tile never sees are never visited:
//     history tile t visits key tiles 0..t, candidate rows visit the history only.
//   * Warp 4 loads Q, K, V tiles with TMA (128B swizzle, no multicast) into a
//     two-stage ring and writes the per-key bias column for the stage.
//   * Warp 5 issues tcgen05.mma: S = Q K^T (128x128, fp32 in TMEM, two buffers)
//     and O_part = P V (128x64, fp32 in TMEM, two buffers).
//   * Warps 0-3 (one thread per query row, one TMEM lane each) run the online
//     softmax on S, write P in bf16 to shared memory in the UMMA K-major
//     swizzled layout, and fold each O_part into a register-resident O.
//   * On visible pairs p_i >= p_j and t_i >= t_j, so the bias splits into a row
//     term that cancels in the softmax and a column term c_j = m p_j + m_t (t_j - t_0);
//     only c_j is added per element.  The literal LSE is recovered in the epilogue.
//   * A candidate's own key lies outside the tiles it visits; its score (bias 0)
//     is merged into the softmax state in the epilogue on CUDA cores.
//   * Masks are evaluated only on tiles that straddle a row's last visible key.
// Every mbarrier wait is bounded in time; a timeout sets GENRANK_DERR_TIMEOUT,
// every role drains out of its loop and the CTA frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace gr {
namespace tc {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int DH = 64;   // head dim
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = BM * DH * 2;  // one Q, K or V tile (16 KB)
constexpr uint32_t kPBytes = BM * BN * 2;     // one P tile (32 KB)

// dynamic shared memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                          // 2 x 16 KB
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;     // 2 x 16 KB
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;     // 2 x 16 KB
constexpr uint32_t kOffP = kOffV + 2 * kTileBytes;     // 2 x 32 KB
constexpr uint32_t kOffCB = kOffP + 2 * kPBytes;       // 2 x 128 floats
constexpr uint32_t kOffBar = kOffCB + 2 * BN * 4;      // barriers
constexpr uint32_t kNumBars = 18;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S buffers at 0 and 128
constexpr uint32_t kColO = 256;  // O_part buffers at 256 and 320

constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, 0, 0);   // Q K-major, K K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, DH, 0, 1);  // P K-major, V MN-major

constexpr int kItemTileBits = 10;  // item = (user << 10) | query tile

struct Params {
  CUtensorMap tq, tk, tv;
  AttnArgs a;
  const int32_t* items;  // [count] sorted (user, tile) pairs
  const int32_t* count;
};

enum Bar {
  kQFull = 0, kQEmpty = 2, kKFull = 4, kVFull = 6, kKVEmpty = 8, kCBFull = 10, kSFull = 12,
  kPFull = 14, kPVFull = 16
};

struct Item {
  long long s;  // first token of the user
  int L, n;     // tokens, history tokens
  int q0;       // first query row (local)
  int nk;       // key tiles visited
  int h;
  bool ok;
};

GR_DEVICE Item load_item(const Params& P, int w) {
  const AttnArgs& a = P.a;
  Item it;
  const int pair = w / a.H;
  it.h = w - pair * a.H;
  const int rec = P.items[pair];
  const int u = rec >> kItemTileBits;
  const int t = rec & ((1 << kItemTileBits) - 1);
  it.s = a.off[u];
  const long long e = a.off[u + 1];
  it.ok = !(it.s < 0 || e < it.s || e > a.T);
  it.L = it.ok ? (int)(e - it.s) : 0;
  it.n = max(0, min(a.hist_len[u], it.L));
  it.q0 = t * BM;
  const int kmax = min(it.q0 + BM, it.n);  // keys [0, kmax) are visited
  it.nk = (it.ok && kmax > 0) ? (kmax + BN - 1) / BN : 0;
  return it;
}

// ------------------------------------------------------------------------------------------
// scheduling: (user, query tile) pairs sorted by visited key tiles, longest first
// ------------------------------------------------------------------------------------------
constexpr int kMaxNkBuckets = 257;

__global__ void __launch_bounds__(1024) k_schedule(int B, long long T, const int32_t* off,
                                                   const int32_t* hist_len, int max_tiles,
                                                   int32_t* items, int32_t* count,
                                                   int32_t* err) {
  __shared__ int hist[kMaxNkBuckets];
  __shared__ int cursor[kMaxNkBuckets];
  for (int i = threadIdx.x; i < kMaxNkBuckets; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  // pass 1: histogram of visited key tiles
  for (int u = threadIdx.x; u < B; u += blockDim.x) {
    const long long s = off[u], e = off[u + 1];
    if (s < 0 || e < s || e > T) {
      flag(err, GENRANK_DERR_LAYOUT);
      continue;
    }
    const int L = (int)(e - s);
    const int n = max(0, min(hist_len[u], L));
    const int tiles = min((L + BM - 1) / BM, max_tiles);
    if ((L + BM - 1) / BM > max_tiles) flag(err, GENRANK_DERR_LAYOUT);
    for (int t = 0; t < tiles; ++t) {
      const int kmax = min(t * BM + BM, n);
      const int nk = min(kmax > 0 ? (kmax + BN - 1) / BN : 0, kMaxNkBuckets - 1);
      atomicAdd(&hist[nk], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int b = kMaxNkBuckets - 1; b >= 0; --b) {
      cursor[b] = acc;
      acc += hist[b];
    }
    *count = acc;
  }
  __syncthreads();
  // pass 2: scatter
  for (int u = threadIdx.x; u < B; u += blockDim.x) {
    const long long s = off[u], e = off[u + 1];
    if (s < 0 || e < s || e > T) continue;
    const int L = (int)(e - s);
    const int n = max(0, min(hist_len[u], L));
    const int tiles = min((L + BM - 1) / BM, max_tiles);
    for (int t = 0; t < tiles; ++t) {
      const int kmax = min(t * BM + BM, n);
      const int nk = min(kmax > 0 ? (kmax + BN - 1) / BN : 0, kMaxNkBuckets - 1);
      const int slot = atomicAdd(&cursor[nk], 1);
      items[slot] = (u << kItemTileBits) | t;
    }
  }
}

// ------------------------------------------------------------------------------------------
// the attention kernel
// ------------------------------------------------------------------------------------------
GR_DEVICE uint32_t parity(int fill) { return (uint32_t)(fill & 1); }

// Every lane waits (bounded), then the warp agrees, so that the warp stays
// converged for the .sync.aligned tcgen05 instructions that follow.
GR_DEVICE bool wait_warp(uint64_t* bar, uint32_t par, volatile int* abort_flag, int32_t* err) {
  const bool ok = mbar_wait(bar, par, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1) k_attn_fwd_tc(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnArgs& a = P.a;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* sCB = reinterpret_cast<float*>(smem + kOffCB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kQFull + i], 1);
      mbar_init(&bars[kQEmpty + i], 1);
      mbar_init(&bars[kKFull + i], 1);
      mbar_init(&bars[kVFull + i], 1);
      mbar_init(&bars[kKVEmpty + i], 1);
      mbar_init(&bars[kCBFull + i], 32);
      mbar_init(&bars[kSFull + i], 1);
      mbar_init(&bars[kPFull + i], 128);
      mbar_init(&bars[kPVFull + i], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&P.tq);
    tma_prefetch_desc(&P.tk);
    tma_prefetch_desc(&P.tv);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = *P.count * a.H;

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA producer
    int qi = 0, g = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Item it = load_item(P, w);
      if (it.nk == 0) continue;
      const int qb = qi & 1;
      if (!wait_warp(&bars[kQEmpty + qb], parity(qi >> 1) ^ 1u, abort_flag, a.err)) break;
      if (lane == 0) {
        mbar_expect_tx(&bars[kQFull + qb], kTileBytes);
        tma_load_3d(smem + kOffQ + qb * kTileBytes, &P.tq, &bars[kQFull + qb], 0, it.h,
                    (int)(it.s + it.q0));
      }
      const float spos = a.slope_pos[it.h] * kLog2e, stime = a.slope_time[it.h] * kLog2e;
      const long long t0 = a.ts[it.s];
      bool ok = true;
      for (int j = 0; j < it.nk; ++j, ++g) {
        const int st = g & 1;
        if (!wait_warp(&bars[kKVEmpty + st], parity(g >> 1) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        const int kv0 = j * BN;
        if (lane == 0) {
          mbar_expect_tx(&bars[kKFull + st], kTileBytes);
          tma_load_3d(smem + kOffK + st * kTileBytes, &P.tk, &bars[kKFull + st], 0, it.h,
                      (int)(it.s + kv0));
          mbar_expect_tx(&bars[kVFull + st], kTileBytes);
          tma_load_3d(smem + kOffV + st * kTileBytes, &P.tv, &bars[kVFull + st], 0, it.h,
                      (int)(it.s + kv0));
        }
        // bias column of this key tile, in log2 units: c_j = log2e (m p_j + m_t (t_j - t_0))
        for (int c = lane; c < BN; c += 32) {
          const int key = kv0 + c;
          float cb = 0.f;
          if (key < it.n) {
            const long long tk = a.ts[it.s + key];
            cb = spos * (float)a.pos[it.s + key] + stime * (float)(tk - t0);
          }
          sCB[st * BN + c] = cb;
        }
        mbar_arrive(&bars[kCBFull + st]);
      }
      if (!ok) break;
      ++qi;
    }
  } else if (warp == 5 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer (one thread)
    int qi = 0, g = 0;
    const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK),
                   sV = smem_u32(smem + kOffV), sPb = smem_u32(smem + kOffP);
    for (int w = blockIdx.x; w < total && !*abort_flag; w += gridDim.x) {
      const Item it = load_item(P, w);
      if (it.nk == 0) continue;
      const int qb = qi & 1;
      if (!mbar_wait(&bars[kQFull + qb], parity(qi >> 1), abort_flag, a.err)) break;
      tc_fence_after();
      bool ok = true;
      auto issue_s = [&](int gg) -> bool {
        const int st = gg & 1;
        if (!mbar_wait(&bars[kKFull + st], parity(gg >> 1), abort_flag, a.err)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kColS + (uint32_t)(gg & 1) * BN;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(sQ + qb * kTileBytes + k * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + st * kTileBytes + k * 32, 16, 1024);
          mma_bf16_ss(d, ad, bd, kIdescS, k > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kSFull + (gg & 1)]);
        return true;
      };
      if (!issue_s(g)) break;
      for (int j = 0; j < it.nk; ++j) {
        const int gj = g + j;
        if (j + 1 < it.nk && !issue_s(gj + 1)) {
          ok = false;
          break;
        }
        const int b = gj & 1;
        if (!mbar_wait(&bars[kPFull + b], parity(gj >> 1), abort_flag, a.err) ||
            !mbar_wait(&bars[kVFull + b], parity(gj >> 1), abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + kColO + (uint32_t)b * DH;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t ad =
              smem_desc_sw128(sPb + b * kPBytes + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sV + b * kTileBytes + k * 16 * 128, kTileBytes, 1024);
          mma_bf16_ss(d, ad, bd, kIdescPV, k > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kPVFull + b]);
        mma_commit(&bars[kKVEmpty + b]);
      }
      if (!ok) break;
      mma_commit(&bars[kQEmpty + qb]);
      g += it.nk;
      ++qi;
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint8_t* sPbase = smem + kOffP;
    const float scale_log2 = a.scale * kLog2e;
    int g = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      __syncwarp();
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Item it = load_item(P, w);
      if (!it.ok) continue;
      const int i = it.q0 + r;
      const bool row = i < it.L;
      const int lim = min(i, it.n - 1);
      const int mask_from = min(it.q0, it.n - 1);  // tiles with kv0 + 127 > this need masks
      float m = -INFINITY, l = 0.f, alpha_prev = 1.f;
      float o[DH];
#pragma unroll
      for (int c = 0; c < DH; ++c) o[c] = 0.f;
      bool ok = true;
      for (int j = 0; j < it.nk; ++j) {
        const int gj = g + j, b = gj & 1;
        const int kv0 = j * BN;
        if (!wait_warp(&bars[kCBFull + b], parity(gj >> 1), abort_flag, a.err) ||
            !wait_warp(&bars[kSFull + b], parity(gj >> 1), abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float x[BN];
        tmem_ld128(tmem + lane_base + kColS + b * BN, x);
        const float* cb = sCB + b * BN;
        float mx = -INFINITY;
        if (kv0 + BN - 1 > mask_from) {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const float v = fmaf(x[c], scale_log2, cb[c]);
            x[c] = (kv0 + c <= lim) ? v : -INFINITY;
            mx = fmaxf(mx, x[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            x[c] = fmaf(x[c], scale_log2, cb[c]);
            mx = fmaxf(mx, x[c]);
          }
        }
        const float m_new = fmaxf(m, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = ex2(m - m_use);
        float rs = 0.f;
        uint8_t* prow = sPbase + b * kPBytes + r * 128;
#pragma unroll
        for (int c16 = 0; c16 < BN / 8; ++c16) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2(x[c16 * 8 + e] - m_use);
            rs += p[e];
          }
          uint4 pk = make_uint4(pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]),
                                pack_bf16(p[4], p[5]), pack_bf16(p[6], p[7]));
          const int blk = c16 >> 3, cc = c16 & 7;
          *reinterpret_cast<uint4*>(prow + blk * (BM * 128) + ((cc ^ (r & 7)) << 4)) = pk;
        }
        l = l * alpha + rs;
        m = m_new;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[kPFull + b]);
        if (j >= 1) {
          const int pb = (gj - 1) & 1;
          if (!wait_warp(&bars[kPVFull + pb], parity((gj - 1) >> 1), abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          float t[DH];
          tmem_ld64(tmem + lane_base + kColO + pb * DH, t);
#pragma unroll
          for (int e = 0; e < DH; ++e) o[e] = fmaf(o[e], alpha_prev, t[e]);
          tc_fence_before();
        }
        alpha_prev = alpha;
      }
      if (!ok) break;
      if (it.nk > 0) {
        const int gl = g + it.nk - 1, pb = gl & 1;
        if (!wait_warp(&bars[kPVFull + pb], parity(gl >> 1), abort_flag, a.err)) break;
        tc_fence_after();
        float t[DH];
        tmem_ld64(tmem + lane_base + kColO + pb * DH, t);
#pragma unroll
        for (int e = 0; e < DH; ++e) o[e] = fmaf(o[e], alpha_prev, t[e]);
        tc_fence_before();
      }
      g += it.nk;
      if (!row) continue;
      const long long tok = it.s + i;
      const float spos = a.slope_pos[it.h], stime = a.slope_time[it.h];
      const long long t0 = a.ts[it.s];
      const float rowterm = spos * (float)a.pos[tok] + stime * (float)(a.ts[tok] - t0);
      if (i >= it.n) {
        // the candidate's own key: literal bias 0, i.e. column term == row term
        const __nv_bfloat16* qp = (const __nv_bfloat16*)a.q + tok * a.tok_stride + it.h * DH;
        const __nv_bfloat16* kp = (const __nv_bfloat16*)a.k + tok * a.tok_stride + it.h * DH;
        const __nv_bfloat16* vp = (const __nv_bfloat16*)a.v + tok * a.tok_stride + it.h * DH;
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < DH; c += 8) {
          const uint4 qa = *reinterpret_cast<const uint4*>(qp + c);
          const uint4 ka = *reinterpret_cast<const uint4*>(kp + c);
          float qf[8], kf[8];
          Elem<__nv_bfloat16>::unpack(qa, qf);
          Elem<__nv_bfloat16>::unpack(ka, kf);
#pragma unroll
          for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
        }
        const float xs = fmaf(dot, scale_log2, rowterm * kLog2e);
        const float m_new = fmaxf(m, xs);
        const float al = ex2(m - m_new), p = ex2(xs - m_new);
        l = l * al + p;
#pragma unroll
        for (int c = 0; c < DH; c += 8) {
          const uint4 va = *reinterpret_cast<const uint4*>(vp + c);
          float vf[8];
          Elem<__nv_bfloat16>::unpack(va, vf);
#pragma unroll
          for (int e = 0; e < 8; ++e) o[c + e] = fmaf(o[c + e], al, p * vf[e]);
        }
        m = m_new;
      }
      const float inv = 1.f / l;
      uint4* op = reinterpret_cast<uint4*>((__nv_bfloat16*)a.o + tok * a.o_stride + it.h * DH);
#pragma unroll
      for (int c = 0; c < DH; c += 8) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = o[c + e] * inv;
        op[c / 8] = Elem<__nv_bfloat16>::pack(f);
      }
      if (a.lse) a.lse[(long long)it.h * a.T + tok] = (m + __log2f(l)) * kLn2 - rowterm;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
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

// [T] rows of H heads x 64 bf16; box = one head x 128 rows, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, long long T, int H, long long tok_stride) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)DH * 2, (cuuint64_t)tok_stride * 2};
  cuuint32_t box[3] = {(cuuint32_t)DH, 1, (cuuint32_t)BM};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int max_tiles_of(int max_seqlen) { return (max_seqlen + BM - 1) / BM; }

}  // namespace tc

size_t attn_fwd_tc_workspace(int B, long long T, int H, int max_seqlen) {
  (void)T;
  (void)H;
  return 256 + (size_t)B * tc::max_tiles_of(max_seqlen) * sizeof(int32_t);
}

int launch_attn_fwd_tc(const AttnArgs& a, cudaStream_t st) {
  using namespace tc;
  if (a.dh != DH || a.dtype != GENRANK_BF16) return GENRANK_ERR_UNSUPPORTED;
  const int max_tiles = max_tiles_of(a.max_seqlen);
  if (max_tiles >= (1 << kItemTileBits) || a.B >= (1 << (31 - kItemTileBits)))
    return GENRANK_ERR_UNSUPPORTED;
  if (a.T > INT32_MAX - 2 * BM) return GENRANK_ERR_UNSUPPORTED;
  Params p;
  if (!make_map(&p.tq, a.q, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tk, a.k, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tv, a.v, a.T, a.H, a.tok_stride))
    return GENRANK_ERR_CUDA;
  p.a = a;
  int32_t* ws = (int32_t*)a.ws;
  p.count = ws;
  p.items = ws + 64;
  k_schedule<<<1, 1024, 0, st>>>(a.B, a.T, a.off, a.hist_len, max_tiles, ws + 64, ws, a.err);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
      return GENRANK_ERR_CUDA;
    attr = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  k_attn_fwd_tc<<<sms, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace gr
