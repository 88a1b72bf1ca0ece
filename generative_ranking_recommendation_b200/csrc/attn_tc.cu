// Jagged masked ALiBi attention forward on 5th-generation tensor cores (sm_100a).
//
// Semantics ("GenRank [2025]" chapter notes, §1.4.1 candidate mask and §1.4.2
// ALiBi score; fun-rec "The Overall Generative Ranking Paradigm" §7.2.2):
//   s_ij = scale q_i.k_j - m_h |p_i - p_j| - m_t,h |t_i - t_j|, history rows causal,
//   candidate rows see all history and themselves.
//
// Design (bf16 inputs, head dim 64, fp32 accumulation):
//   * A prologue kernel lists (user, 128-row query tile) work records sorted by the
//     number of 128-key tiles they visit (longest first), and writes the ALiBi
//     column term c_j = log2(e) (m_h p_j + m_t,h (t_j - t_0)) for every token and
//     head into a 16-byte aligned scratch layout.  On visible pairs p_i >= p_j and
//     t_i >= t_j, so the bias is c_j - c_i; c_i cancels in the softmax and only c_j
//     is added per element; the literal LSE subtracts c_i in the epilogue.
//   * Persistent grid, two CTAs per SM; each CTA walks the records round-robin
//     (one head per work item).  Key tiles a query tile never sees are never
//     visited: history tile t visits key tiles 0..t, candidate rows the history only.
//   * Warp 4 issues TMA loads (Q; K, V two-stage ring; 128B swizzle, no multicast)
//     and a bulk copy of the key tile's column terms.
//   * Warp 5 (one thread) issues tcgen05.mma: S = Q K^T (128 x 128, fp32 in TMEM)
//     from shared memory, then O += P V (128 x 64, fp32 in TMEM) with P read from
//     tensor memory, where the softmax left it in place of S (bf16 pairs).
//   * Warps 0-3 (one query row per thread, one TMEM lane each) load S, add the
//     column term, mask only tiles that straddle a row's last visible key, and run
//     the online softmax with a lazily updated offset: O in TMEM is rescaled only
//     when a row's maximum grows by more than 2^8, so most tiles touch O not at all.
//   * The other CTA on the SM hides each CTA's per-item latencies (work-record
//     loads, the epilogue's global loads and stores).
//   * A candidate's own key lies outside the tiles it visits; its score (bias 0)
//     is merged into the softmax state in the epilogue on CUDA cores.
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
constexpr int kThreads = 192;  // warps 0-3 softmax, warp 4 TMA, warp 5 MMA
constexpr uint32_t kTileBytes = BM * DH * 2;  // one Q, K or V tile (16 KB)
constexpr uint32_t kCBBytes = BN * 4;         // column terms of one key tile
constexpr float kOverflowSum = 1.2676506e30f;   // 2^100: a tile's row sum above this is redone
constexpr float kUnderflowSum = 7.8886091e-31f;  // 2^-100: a first tile's row sum below this too

// dynamic shared memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                          // 16 KB
constexpr uint32_t kOffK = kOffQ + kTileBytes;         // 2 x 16 KB
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;     // 2 x 16 KB
constexpr uint32_t kOffCB = kOffV + 2 * kTileBytes;    // 2 x 512 B
constexpr uint32_t kOffBar = kOffCB + 2 * kCBBytes;    // barriers
constexpr uint32_t kNumBars = 12;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack

// TMEM columns (per CTA; two CTAs share an SM's 512)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;    // S (fp32, 128 columns)
constexpr uint32_t kColO = 128;  // O (fp32, 64 columns)
constexpr uint32_t kColP = 192;  // P (bf16 pairs, 64 columns)

constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, 0, 0);   // Q K-major, K K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, DH, 0, 1);  // P K-major (TMEM), V MN-major

// scratch layout
constexpr size_t kHeaderBytes = 256;
constexpr int kRecInts = 8;  // s, L, n, q0, nk, spad, u, unused

struct Params {
  CUtensorMap tq, tk, tv;
  AttnArgs a;
  const int4* recs;      // [count][2] work records
  const int32_t* count;  // number of records
  const float* cbias;    // [H][Tp] column terms (log2 units)
  long long Tp;
};

enum Bar { kQFull = 0, kQEmpty = 1, kKFull = 2, kVFull = 4, kKVEmpty = 6, kSFull = 8,
           kPFull = 9, kPVFull = 10 };

struct Item {
  int s, L, n, q0, nk, spad, h;
};

GR_DEVICE Item load_item(const Params& P, int w) {
  const int pair = w / P.a.H;
  const int4 r0 = P.recs[2 * pair];
  const int4 r1 = P.recs[2 * pair + 1];
  Item it;
  it.h = w - pair * P.a.H;
  it.s = r0.x;
  it.L = r0.y;
  it.n = r0.z;
  it.q0 = r0.w;
  it.nk = r1.x;
  it.spad = r1.y;
  return it;
}

// Start of user u's segment in the column-term scratch: 16-byte aligned and
// disjoint from the previous user's (4 ceil(s/4) + 4u grows by at least L + 1).
__host__ __device__ inline long long seg_start(long long s, int u) {
  return 4 * ((s + 3) / 4) + 4LL * u;
}
__host__ __device__ inline long long scratch_tp(long long T, int B) {
  return ((T + 4LL * B + 4 + BN) + 3) / 4 * 4;
}

// ------------------------------------------------------------------------------------------
// prologue: work records (block B) and column terms (blocks 0..B-1)
// ------------------------------------------------------------------------------------------
constexpr int kMaxNkBuckets = 257;

__global__ void __launch_bounds__(256) k_prologue(const __grid_constant__ AttnArgs a,
                                                  int max_tiles, int4* recs, int32_t* count,
                                                  float* cbias, long long Tp) {
  const int b = blockIdx.x;
  if (b < a.B) {
    const long long s = a.off[b], e = a.off[b + 1];
    if (s < 0 || e < s || e > a.T) return;  // flagged by the schedule block
    const int L = (int)(e - s);
    const long long base = seg_start(s, b);
    const long long t0 = L > 0 ? a.ts[s] : 0;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
      const float p = (float)a.pos[s + i];
      const float dt = (float)(a.ts[s + i] - t0);
      for (int h = 0; h < a.H; ++h)
        cbias[(long long)h * Tp + base + i] = kLog2e * (a.slope_pos[h] * p + a.slope_time[h] * dt);
    }
    return;
  }
  // schedule: histogram of visited key tiles, then a scatter longest first
  __shared__ int hist[kMaxNkBuckets];
  __shared__ int cursor[kMaxNkBuckets];
  for (int i = threadIdx.x; i < kMaxNkBuckets; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int pass = 0; pass < 2; ++pass) {
    for (int u = threadIdx.x; u < a.B; u += blockDim.x) {
      const long long s = a.off[u], e = a.off[u + 1];
      if (s < 0 || e < s || e > a.T) {
        if (pass == 0) flag(a.err, GENRANK_DERR_LAYOUT);
        continue;
      }
      const int L = (int)(e - s);
      const int n = max(0, min(a.hist_len[u], L));
      const int tiles_all = (L + BM - 1) / BM;
      if (pass == 0 && tiles_all > max_tiles) flag(a.err, GENRANK_DERR_LAYOUT);
      const int tiles = min(tiles_all, max_tiles);
      for (int t = 0; t < tiles; ++t) {
        const int kmax = min(t * BM + BM, n);
        const int nk = kmax > 0 ? (kmax + BN - 1) / BN : 0;
        const int bucket = min(nk, kMaxNkBuckets - 1);
        if (pass == 0) {
          atomicAdd(&hist[bucket], 1);
        } else {
          const int slot = atomicAdd(&cursor[bucket], 1);
          recs[2 * slot] = make_int4((int)s, L, n, t * BM);
          recs[2 * slot + 1] = make_int4(nk, (int)seg_start(s, u), u, 0);
        }
      }
    }
    __syncthreads();
    if (pass == 0 && threadIdx.x == 0) {
      int acc = 0;
      for (int q = kMaxNkBuckets - 1; q >= 0; --q) {
        cursor[q] = acc;
        acc += hist[q];
      }
      *count = acc;
    }
    __syncthreads();
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

// x = s * scale + c_j for 32 columns starting at key c0 of the tile; columns at or
// beyond nvalid are masked.  Four independent running maxima shorten the chain.
template <bool kMasked>
GR_DEVICE void row_max_chunk(const uint32_t (&s)[32], const float* cb, int c0, int nvalid,
                             float scale_log2, float (&mx4)[4]) {
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    const float4 b4 = *reinterpret_cast<const float4*>(cb + c);
    const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = fmaf(__uint_as_float(s[c + e]), scale_log2, bb[e]);
      mx4[e] = fmaxf(mx4[e], (!kMasked || c0 + c + e < nvalid) ? v : -INFINITY);
    }
  }
}

// p = 2^(x - m) for 32 columns, summed into four partial row sums, packed to bf16
// pairs and stored to 16 TMEM columns at taddr.
template <bool kMasked>
GR_DEVICE void exp_pack_store(const uint32_t (&s)[32], const float* cb, int c0, int nvalid,
                              float scale_log2, float m_use, float (&rs4)[4], uint32_t taddr) {
  uint32_t pk[16];
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    const float4 b4 = *reinterpret_cast<const float4*>(cb + c);
    const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = fmaf(__uint_as_float(s[c + e]), scale_log2, bb[e] - m_use);
      p[e] = (!kMasked || c0 + c + e < nvalid) ? ex2(v) : 0.f;
      rs4[e] += p[e];
    }
    pk[c / 2] = pack_bf16(p[0], p[1]);
    pk[c / 2 + 1] = pack_bf16(p[2], p[3]);
  }
  tmem_st16(taddr, pk);
}

// Row maximum of x = s * scale + c_j over the tile, 32 columns at a time with the
// next chunk's TMEM load in flight.
template <bool kMasked>
GR_DEVICE float tile_max(uint32_t tmem_lane, const float* cb, int nvalid, float scale_log2) {
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  uint32_t xa[32], xb[32];
  tmem_ld32_async(tmem_lane + kColS, xa);
  tmem_ld_wait(xa);
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 64) {
    tmem_ld32_async(tmem_lane + kColS + c0 + 32, xb);
    row_max_chunk<kMasked>(xa, cb + c0, c0, nvalid, scale_log2, mx4);
    tmem_ld_wait(xb);
    if (c0 + 64 < BN) tmem_ld32_async(tmem_lane + kColS + c0 + 64, xa);
    row_max_chunk<kMasked>(xb, cb + c0 + 32, c0 + 32, nvalid, scale_log2, mx4);
    if (c0 + 64 < BN) tmem_ld_wait(xa);
  }
  return fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
}

// P = 2^(x - m) for the tile, written as bf16 pairs to the P columns, 32 keys at a
// time with the next chunk's TMEM load in flight.  Returns the row sum.
template <bool kMasked>
GR_DEVICE float tile_exp(uint32_t tmem_lane, const float* cb, int nvalid, float scale_log2,
                         float m) {
  float rs4[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t xa[32], xb[32];
  tmem_ld32_async(tmem_lane + kColS, xa);
  tmem_ld_wait(xa);
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 64) {
    tmem_ld32_async(tmem_lane + kColS + c0 + 32, xb);
    exp_pack_store<kMasked>(xa, cb + c0, c0, nvalid, scale_log2, m, rs4,
                            tmem_lane + kColP + c0 / 2);
    tmem_ld_wait(xb);
    if (c0 + 64 < BN) tmem_ld32_async(tmem_lane + kColS + c0 + 64, xa);
    exp_pack_store<kMasked>(xb, cb + c0 + 32, c0 + 32, nvalid, scale_log2, m, rs4,
                            tmem_lane + kColP + (c0 + 32) / 2);
    if (c0 + 64 < BN) tmem_ld_wait(xa);
  }
  return (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
}

// One key tile of the online softmax for this thread's row (TMEM lane).  The offset
// m starts at the row's own column term c_i: every visible key has c_j <= c_i, so
// 2^(x - m) <= 2^(scale q.k log2 e), which overflows only for extreme scores.  Each
// tile is one pass; a tile whose row sum leaves [2^-100, 2^100] on the first tile
// (every key far below the offset) or exceeds 2^100 later is redone with the exact
// offset max(m, tile max), rescaling O in TMEM.  Before P is written, the previous
// P V must have finished (it reads P and adds to O).
template <bool kMasked>
GR_DEVICE bool softmax_tile(uint32_t tmem_lane, const float* cb, int nvalid, float scale_log2,
                            bool first, float& m, float& l, uint64_t* pv_bar, int g,
                            volatile int* abort_flag, int32_t* err) {
  if (g > 0 && !wait_warp(pv_bar, parity(g - 1), abort_flag, err)) return false;
  tc_fence_after();
  float rs = tile_exp<kMasked>(tmem_lane, cb, nvalid, scale_log2, m);
  const bool redo = !(rs <= kOverflowSum) || (first && rs < kUnderflowSum);
  if (__any_sync(0xffffffffu, redo)) {
    // every lane takes part in the .sync.aligned TMEM loads; only redo lanes move m
    const float mx = tile_max<kMasked>(tmem_lane, cb, nvalid, scale_log2);
    const float m_new = redo ? (first ? mx : fmaxf(m, mx)) : m;
    const float alpha = first ? 1.f : ex2(m - m_new);
    m = m_new;
    if (!first) {
#pragma unroll 1
      for (int c0 = 0; c0 < DH; c0 += 32) {
        float o[32];
        tmem_ld32(tmem_lane + kColO + c0, o);
        uint32_t ob[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) ob[c] = __float_as_uint(o[c] * alpha);
        tmem_st32(tmem_lane + kColO + c0, ob);
      }
    }
    l *= alpha;
    rs = tile_exp<kMasked>(tmem_lane, cb, nvalid, scale_log2, m);
  }
  l = first ? rs : l + rs;
  return true;
}

__global__ void __launch_bounds__(kThreads, 2) k_attn_fwd_tc(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnArgs& a = P.a;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  const float* sCB = reinterpret_cast<const float*>(smem + kOffCB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    mbar_init(&bars[kQEmpty], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kKFull + i], 1);
      mbar_init(&bars[kVFull + i], 1);
      mbar_init(&bars[kKVEmpty + i], 1);
    }
    mbar_init(&bars[kSFull], 1);
    mbar_init(&bars[kPFull], 128);
    mbar_init(&bars[kPVFull], 1);
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
      if (!wait_warp(&bars[kQEmpty], parity(qi) ^ 1u, abort_flag, a.err)) break;
      if (lane == 0) {
        mbar_expect_tx(&bars[kQFull], kTileBytes);
        tma_load_3d(smem + kOffQ, &P.tq, &bars[kQFull], 0, it.h, it.s + it.q0);
      }
      const float* cb_src = P.cbias + (long long)it.h * P.Tp + it.spad;
      bool ok = true;
      for (int j = 0; j < it.nk; ++j, ++g) {
        const int st = g & 1;
        if (!wait_warp(&bars[kKVEmpty + st], parity(g >> 1) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const int kv0 = (it.nk - 1 - j) * BN;  // most recent keys first
          mbar_expect_tx(&bars[kKFull + st], kTileBytes + kCBBytes);
          tma_load_3d(smem + kOffK + st * kTileBytes, &P.tk, &bars[kKFull + st], 0, it.h,
                      it.s + kv0);
          bulk_load(smem + kOffCB + st * kCBBytes, cb_src + kv0, kCBBytes, &bars[kKFull + st]);
          mbar_expect_tx(&bars[kVFull + st], kTileBytes);
          tma_load_3d(smem + kOffV + st * kTileBytes, &P.tv, &bars[kVFull + st], 0, it.h,
                      it.s + kv0);
        }
      }
      if (!ok) break;
      ++qi;
    }
  } else if (warp == 5 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer (one thread)
    // Per tile g: S_g = Q K_g^T is issued as soon as the softmax has released S_{g-1}
    // (P lives in its own columns), so it overlaps P_{g-1} V_{g-1}.
    const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK),
                   sV = smem_u32(smem + kOffV);
    auto next_item = [&](int from, Item& out) -> int {
      for (int x = from; x < total; x += gridDim.x) {
        out = load_item(P, x);
        if (out.nk > 0) return x;
      }
      return -1;
    };
    auto issue_s = [&](int gg) {
      const int st = gg & 1;
#pragma unroll
      for (int k = 0; k < DH / 16; ++k) {
        const uint64_t ad = smem_desc_sw128(sQ + k * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(sK + st * kTileBytes + k * 32, 16, 1024);
        mma_bf16_ss(tmem + kColS, ad, bd, kIdescS, k > 0 ? 1u : 0u);
      }
      mma_commit(&bars[kSFull]);
    };
    Item it;
    int w = next_item(blockIdx.x, it);
    // the record after the current item, loaded one item ahead of its use
    Item pre = (w >= 0 && w + (int)gridDim.x < total) ? load_item(P, w + gridDim.x) : Item{};
    int qi = 0, g = 0, j = 0;
    bool ok = w >= 0 && mbar_wait(&bars[kQFull], parity(0), abort_flag, a.err) &&
              mbar_wait(&bars[kKFull], parity(0), abort_flag, a.err);
    if (ok) {
      tc_fence_after();
      issue_s(0);
      if (it.nk == 1) mma_commit(&bars[kQEmpty]);
    }
    while (ok && !*abort_flag) {
      if (!mbar_wait(&bars[kPFull], parity(g), abort_flag, a.err)) break;
      // look ahead: the next tile of this item, or the first tile of the next item
      Item it2 = it;
      int w2 = w, j2 = j + 1;
      if (j2 == it.nk) {
        j2 = 0;
        w2 = w + gridDim.x;
        if (w2 >= total) {
          w2 = -1;
        } else if (pre.nk > 0) {
          it2 = pre;
        } else {
          w2 = next_item(w2 + gridDim.x, it2);  // rare: items without keys to visit
        }
        if (w2 >= 0 && w2 + (int)gridDim.x < total) pre = load_item(P, w2 + gridDim.x);
      }
      if (w2 >= 0) {
        if (j2 == 0 && !mbar_wait(&bars[kQFull], parity(qi + 1), abort_flag, a.err)) break;
        if (!mbar_wait(&bars[kKFull + ((g + 1) & 1)], parity((g + 1) >> 1), abort_flag, a.err))
          break;
        tc_fence_after();
        issue_s(g + 1);
        if (j2 == it2.nk - 1) mma_commit(&bars[kQEmpty]);
      }
      const int st = g & 1;
      if (!mbar_wait(&bars[kVFull + st], parity(g >> 1), abort_flag, a.err)) break;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < BN / 16; ++k) {
        const uint64_t bd = smem_desc_sw128(sV + st * kTileBytes + k * 16 * 128, kTileBytes, 1024);
        mma_bf16_ts(tmem + kColO, tmem + kColP + k * 8, bd, kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
      }
      mma_commit(&bars[kPVFull]);
      mma_commit(&bars[kKVEmpty + st]);
      ++g;
      if (w2 < 0) break;
      if (j2 == 0) ++qi;
      w = w2;
      j = j2;
      it = it2;
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float scale_log2 = a.scale * kLog2e;
    const __nv_bfloat16* Qg = (const __nv_bfloat16*)a.q;
    const __nv_bfloat16* Kg = (const __nv_bfloat16*)a.k;
    const __nv_bfloat16* Vg = (const __nv_bfloat16*)a.v;
    int g = 0;
    // the next work item's record is loaded one item ahead, and its candidate rows are
    // warmed in L2, so that an item starts without a dependent global-load chain
    Item nx = blockIdx.x < total ? load_item(P, blockIdx.x) : Item{};
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      __syncwarp();
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Item it = nx;
      if (w + (int)gridDim.x < total) nx = load_item(P, w + gridDim.x);
      const int i = it.q0 + r;
      const bool row = i < it.L;
      const long long tok = (long long)it.s + i;
      const bool cand = row && i >= it.n;
      const float rowcb = row ? P.cbias[(long long)it.h * P.Tp + it.spad + i] : 0.f;
      // candidate self-term: its score now, its value row kept packed until the epilogue
      float xs = -INFINITY;
      uint4 va[DH / 8];
      if (cand) {
        const uint4* qp = reinterpret_cast<const uint4*>(Qg + tok * a.tok_stride + it.h * DH);
        const uint4* kp = reinterpret_cast<const uint4*>(Kg + tok * a.tok_stride + it.h * DH);
        const uint4* vp = reinterpret_cast<const uint4*>(Vg + tok * a.tok_stride + it.h * DH);
        uint4 qa[DH / 8], ka[DH / 8];
#pragma unroll
        for (int c = 0; c < DH / 8; ++c) {
          qa[c] = qp[c];
          ka[c] = kp[c];
          va[c] = vp[c];
        }
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < DH / 8; ++c) {
          float qf[8], kf[8];
          Elem<__nv_bfloat16>::unpack(qa[c], qf);
          Elem<__nv_bfloat16>::unpack(ka[c], kf);
#pragma unroll
          for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
        }
        xs = fmaf(dot, scale_log2, rowcb);
      }
      const int lim = min(i, it.n - 1);
      const int mask_from = min(it.q0, it.n - 1);  // a tile needs masks if kv0 + 127 > this
      float m = rowcb, l = 0.f;
      bool ok = true;
      for (int j = 0; j < it.nk; ++j, ++g) {
        const int st = g & 1;
        const int kv0 = (it.nk - 1 - j) * BN;  // most recent keys first
        if (!wait_warp(&bars[kSFull], parity(g), abort_flag, a.err) ||
            !wait_warp(&bars[kKFull + st], parity(g >> 1), abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* cb = sCB + st * BN;
        const bool masked = kv0 + BN - 1 > mask_from;
        const int nvalid = masked ? max(0, min(BN, lim - kv0 + 1)) : BN;
        ok = masked ? softmax_tile<true>(tmem + lane_base, cb, nvalid, scale_log2, j == 0, m, l,
                                         &bars[kPVFull], g, abort_flag, a.err)
                    : softmax_tile<false>(tmem + lane_base, cb, nvalid, scale_log2, j == 0, m, l,
                                          &bars[kPVFull], g, abort_flag, a.err);
        if (!ok) break;
        tc_fence_before();
        mbar_arrive(&bars[kPFull]);
      }
      if (!ok) break;
      {  // warm L2 for the next item's candidate rows while this item's P V finishes
        const int ni = nx.q0 + r;
        if (w + (int)gridDim.x < total && ni < nx.L && ni >= nx.n) {
          const long long nt = (long long)nx.s + ni;
          prefetch_l2(Qg + nt * a.tok_stride + nx.h * DH);
          prefetch_l2(Kg + nt * a.tok_stride + nx.h * DH);
          prefetch_l2(Vg + nt * a.tok_stride + nx.h * DH);
        }
      }
      float o[DH];
      if (it.nk > 0) {
        if (!wait_warp(&bars[kPVFull], parity(g - 1), abort_flag, a.err)) break;
        tc_fence_after();
        tmem_ld64(tmem + lane_base + kColO, o);
        tc_fence_before();
      } else {
#pragma unroll
        for (int c = 0; c < DH; ++c) o[c] = 0.f;
        m = xs;  // nothing visible but the candidate itself
      }
      if (!row) continue;
      if (cand) {
        const float m_new = fmaxf(m, xs);
        const float al = ex2(m - m_new), p = ex2(xs - m_new);
        l = l * al + p;
#pragma unroll
        for (int c = 0; c < DH / 8; ++c) {
          float vf[8];
          Elem<__nv_bfloat16>::unpack(va[c], vf);
#pragma unroll
          for (int e = 0; e < 8; ++e) o[c * 8 + e] = fmaf(o[c * 8 + e], al, p * vf[e]);
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
      if (a.lse) a.lse[(long long)it.h * a.T + tok] = (m + __log2f(l) - rowcb) * kLn2;
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

static size_t recs_bytes(int B, int max_seqlen) {
  return ((size_t)B * max_tiles_of(max_seqlen) * kRecInts * 4 + 15) / 16 * 16;
}

}  // namespace tc

size_t attn_fwd_tc_workspace(int B, long long T, int H, int max_seqlen) {
  using namespace tc;
  return kHeaderBytes + recs_bytes(B, max_seqlen) + (size_t)H * scratch_tp(T, B) * sizeof(float);
}

int launch_attn_fwd_tc(const AttnArgs& a, cudaStream_t st) {
  using namespace tc;
  if (a.dh != DH || a.dtype != GENRANK_BF16) return GENRANK_ERR_UNSUPPORTED;
  const int max_tiles = max_tiles_of(a.max_seqlen);
  if (a.T + (long long)BM >= INT32_MAX / 2) return GENRANK_ERR_UNSUPPORTED;
  Params p;
  if (!make_map(&p.tq, a.q, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tk, a.k, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tv, a.v, a.T, a.H, a.tok_stride))
    return GENRANK_ERR_CUDA;
  p.a = a;
  uint8_t* ws = (uint8_t*)a.ws;
  int32_t* count = (int32_t*)ws;
  int4* recs = (int4*)(ws + kHeaderBytes);
  float* cbias = (float*)(ws + kHeaderBytes + recs_bytes(a.B, a.max_seqlen));
  p.count = count;
  p.recs = recs;
  p.cbias = cbias;
  p.Tp = scratch_tp(a.T, a.B);
  k_prologue<<<a.B + 1, 256, 0, st>>>(a, max_tiles, recs, count, cbias, p.Tp);
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
  k_attn_fwd_tc<<<2 * sms, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace gr

