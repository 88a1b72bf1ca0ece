// Backward of the jagged masked ALiBi attention on 5th-generation tensor cores.
//
// Gradients of O = softmax(S) V with s_ij = scale q_i.k_j - m|p_i - p_j| - m_t|t_i - t_j|
// ("GenRank [2025]" chapter notes §1.4.2 ALiBi score; §1.4.1 candidate mask): the
// biases have no parameters, so only dQ, dK, dV exist:
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D_i = rowsum(dO_i * O_i),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Decomposition (bf16 inputs, head dim 64, fp32 accumulation):
//   * A prologue lists (user, 128-key history tile) work records, longest first, and
//     a record per token (its user's scratch offset, candidate bit, time since the
//     user's first token).  A per-row pass then writes per token and head the ALiBi
//     column term c_j (log2 units), the log2-domain LSE in column-term form
//     lse2_i = LSE_i log2 e + c_i, and D_i, so that
//     p_ij = 2^(scale log2e q_i.k_j + c_j - lse2_i) on every visible pair.
//   * One CTA per SM walks the records.  For a history key tile [k0, k0+128) the
//     visible queries are the user's rows i >= j (later history rows and every
//     candidate); they are visited one 128-row query tile at a time.
//   * Warp 1 loads K, V once per record and Q, dO, lse2, D per query tile (TMA,
//     128B swizzle, no multicast; bulk copies for the per-row terms).
//   * Warp 0 (one thread) issues tcgen05.mma.  Each query tile is taken as two halves
//     of 64 queries: S^T = K Q_x^T and dP^T = V dO_x^T of half x go into TMEM.  The
//     softmax warps write P^T (bf16) into TMEM over S^T columns they have read and
//     dS^T into shared memory (UMMA 128B-swizzled K-major layout, two buffers).  When
//     half x is done, dV += P^T dO_x (P^T from TMEM) and dK += dS^T Q_x are issued,
//     then half x of the next query tile (of this record or of the next one), which
//     overwrites P^T in order and runs while the softmax works on the other half.
//     dQ_part = dS K (dS^T read as an MN-major operand) follows the second half.
//   * Warps 2-9 (two threads per key row and half, each on 32 of its 64 query
//     columns, TMEM access shape 16x32bx2, so two of these warps share each SM
//     sub-partition) compute P^T and dS^T.
//   * Warps 10-13 (one query row per thread) add each dQ_part into an fp32 dQ
//     accumulator in global memory: 32 rows x 32 columns at a time are staged in shared
//     memory and reduced by the TMA engine (cp.reduce.async.bulk.tensor add), which
//     keeps the load/store path free for the operand traffic of the tensor cores.  Per
//     record they move dK (times scale) and dV from TMEM to global memory through the
//     same staging box, as whole 128-byte rows.
//   * K and V are double-buffered by record, so the next record's loads and its
//     first S^T, dP^T overlap the end of the current one.
//   * Candidate keys are seen only by their own row; a small kernel applies that self
//     term (dk, dv of candidate tokens, and ds k into the dQ accumulator), and a
//     streaming pass writes dq = scale * dQ_acc.
// Every mbarrier wait is bounded in time; a timeout sets GENRANK_DERR_TIMEOUT, every
// role drains out of its loop, the copies, MMAs and bulk reductions already issued are
// waited for (bounded), and the CTA frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {
namespace tcb {

constexpr int BM = 128;  // keys per record tile / queries per query tile
constexpr int DH = 64;
constexpr int kThreads = 448;  // warp 0 MMA, 1 TMA, 2-9 softmax, 10-13 dQ reduction
constexpr int kSoftmaxWarps = 8;
constexpr uint32_t kTileBytes = BM * DH * 2;  // 16 KB
constexpr uint32_t kRowBytes = BM * 4;        // one per-row fp32 vector of a tile
constexpr uint32_t kPSBytes = BM * BM * 2;    // 32 KB (P^T or dS^T)

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffK = 0;                          // 2 stages (one per record)
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;     // 2 stages
constexpr uint32_t kOffQ = kOffV + 2 * kTileBytes;     // 2 stages
constexpr uint32_t kOffDO = kOffQ + 2 * kTileBytes;    // 2 stages
constexpr uint32_t kOffL2 = kOffDO + 2 * kTileBytes;   // lse2, 2 stages
constexpr uint32_t kOffD = kOffL2 + 2 * kRowBytes;     // D, 2 stages
constexpr uint32_t kOffTQ = kOffD + 2 * kRowBytes;     // bucketed bias: query times, 2 stages
constexpr uint32_t kOffDS = kOffTQ + 2 * kRowBytes;    // dS^T, 2 buffers
constexpr uint32_t kOffStage = kOffDS + 2 * kPSBytes;  // dQ_part staging, 4 x 4 KB
constexpr uint32_t kStageBytes = 32 * 32 * 4;           // 32 rows x 32 fp32 columns
constexpr uint32_t kOffBar = kOffStage + 4 * kStageBytes;
constexpr uint32_t kNumBars = 21;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kOffStage % 1024 == 0, "128B-swizzled staging must be 1024-byte aligned");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// tensor memory
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // S^T  (keys x queries, fp32); then P^T over it (bf16)
constexpr uint32_t kColDP = 128;  // dP^T
constexpr uint32_t kColDV = 256;  // dV   (keys x dh)
constexpr uint32_t kColDK = 320;  // dK
constexpr uint32_t kColDQ = 384;  // dQ_part, two buffers of 64 (queries x dh)

constexpr int kQH = BM / 2;  // queries per half tile
constexpr uint32_t kIdescS = idesc_bf16_f32(BM, kQH, 0, 0);  // K / V K-major, Q / dO K-major
constexpr uint32_t kIdescKV = idesc_bf16_f32(BM, DH, 0, 1);  // P^T, dS^T K-major; dO, Q MN-major
constexpr uint32_t kIdescQ = idesc_bf16_f32(BM, DH, 1, 1);   // dS MN-major; K MN-major

constexpr size_t kHeaderBytes = 256;

// S^T / dP^T and P^T are handled per query half (64 queries): one S-full and one
// P-full barrier per half.
enum Bar { kKVFull = 0, kKVEmpty = 2, kQDFull = 4, kQDEmpty = 6, kSFull = 8, kPFull = 10,
           kDSFree = 12, kDQFull = 14, kDQEmpty = 16, kDKVFull = 18, kDKVEmpty = 19, kDone = 20 };

struct Params {
  CUtensorMap tq, tk, tv, tdo;
  CUtensorMap tdq;  // the fp32 dQ accumulator [T][H][64], box 32 columns x 32 rows
  AttnArgs a;
  const int4* recs;
  const int32_t* count;
  const float* cbias;  // [H][Tp]
  const float* lse2;   // [H][Tp]
  const float* dsum;   // [H][Tp]  (D)
  const int32_t* trel; // [Tp] bucketed bias: per-token time since the user's first token
  float* dqacc;        // [T][H][64]
  long long Tp;
};

struct Rec {
  int s, L, n, k0, nq, spad, h;
};

GR_DEVICE Rec load_rec(const Params& P, int w) {
  const int pair = w / P.a.H;
  const int4 r0 = P.recs[2 * pair];
  const int4 r1 = P.recs[2 * pair + 1];
  Rec r;
  r.h = w - pair * P.a.H;
  r.s = r0.x;
  r.L = r0.y;
  r.n = r0.z;
  r.k0 = r0.w;
  r.nq = r1.x;
  r.spad = r1.y;
  return r;
}

__host__ __device__ inline long long seg_start(long long s, int u) {
  return 4 * ((s + 3) / 4) + 4LL * u;
}
__host__ __device__ inline long long scratch_tp(long long T, int B) {
  return ((T + 4LL * B + 4 + BM) + 3) / 4 * 4;
}

// ------------------------------------------------------------------------------------------
// prologue: records (block B) and per-row terms (blocks 0..B-1)
// ------------------------------------------------------------------------------------------
constexpr int kMaxBuckets = 257;
// Per-token info: x = (user segment start in the scratch - user start) | kCandBit for a
// candidate token; y = the float bits of t - t_0 (seconds since the user's first token),
// or for the bucketed time bias t - t_0 itself as an int, clamped to [0, kMaxRelTime).
// Tokens of no valid user keep the memset value, x = -1.
constexpr int kCandBit = 1 << 30;
constexpr int kMaxRelTime = 1 << 29;
// bucketed time bias: see the forward kernel (gap biased so its bits read as the float
// 2^23 + gap + 1; the bucket is the binary exponent of (gap + 1)^4, capped at 62)
constexpr int kTimeMagic = 0x4B000001;
constexpr int kTimeCap = kTimeMagic + 46340;
constexpr float kTwo23 = 8388608.f;

__global__ void __launch_bounds__(256) k_bwd_prologue(const __grid_constant__ AttnArgs a,
                                                      int max_tiles, int4* recs, int32_t* count,
                                                      int32_t* uorder, int2* tinfo) {
  const int b = blockIdx.x;
  if (b < a.B) {  // per-token facts for the per-row kernels (one independent load there)
    const long long s = a.off[b], e = a.off[b + 1];
    if (s < 0 || e < s || e > a.T) return;
    const int n = (int)max(0LL, min((long long)a.hist_len[b], e - s));
    const int segoff = (int)(seg_start(s, b) - s);
    const long long t0 = e > s ? a.ts[s] : 0;  // (an empty user reads nothing)
    const bool bucket = a.time_bias == kTimeBiasBucketed;
    for (long long t = s + threadIdx.x; t < e; t += blockDim.x) {
      const long long dt = a.ts[t] - t0;
      tinfo[t] = make_int2(segoff | (t - s >= n ? kCandBit : 0),
                           bucket ? (int)min(max(dt, 0LL), (long long)kMaxRelTime - 1)
                                  : __float_as_int((float)dt));
    }
    return;
  }
  // Records go out user by user (users with the most history key tiles first, each
  // user's key tiles in order, so the most query tiles first): the persistent grid
  // takes consecutive records (times H heads) together, so one user's records run
  // side by side and share its Q, dO tiles in L2.
  __shared__ int hist[kMaxBuckets];
  __shared__ int warp_sums[8];
  for (int i = threadIdx.x; i < kMaxBuckets; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  auto tiles_of_user = [&](int u, bool check, int* qtiles_out) -> int {
    const long long s = a.off[u], e = a.off[u + 1];
    if (s < 0 || e < s || e > a.T) {
      if (check) flag(a.err, GENRANK_DERR_LAYOUT);
      *qtiles_out = 0;
      return 0;
    }
    const int L = (int)(e - s);
    const int n = max(0, min(a.hist_len[u], L));
    const int qtiles = (L + BM - 1) / BM;
    if (check && qtiles > max_tiles) flag(a.err, GENRANK_DERR_LAYOUT);
    *qtiles_out = min(qtiles, max_tiles);
    return min((n + BM - 1) / BM, max_tiles);
  };
  int qt = 0;
  for (int u = threadIdx.x; u < a.B; u += blockDim.x)
    atomicAdd(&hist[min(tiles_of_user(u, true, &qt), kMaxBuckets - 1)], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = kMaxBuckets - 1; q >= 0; --q) {
      const int c = hist[q];
      hist[q] = acc;
      acc += c;
    }
  }
  __syncthreads();
  for (int u = threadIdx.x; u < a.B; u += blockDim.x)
    uorder[atomicAdd(&hist[min(tiles_of_user(u, false, &qt), kMaxBuckets - 1)], 1)] = u;
  __syncthreads();
  // record slots: exclusive prefix sum of the ordered users' key-tile counts
  const int chunk = (a.B + 255) / 256;
  const int k0 = min(a.B, (int)threadIdx.x * chunk), k1 = min(a.B, k0 + chunk);
  int mine = 0;
  for (int k = k0; k < k1; ++k) mine += tiles_of_user(uorder[k], false, &qt);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  int before = 0, total = 0;
  for (int q = 0; q < 8; ++q) {
    if (q < wid) before += warp_sums[q];
    total += warp_sums[q];
  }
  int slot = before + x - mine;
  for (int k = k0; k < k1; ++k) {
    const int u = uorder[k];
    const int ktiles = tiles_of_user(u, false, &qt);
    const int s = a.off[u];
    const int L = a.off[u + 1] - s;
    const int n = max(0, min(a.hist_len[u], L));
    for (int kt = 0; kt < ktiles; ++kt, ++slot) {
      recs[2 * slot] = make_int4(s, L, n, kt * BM);
      recs[2 * slot + 1] = make_int4(qt - kt, (int)seg_start(s, u), u, 0);
    }
  }
  if (threadIdx.x == 0) *count = total;
}

// Per (token, head) terms, eight lanes per pair (16-byte loads of O and dO rows):
// c_j = log2 e (m_h p_j + m_t,h (t_j - t_0)), lse2_i = LSE_i log2 e + c_i and
// D_i = rowsum(dO_i * O_i), at the user's segment of the [H][Tp] scratch.  Every load
// is issued up front (the per-token info replaces a chain through the user's offsets).
// With the bucketed time bias, c_j holds the position part only and the token's time
// goes to trel (written by the head-0 lane).
__global__ void __launch_bounds__(256) k_bwd_rows(const __grid_constant__ AttnArgs a,
                                                  const int2* __restrict__ tinfo,
                                                  float* cbias, float* lse2, float* dsum,
                                                  int32_t* trel, long long Tp) {
  const long long x = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 3;  // pair
  const int sub = threadIdx.x & 7;
  const long long tend = min(a.T, (long long)a.off[a.B]);
  const long long tok = x / a.H;
  const int h = (int)(x - tok * a.H);
  const bool live = tok < tend;
  float dd = 0.f, lse = 0.f;
  int2 ti = make_int2(-1, 0);
  int pos = 0;
  if (live) {
    ti = tinfo[tok];
    pos = a.pos[tok];
    lse = a.lse_in[(long long)h * a.T + tok];
    const uint4 ov = *reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.o + tok * a.o_stride +
                                                     h * DH + 8 * sub);
    const uint4 gv = *reinterpret_cast<const uint4*>(
        (const __nv_bfloat16*)a.dO + tok * a.o_stride + h * DH + 8 * sub);
    float of[8], gf[8];
    Elem<__nv_bfloat16>::unpack(ov, of);
    Elem<__nv_bfloat16>::unpack(gv, gf);
#pragma unroll
    for (int e = 0; e < 8; ++e) dd = fmaf(of[e], gf[e], dd);
  }
  dd += __shfl_xor_sync(0xffffffffu, dd, 4);
  dd += __shfl_xor_sync(0xffffffffu, dd, 2);
  dd += __shfl_xor_sync(0xffffffffu, dd, 1);
  if (!live || sub != 0) return;
  if (ti.x < 0) return;  // tokens of no valid user (the schedule flags the layout)
  const long long seg_tok = tok + (ti.x & (kCandBit - 1));
  float c;
  if (a.time_bias == kTimeBiasBucketed) {
    c = kLog2e * (a.slope_pos[h] * (float)pos);
    if (h == 0) trel[seg_tok] = ti.y;
  } else {
    c = kLog2e * (a.slope_pos[h] * (float)pos + a.slope_time[h] * __int_as_float(ti.y));
  }
  const long long idx = (long long)h * Tp + seg_tok;
  cbias[idx] = c;
  lse2[idx] = lse * kLog2e + c;
  dsum[idx] = dd;
}

// ------------------------------------------------------------------------------------------
// main kernel
// ------------------------------------------------------------------------------------------
GR_DEVICE uint32_t parity(int fill) { return (uint32_t)(fill & 1); }

GR_DEVICE bool wait_warp(uint64_t* bar, uint32_t par, volatile int* abort_flag, int32_t* err) {
  const bool ok = mbar_wait(bar, par, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

// Write 16 bf16 values (8 packed words) of row r, keys/queries [c0, c0+16) with
// c0 % 16 == 0, into a 128-column operand tile laid out as two 64-column blocks of
// 128-byte rows with 16-byte chunks XOR-swizzled by row (the UMMA 128B-swizzle
// canonical layout).
GR_DEVICE void store_row_chunk16(uint8_t* tile, int r, int c0, const uint32_t (&pk)[8]) {
  const int blk = c0 >> 6;
  uint8_t* row = tile + blk * (BM * 128) + r * 128;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int cc = ((c0 & 63) >> 3) + q;
    *reinterpret_cast<uint4*>(row + ((cc ^ (r & 7)) << 4)) =
        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  }
}

template <bool kBucket>
__global__ void __launch_bounds__(kThreads, 1) k_attn_bwd_tc(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnArgs& a = P.a;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kKVFull + i], 1);
      mbar_init(&bars[kKVEmpty + i], 1);
    }
    mbar_init(&bars[kDKVFull], 1);
    mbar_init(&bars[kDKVEmpty], 4);  // one arrival per dK/dV-storing warp
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[kQDFull + i], 1);
      mbar_init(&bars[kQDEmpty + i], 1);
      mbar_init(&bars[kDQFull + i], 1);
      mbar_init(&bars[kDQEmpty + i], 4);  // one arrival per reducing warp
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars[kSFull + x], 1);
      mbar_init(&bars[kPFull + x], kSoftmaxWarps);
    }
    mbar_init(&bars[kDSFree], 1);
    mbar_init(&bars[kDSFree + 1], 1);
    mbar_init(&bars[kDone], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&P.tq);
    tma_prefetch_desc(&P.tk);
    tma_prefetch_desc(&P.tv);
    tma_prefetch_desc(&P.tdo);
    tma_prefetch_desc(&P.tdq);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = *P.count * a.H;

  if (warp == 1) {
    // ---------------------------------------------------------------- TMA producer
    int it = 0, g = 0;
    int kv_n = 0, qd_n = 0;  // K/V and Q/dO loads issued
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Rec rc = load_rec(P, w);
      const int kvs = it & 1;
      if (!wait_warp(&bars[kKVEmpty + kvs], parity(it >> 1) ^ 1u, abort_flag, a.err)) break;
      if (lane == 0) {
        mbar_expect_tx(&bars[kKVFull + kvs], 2 * kTileBytes);
        tma_load_3d(smem + kOffK + kvs * kTileBytes, &P.tk, &bars[kKVFull + kvs], 0, rc.h,
                    rc.s + rc.k0);
        tma_load_3d(smem + kOffV + kvs * kTileBytes, &P.tv, &bars[kKVFull + kvs], 0, rc.h,
                    rc.s + rc.k0);
      }
      kv_n = it + 1;
      const long long roff = (long long)rc.h * P.Tp + rc.spad;
      bool ok = true;
      for (int t = 0; t < rc.nq; ++t, ++g) {
        const int st = g & 1;
        if (!wait_warp(&bars[kQDEmpty + st], parity(g >> 1) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const int q0 = rc.k0 + t * BM;
          mbar_expect_tx(&bars[kQDFull + st], 2 * kTileBytes + (kBucket ? 3 : 2) * kRowBytes);
          tma_load_3d(smem + kOffQ + st * kTileBytes, &P.tq, &bars[kQDFull + st], 0, rc.h,
                      rc.s + q0);
          tma_load_3d(smem + kOffDO + st * kTileBytes, &P.tdo, &bars[kQDFull + st], 0, rc.h,
                      rc.s + q0);
          bulk_load(smem + kOffL2 + st * kRowBytes, P.lse2 + roff + q0, kRowBytes,
                    &bars[kQDFull + st]);
          bulk_load(smem + kOffD + st * kRowBytes, P.dsum + roff + q0, kRowBytes,
                    &bars[kQDFull + st]);
          if (kBucket)
            bulk_load(smem + kOffTQ + st * kRowBytes, P.trel + rc.spad + q0, kRowBytes,
                      &bars[kQDFull + st]);
        }
        qd_n = g + 1;
      }
      if (!ok) break;
    }
    // on the way out (a timeout included), the copies issued last land before the CTA
    // exits; in a normal run they have long been consumed
    if (lane == 0) {
      for (int x = max(0, kv_n - 2); x < kv_n; ++x)
        mbar_drain(&bars[kKVFull + (x & 1)], parity(x >> 1));
      for (int x = max(0, qd_n - 2); x < qd_n; ++x)
        mbar_drain(&bars[kQDFull + (x & 1)], parity(x >> 1));
    }
  } else if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    // Tiles g = 0, 1, ... run across records; each tile is handled as two query halves
    // X = 0, 1.  When the softmax has finished half X of tile g, dV and dK take that
    // half, and half X of the next tile (of this record or of the next one) is issued
    // at once: it runs while the softmax works on the other half.  dQ of tile g comes
    // after both halves.
    // Descriptor bases, built once: an operand's descriptor is its base plus the byte
    // offset / 16 of the stage, half and k-step (the 14-bit address field never
    // carries: shared memory is below 256 KB).  Each MMA then costs two adds, which
    // keeps this thread's instructions between MMAs few: the tensor pipe takes about
    // one MMA ahead, and this warp shares its sub-partition with the softmax warps.
    constexpr uint32_t kTileD = kTileBytes >> 4, kPSD = kPSBytes >> 4, kRowD = (16 * 128) >> 4;
    const uint64_t kmK = smem_desc_sw128(smem_u32(smem + kOffK), 16, 1024);
    const uint64_t kmV = smem_desc_sw128(smem_u32(smem + kOffV), 16, 1024);
    const uint64_t kmQ = smem_desc_sw128(smem_u32(smem + kOffQ), 16, 1024);
    const uint64_t kmDO = smem_desc_sw128(smem_u32(smem + kOffDO), 16, 1024);
    const uint64_t kmDS = smem_desc_sw128(smem_u32(smem + kOffDS), 16, 1024);
    const uint64_t mnQ = smem_desc_sw128(smem_u32(smem + kOffQ), kTileBytes, 1024);
    const uint64_t mnDO = smem_desc_sw128(smem_u32(smem + kOffDO), kTileBytes, 1024);
    const uint64_t mnK = smem_desc_sw128(smem_u32(smem + kOffK), kTileBytes, 1024);
    const uint64_t mnDS = smem_desc_sw128(smem_u32(smem + kOffDS), BM * 128, 1024);
    // S^T = K Q_X^T and dP^T = V dO_X^T for query half X of tile gg (keys of stage kvs)
    auto issue_sdp = [&](int gg, int kvs, int x) {
      const uint64_t a_k = kmK + kvs * kTileD, a_v = kmV + kvs * kTileD;
      const uint32_t qo = (gg & 1) * kTileD + x * ((kQH * 128) >> 4);
      const uint64_t b_q = kmQ + qo, b_do = kmDO + qo;
#pragma unroll
      for (int k = 0; k < DH / 16; ++k)
        mma_bf16_ss(tmem + kColS + kQH * x, a_k + 2 * k, b_q + 2 * k, kIdescS, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < DH / 16; ++k)
        mma_bf16_ss(tmem + kColDP + kQH * x, a_v + 2 * k, b_do + 2 * k, kIdescS,
                    k > 0 ? 1u : 0u);
      mma_commit(&bars[kSFull + x]);
    };
    // dV += P^T dO_X with P^T read from TMEM, and dK += dS^T Q_X, over query half X
    // (K = 64 queries).  The softmax wrote P^T over the S^T columns it had read:
    // queries [16k, 16k + 16) of the half at column 64 x + 32 (k / 2) + 8 (k % 2).
    auto issue_dvdk = [&](int gg, int x, bool first) {
      const uint32_t st = gg & 1;
      const uint32_t ro = st * kTileD + x * (kQH / 16) * kRowD;  // 16-query steps of the half
      const uint64_t b_do = mnDO + ro, b_q = mnQ + ro;
      const uint64_t a_ds = kmDS + st * kPSD + x * ((BM * 128) >> 4);
      const uint32_t a_p = tmem + kColS + kQH * x;
#pragma unroll
      for (int k = 0; k < kQH / 16; ++k)
        mma_bf16_ts(tmem + kColDV, a_p + 32 * (k >> 1) + 8 * (k & 1), b_do + k * kRowD,
                    kIdescKV, (!first || k > 0) ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < kQH / 16; ++k)
        mma_bf16_ss(tmem + kColDK, a_ds + 2 * k, b_q + k * kRowD, kIdescKV,
                    (!first || k > 0) ? 1u : 0u);
    };
    int it = 0, g = 0;
    bool ok = blockIdx.x < total;
    if (ok) {
      ok = mbar_wait(&bars[kKVFull], 0u, abort_flag, a.err) &&
           mbar_wait(&bars[kQDFull], 0u, abort_flag, a.err);
      if (ok) {
        tc_fence_after();
        issue_sdp(0, 0, 0);
        issue_sdp(0, 0, 1);
      }
    }
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
      const Rec rc = load_rec(P, w);
      const int kvs = it & 1;
      for (int t = 0; t < rc.nq; ++t, ++g) {
        const int st = g & 1;
        // the next tile: this record's next query tile, or the next record's first
        const bool last = t + 1 == rc.nq;
        const bool has_next = !last || w + (int)gridDim.x < total;
        const int nkvs = last ? kvs ^ 1 : kvs;
        // ---- half 0
        if (!mbar_wait(&bars[kPFull], parity(g), abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the record's first dV, dK overwrite the accumulators: the previous record's
        // dV, dK must have been read out
        if (t == 0 && !mbar_wait(&bars[kDKVEmpty], parity(it) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_dvdk(g, 0, t == 0);
        if (has_next) {
          if ((last && !mbar_wait(&bars[kKVFull + nkvs], parity((it + 1) >> 1), abort_flag,
                                  a.err)) ||
              !mbar_wait(&bars[kQDFull + (st ^ 1)], parity((g + 1) >> 1), abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_sdp(g + 1, nkvs, 0);  // after dV has read P^T of half 0 (in order)
        }
        // ---- half 1
        if (!mbar_wait(&bars[kPFull + 1], parity(g), abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_dvdk(g, 1, false);
        mma_commit(&bars[kQDEmpty + st]);  // Q, dO of this tile are read for the last time
        if (last) mma_commit(&bars[kDKVFull]);
        if (has_next) issue_sdp(g + 1, nkvs, 1);
        // dQ_part = dS K  (M = queries read from dS^T as MN-major, K = 128 keys)
        if (!mbar_wait(&bars[kDQEmpty + st], parity(g >> 1) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          const uint64_t a_ds = mnDS + st * kPSD, b_k = mnK + kvs * kTileD;
#pragma unroll
          for (int k = 0; k < BM / 16; ++k)
            mma_bf16_ss(tmem + kColDQ + st * DH, a_ds + k * kRowD, b_k + k * kRowD, kIdescQ,
                        k > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kDQFull + st]);
        mma_commit(&bars[kDSFree + st]);
        if (last) mma_commit(&bars[kKVEmpty + kvs]);
      }
      if (*abort_flag) ok = false;
    }
    // every MMA issued (on a timeout too) has completed before TMEM is freed
    mma_commit(&bars[kDone]);
    mbar_drain(&bars[kDone], 0);
  } else if (warp >= 2 && warp < 2 + kSoftmaxWarps) {
    // ---------------------------------------------------------------- softmax (key rows)
    const int quad = warp & 3;              // TMEM lane quadrant of the warp
    const int rh = (warp - 2) >> 2;         // upper or lower 16 lanes of the quadrant
    const int hq = lane >> 4;               // which 32 queries of each half
    const int r = quad * 32 + rh * 16 + (lane & 15);  // key row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32 + rh * 16) << 16);
    const float scale_log2 = a.scale * kLog2e;
    const float* sL2 = reinterpret_cast<const float*>(smem + kOffL2);
    const float* sD = reinterpret_cast<const float*>(smem + kOffD);
    const int* sTQ = reinterpret_cast<const int*>(smem + kOffTQ);
    uint8_t* sDS = smem + kOffDS;
    int g = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      __syncwarp();
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Rec rc = load_rec(P, w);
      const int j = rc.k0 + r;  // this thread's key (local index)
      const bool key = j < rc.n;
      const float cbj = key ? P.cbias[(long long)rc.h * P.Tp + rc.spad + j] : 0.f;
      const uint64_t sl2 = f2_pack(scale_log2, scale_log2), cb2 = f2_pack(cbj, cbj);
      // on a query tile wholly inside the user and past the diagonal every query sees
      // every key row, so only the key row's own validity is left: a row past the
      // user's history gets c_j = -inf there, and 2^-inf = 0 needs no select
      const float cbf = key ? cbj : -INFINITY;
      const uint64_t cb2f = f2_pack(cbf, cbf);
      // bucketed time bias: this key's time, biased (see kTimeMagic), and -m_t log2 e
      const int tj_m = kBucket && key ? kTimeMagic - P.trel[rc.spad + j] : 0;
      const float nmt2 = kBucket ? -a.slope_time[rc.h] * kLog2e : 0.f;
      bool ok = true;
      for (int t = 0; t < rc.nq && ok; ++t, ++g) {
        const int st = g & 1;
        const int q0 = rc.k0 + t * BM;
        // visible iff key valid, query row inside the user and i >= j
        const int ilo = max(j, q0);  // first visible query (local index)
        const int ihi = rc.L;        // one past the last
        uint8_t* sDSb = sDS + st * kPSBytes;
        for (int x = 0; x < 2; ++x) {
          // half x of S^T was issued after dV had read this half's previous P^T
          if (!wait_warp(&bars[kSFull + x], parity(g), abort_flag, a.err) ||
              (x == 0 && !wait_warp(&bars[kQDFull + st], parity(g >> 1), abort_flag, a.err))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int qc = kQH * x + 32 * hq;  // this thread's first query column in the tile
          const float* l2 = sL2 + st * BM + qc;
          const float* dd = sD + st * BM + qc;
          const int* tq = sTQ + st * BM + qc;
          const int qbase = q0 + qc;
          const uint32_t s_addr = lane_base + kColS + kQH * x;
          const uint32_t dp_addr = lane_base + kColDP + kQH * x;
          uint32_t sa[16], da[16], sb[16], db[16];
          tmem_ld_half16_async<32>(s_addr, sa);
          tmem_ld_half16_async<32>(dp_addr, da);
          tmem_ld_wait(sa);
          tmem_ld_wait(da);
          tmem_ld_half16_async<32>(s_addr + 16, sb);
          tmem_ld_half16_async<32>(dp_addr + 16, db);
          // this dS^T buffer was last read by dK, dQ of tile g - 2
          if (x == 0 &&
              !wait_warp(&bars[kDSFree + st], parity(g >> 1) ^ 1u, abort_flag, a.err)) {
            tmem_ld_wait(sb);
            ok = false;
            break;
          }
          // 16 query columns: p = 2^(s scale log2e + c_j - lse2_i) on visible pairs and
          // ds = p (dP - D_i), with the per-query terms read as 16-byte vectors and the
          // arithmetic on column pairs (two-wide fp32 instructions).  P^T goes over the
          // first 16 S^T columns this thread has read (16x32bx2: the upper lanes at
          // +32), dS^T to shared memory.
          auto chunk = [&](const uint32_t (&sv)[16], const uint32_t (&dp)[16], int c0,
                           auto full_tile) {
            constexpr bool kFull = decltype(full_tile)::value;
            uint32_t pk[8], dk[8];
#pragma unroll
            for (int c = 0; c < 16; c += 4) {
              const float4 l4 = *reinterpret_cast<const float4*>(l2 + c0 + c);
              const float4 d4 = *reinterpret_cast<const float4*>(dd + c0 + c);
              uint64_t t01 = f2_sub(kFull ? cb2f : cb2, f2_pack(l4.x, l4.y));
              uint64_t t23 = f2_sub(kFull ? cb2f : cb2, f2_pack(l4.z, l4.w));
              if (kBucket) {  // - m_t bucket(t_i - t_j), four queries at a time
                const int4 ti = *reinterpret_cast<const int4*>(tq + c0 + c);
                const uint64_t two23 = f2_pack(kTwo23, kTwo23);
                const uint64_t g01 = f2_sub(f2_pack(__int_as_float(min(ti.x + tj_m, kTimeCap)),
                                                    __int_as_float(min(ti.y + tj_m, kTimeCap))),
                                            two23);
                const uint64_t g23 = f2_sub(f2_pack(__int_as_float(min(ti.z + tj_m, kTimeCap)),
                                                    __int_as_float(min(ti.w + tj_m, kTimeCap))),
                                            two23);
                const uint64_t s01 = f2_mul(g01, g01), s23 = f2_mul(g23, g23);
                float q4[4];
                f2_unpack(f2_mul(s01, s01), q4[0], q4[1]);
                f2_unpack(f2_mul(s23, s23), q4[2], q4[3]);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  q4[e] = __int_as_float((__float_as_int(q4[e]) >> 23) | 0x4B000000);
                const uint64_t base = f2_pack(kTwo23 + 127.f, kTwo23 + 127.f);
                const uint64_t nm2 = f2_pack(nmt2, nmt2);
                t01 = f2_fma(f2_sub(f2_pack(q4[0], q4[1]), base), nm2, t01);
                t23 = f2_fma(f2_sub(f2_pack(q4[2], q4[3]), base), nm2, t23);
              }
              const uint64_t x01 =
                  f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2, t01);
              const uint64_t x23 =
                  f2_fma(f2_pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), sl2,
                         t23);
              float xv[4], p[4];
              f2_unpack(x01, xv[0], xv[1]);
              f2_unpack(x23, xv[2], xv[3]);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i = qbase + c0 + c + e;
                p[e] = (kFull || (key && i >= ilo && i < ihi)) ? ex2(xv[e]) : 0.f;
              }
              const uint64_t p01 = f2_pack(p[0], p[1]), p23 = f2_pack(p[2], p[3]);
              const uint64_t ds01 = f2_mul(
                  p01, f2_sub(f2_pack(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                              f2_pack(d4.x, d4.y)));
              const uint64_t ds23 = f2_mul(
                  p23, f2_sub(f2_pack(__uint_as_float(dp[c + 2]), __uint_as_float(dp[c + 3])),
                              f2_pack(d4.z, d4.w)));
              float ds[4];
              f2_unpack(ds01, ds[0], ds[1]);
              f2_unpack(ds23, ds[2], ds[3]);
              pk[c / 2] = pack_bf16(p[0], p[1]);
              pk[c / 2 + 1] = pack_bf16(p[2], p[3]);
              dk[c / 2] = pack_bf16(ds[0], ds[1]);
              dk[c / 2 + 1] = pack_bf16(ds[2], ds[3]);
            }
            tmem_st_half8_nowait<32>(s_addr + c0 / 2, pk);
            store_row_chunk16(sDSb, r, qc + c0, dk);
          };
          auto both = [&](auto full_tile) {
            chunk(sa, da, 0, full_tile);  // stores to columns [0, 8): read, not in flight
            tmem_ld_wait(sb);
            tmem_ld_wait(db);
            chunk(sb, db, 16, full_tile);  // stores to columns [8, 16)
          };
          // the same for the whole warp: the record's tile t and the user's length (the
          // bucketed form keeps one copy of the chunk code: a second one spills there)
          if (!kBucket && t > 0 && q0 + BM <= ihi)
            both(std::true_type{});
          else
            both(std::false_type{});
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kPFull + x]);
        }
      }
      if (!ok) break;
    }
  } else if (warp >= 2 + kSoftmaxWarps) {
    // ---------------------------------------------------------------- dQ reduction (query rows)
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    int g = 0, it = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      __syncwarp();
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Rec rc = load_rec(P, w);
      bool ok = true;
      for (int t = 0; t < rc.nq; ++t, ++g) {
        if (t + 1 == rc.nq) {
          // the record's dK (times scale), then dV, once its last dV, dK MMAs are
          // done (before its last dQ_part); the accumulators are released after the dV
          // load.  Each warp stages its 32 key rows (bf16, 128 bytes each) in its
          // 128B-swizzled box and writes them as whole rows, four rows per store
          // instruction; rows of candidate keys and past the user are skipped.
          if (!wait_warp(&bars[kDKVFull], parity(it), abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* stg = smem + kOffStage + (warp & 3) * kStageBytes;
          const int jr0 = rc.k0 + 32 * (warp & 3);  // the warp's first key row (local)
#pragma unroll 1
          for (int m = 0; m < 2; ++m) {
            const float mul = m ? 1.f : a.scale;
            if (lane == 0) bulk_wait_read_all();  // the box's last reduction has read it
            __syncwarp();
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {  // 32 columns at a time
              float v[32];
              tmem_ld32(tmem + lane_base + (m ? kColDV : kColDK) + 32 * hf, v);
              if (m == 1 && hf == 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kDKVEmpty]);
              }
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const int k = 4 * hf + kk;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = v[8 * kk + e] * mul;
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((k ^ (lane & 7)) << 4)) =
                    Elem<__nv_bfloat16>::pack(f);
              }
            }
            __syncwarp();
            // lane: row 4q + lane / 8 of the box, 16-byte chunk lane % 8
            const int c = lane & 7;
            const int nrows = min(32, rc.n - jr0);  // rows of history keys in the box
            const uint8_t* src = stg + (lane >> 3) * 128;
            __nv_bfloat16* dst = (__nv_bfloat16*)(m ? a.dv : a.dk) +
                                 ((long long)rc.s + jr0 + (lane >> 3)) * a.tok_stride +
                                 rc.h * DH + 8 * c;
            const long long dstep = 4LL * a.tok_stride;
#pragma unroll 2
            for (int q = 0; q < 8; ++q, src += 4 * 128, dst += dstep) {
              const int rr = 4 * q + (lane >> 3);
              if (rr < nrows)
                *reinterpret_cast<uint4*>(dst) =
                    *reinterpret_cast<const uint4*>(src + ((c ^ (rr & 7)) << 4));
            }
            __syncwarp();  // every lane has read the box before it is written again
          }
        }
        const int db = g & 1;
        if (!wait_warp(&bars[kDQFull + db], parity(g >> 1), abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float dq[DH];
        tmem_ld64(tmem + lane_base + kColDQ + db * DH, dq);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kDQEmpty + db]);
        // The warp's 32 query rows go to the accumulator by TMA reduce-add, 32 columns at
        // a time through a 128B-swizzled staging box (one bulk operation instead of 512
        // scattered vector reductions; rows past the user's end are staged as zeros).
        const int r0 = rc.k0 + t * BM + 32 * (warp & 3);  // the warp's first row (local)
        if (r0 < rc.L) {
          const bool live = r0 + lane < rc.L;
          uint8_t* stg = smem + kOffStage + (warp & 3) * kStageBytes;
#pragma unroll
          for (int c = 0; c < DH; c += 32) {
            if (lane == 0) bulk_wait_read_all();  // the last reduction has read the box
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 v = live ? make_float4(dq[c + 4 * k], dq[c + 4 * k + 1],
                                                  dq[c + 4 * k + 2], dq[c + 4 * k + 3])
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
              *reinterpret_cast<float4*>(stg + lane * 128 + ((k ^ (lane & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&P.tdq, stg, c, rc.h, rc.s + r0);
              bulk_commit();
            }
          }
        }
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_all();  // the accumulator is complete when the kernel ends
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------------------------------
// finishing kernels: the candidate self terms, then dq from the accumulator
// ------------------------------------------------------------------------------------------
// gridDim.y blocks per user, eight lanes per (candidate, head), eight of the 64
// columns per lane (16-byte loads).  A candidate token c is seen only by itself (bias 0):
// p = exp(scale q.k - LSE), ds = p (dO.v - D), dv = p dO, dk = scale ds q, and the dQ
// accumulator gains ds k (scaled with the rest by the conversion that follows).  The
// main kernel has finished with the accumulator, so these rows are read and written
// plainly; dk, dv of candidate tokens have no other writer.
__global__ void __launch_bounds__(256) k_bwd_cand(const __grid_constant__ AttnArgs a,
                                                  float* __restrict__ dqacc,
                                                  const float* __restrict__ dsum, long long Tp) {
  const int u = blockIdx.x;
  const long long s = a.off[u], e = a.off[u + 1];
  if (s < 0 || e < s || e > a.T) return;  // flagged by the schedule
  const int L = (int)(e - s);
  const int n = max(0, min(a.hist_len[u], L));
  const int pairs = (L - n) * a.H;
  const long long seg = seg_start(s, u);
  const int sub = threadIdx.x & 7;
  const int step = (int)gridDim.y * (int)(blockDim.x / 8);
  for (int base = (int)blockIdx.y * (int)(blockDim.x / 8); base < pairs;
       base += step) {  // uniform trip count within the block
    const int pr = base + (int)(threadIdx.x >> 3);
    const bool act = pr < pairs;
    const int c = act ? n + pr / a.H : n;
    const int h = act ? pr % a.H : 0;
    const long long tok = s + c;
    const long long qo = tok * a.tok_stride + h * DH + 8 * sub;
    float qf[8], kf[8], vf[8], gf[8];
    float sdot = 0.f, pdot = 0.f;
    if (act) {
      Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.q + qo), qf);
      Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.k + qo), kf);
      Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>((const __nv_bfloat16*)a.v + qo), vf);
      Elem<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(
                                      (const __nv_bfloat16*)a.dO + tok * a.o_stride + h * DH + 8 * sub),
                                  gf);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sdot = fmaf(qf[i], kf[i], sdot);
        pdot = fmaf(gf[i], vf[i], pdot);
      }
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      sdot += __shfl_xor_sync(0xffffffffu, sdot, o);
      pdot += __shfl_xor_sync(0xffffffffu, pdot, o);
    }
    if (!act) continue;
    const float p = expf(sdot * a.scale - a.lse_in[(long long)h * a.T + tok]);
    const float ds = p * (pdot - dsum[(long long)h * Tp + seg + c]);
    float* acc = dqacc + (tok * a.H + h) * DH + 8 * sub;
    float4 a0 = reinterpret_cast<float4*>(acc)[0], a1 = reinterpret_cast<float4*>(acc)[1];
    a0.x = fmaf(ds, kf[0], a0.x); a0.y = fmaf(ds, kf[1], a0.y);
    a0.z = fmaf(ds, kf[2], a0.z); a0.w = fmaf(ds, kf[3], a0.w);
    a1.x = fmaf(ds, kf[4], a1.x); a1.y = fmaf(ds, kf[5], a1.y);
    a1.z = fmaf(ds, kf[6], a1.z); a1.w = fmaf(ds, kf[7], a1.w);
    reinterpret_cast<float4*>(acc)[0] = a0;
    reinterpret_cast<float4*>(acc)[1] = a1;
    float dk[8], dv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dk[i] = a.scale * ds * qf[i];
      dv[i] = p * gf[i];
    }
    *reinterpret_cast<uint4*>((__nv_bfloat16*)a.dk + qo) = Elem<__nv_bfloat16>::pack(dk);
    *reinterpret_cast<uint4*>((__nv_bfloat16*)a.dv + qo) = Elem<__nv_bfloat16>::pack(dv);
  }
}

// dq = scale * dQ_acc for every token of the batch, eight columns per thread: a plain
// stream (two 16-byte loads, one 16-byte store), at full occupancy.
__global__ void __launch_bounds__(256) k_bwd_finish(const __grid_constant__ AttnArgs a,
                                                    const float* __restrict__ dqacc) {
  const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // 8-column chunk
  const long long pair = x >> 3;
  const long long tend = min(a.T, (long long)a.off[a.B]);
  const long long tok = pair / a.H;
  if (tok >= tend) return;
  const int h = (int)(pair - tok * a.H);
  const float4* acc = reinterpret_cast<const float4*>(dqacc) + 2 * x;
  const float4 a0 = acc[0], a1 = acc[1];
  const float f[8] = {a0.x * a.scale, a0.y * a.scale, a0.z * a.scale, a0.w * a.scale,
                      a1.x * a.scale, a1.y * a.scale, a1.z * a.scale, a1.w * a.scale};
  *reinterpret_cast<uint4*>((__nv_bfloat16*)a.dq + tok * a.tok_stride + h * DH +
                            8 * (int)(x & 7)) = Elem<__nv_bfloat16>::pack(f);
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

static bool make_map(CUtensorMap* m, const void* base, long long T, int H, long long stride) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)DH * 2, (cuuint64_t)stride * 2};
  cuuint32_t box[3] = {(cuuint32_t)DH, 1, (cuuint32_t)BM};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// The fp32 dQ accumulator [T][H][64]; box = 32 columns x one head x 32 rows, 128-byte
// swizzle (the staging layout of the reducing warps).
static bool make_map_f32(CUtensorMap* m, const float* base, long long T, int H) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)DH * 4, (cuuint64_t)H * DH * 4};
  cuuint32_t box[3] = {32, 1, 32};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static int max_tiles_of(int max_seqlen) { return (max_seqlen + BM - 1) / BM; }
static size_t recs_bytes(int B, int max_seqlen) {
  return ((size_t)B * max_tiles_of(max_seqlen) * 32 + 15) / 16 * 16;
}
static size_t users_bytes(int B) { return ((size_t)B * 4 + 15) / 16 * 16; }
static size_t tokens_bytes(long long T) { return ((size_t)T * 8 + 15) / 16 * 16; }
static size_t rows_bytes(long long T, int B, int H) {
  return ((size_t)H * scratch_tp(T, B) * sizeof(float) + 15) / 16 * 16;
}

}  // namespace tcb

size_t attn_bwd_tc_workspace(int B, long long T, int H, int max_seqlen) {
  using namespace tcb;
  return kHeaderBytes + recs_bytes(B, max_seqlen) + users_bytes(B) + tokens_bytes(T) +
         rows_bytes(T, B, 1) + 3 * rows_bytes(T, B, H) + (size_t)T * H * DH * sizeof(float);
}

int launch_attn_bwd_tc(const AttnArgs& a, cudaStream_t st) {
  using namespace tcb;
  if (a.dh != DH || a.dtype != GENRANK_BF16) return GENRANK_ERR_UNSUPPORTED;
  if (a.T + (long long)BM >= INT32_MAX / 2) return GENRANK_ERR_UNSUPPORTED;
  Params p;
  if (!make_map(&p.tq, a.q, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tk, a.k, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tv, a.v, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tdo, a.dO, a.T, a.H, a.o_stride))
    return GENRANK_ERR_CUDA;
  p.a = a;
  uint8_t* ws = (uint8_t*)a.ws;
  p.count = (int32_t*)ws;
  p.recs = (int4*)(ws + kHeaderBytes);
  const size_t rb = rows_bytes(a.T, a.B, a.H);
  int32_t* uorder = (int32_t*)(ws + kHeaderBytes + recs_bytes(a.B, a.max_seqlen));
  int2* tinfo = (int2*)((uint8_t*)uorder + users_bytes(a.B));
  int32_t* trel = (int32_t*)((uint8_t*)tinfo + tokens_bytes(a.T));
  uint8_t* rows = (uint8_t*)trel + rows_bytes(a.T, a.B, 1);
  const bool bucket = a.time_bias == kTimeBiasBucketed;
  p.trel = trel;
  p.cbias = (float*)rows;
  p.lse2 = (float*)(rows + rb);
  p.dsum = (float*)(rows + 2 * rb);
  p.dqacc = (float*)(rows + 3 * rb);
  p.Tp = scratch_tp(a.T, a.B);
  if (!make_map_f32(&p.tdq, p.dqacc, a.T, a.H)) return GENRANK_ERR_CUDA;
  // D and the dQ accumulator are adjacent: one memset zeroes both.  A query tile reads D
  // past its user's last row (the gap before the next user's segment), where a masked
  // pair's ds = p (dP - D) with p = 0 must stay 0 whatever the workspace held.
  if (cudaMemsetAsync(rows + 2 * rb, 0, rb + (size_t)a.T * a.H * DH * sizeof(float), st) !=
      cudaSuccess)
    return GENRANK_ERR_CUDA;
  if (a.T > 0 && cudaMemsetAsync(tinfo, 0xff, (size_t)a.T * 8, st) != cudaSuccess)
    return GENRANK_ERR_CUDA;
  k_bwd_prologue<<<a.B + 1, 256, 0, st>>>(a, max_tiles_of(a.max_seqlen), (int4*)p.recs,
                                          (int32_t*)p.count, uorder, tinfo);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  const long long pair_blocks = (a.T * a.H + 31) / 32;  // 8 lanes per (token, head)
  if (pair_blocks > 0) {
    k_bwd_rows<<<(unsigned)pair_blocks, 256, 0, st>>>(a, tinfo, (float*)p.cbias,
                                                      (float*)p.lse2, (float*)p.dsum, trel, p.Tp);
    if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  }
  static DeviceOnce smem_attr[2];
  const void* fn = bucket ? (const void*)k_attn_bwd_tc<true> : (const void*)k_attn_bwd_tc<false>;
  if (!set_smem_limit_once(smem_attr[bucket ? 1 : 0], fn, (int)kSmemBytes))
    return GENRANK_ERR_CUDA;
  const int sms = sm_count_current();
  if (sms <= 0) return GENRANK_ERR_CUDA;
  if (bucket)
    k_attn_bwd_tc<true><<<sms, kThreads, kSmemBytes, st>>>(p);
  else
    k_attn_bwd_tc<false><<<sms, kThreads, kSmemBytes, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  if (a.B > 0) {
    k_bwd_cand<<<dim3((unsigned)a.B, 4), 256, 0, st>>>(a, p.dqacc, p.dsum, p.Tp);
    if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  }
  if (pair_blocks > 0)
    k_bwd_finish<<<(unsigned)pair_blocks, 256, 0, st>>>(a, p.dqacc);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace gr
