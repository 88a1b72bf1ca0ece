// Jagged masked ALiBi attention forward on 5th-generation tensor cores (sm_100a).
//
// Semantics ("GenRank [2025]" chapter notes, §1.4.1 candidate mask and §1.4.2
// ALiBi score; fun-rec "The Overall Generative Ranking Paradigm" §7.2.2):
//   s_ij = scale q_i.k_j - m_h |p_i - p_j| - m_t,h |t_i - t_j|, history rows causal,
//   candidate rows see all history and themselves.
//
// Design (bf16 inputs, head dim 64, fp32 accumulation), one CTA per SM:
//   * A prologue kernel lists (user, 128-row query tile) work records sorted by the
//     number of 128-key tiles they visit (longest first), and writes the ALiBi
//     column term c_j = log2(e) (m_h p_j + m_t,h (t_j - t_0)) for every token and
//     head into a 16-byte aligned scratch layout (entries between users' segments are
//     zeroed, so every term a key tile reads is finite), in fp32 and as three bf16 parts
//     of c_j / (scale log2 e).  On visible pairs p_i >= p_j and t_i >= t_j, so the bias
//     is c_j - c_i; c_i cancels in the softmax (it is the row's fixed offset), c_j is
//     added by the MMA that forms S, and the literal LSE subtracts c_i in the epilogue.
//   * A persistent grid walks the records round-robin (one head per work item).  An
//     item visits its history key tiles (history tile t: key tiles 0..t; candidate
//     rows: the history only; most recent keys first) and, when it holds candidate
//     rows, one diagonal tile: its own rows as keys, of which only each candidate's
//     own key (bias 0) is kept.  Key tiles a query tile never sees are never visited.
//   * Warp 1 issues TMA loads (Q with the rows' own column terms, double-buffered;
//     K, V and the keys' split column terms in a four-stage ring; 128B swizzle, no
//     multicast).
//   * Warp 0 (one thread) issues tcgen05.mma: S = Q K^T + c_j / (scale log2 e) (128 x
//     128, fp32; a fifth K = 16 slice adds the split column terms) into one of two TMEM
//     buffers, the next S before the current P V, and O += P V (128 x 64,
//     fp32) into the item's TMEM O buffer (two, alternating by item), P (bf16 pairs)
//     read from one of two TMEM P buffers.
//   * Warps 2-9 stream the softmax with two threads per query row, each on one half
//     of the key columns (TMEM access shape 16x32bx2), so two softmax warps share
//     each SM sub-partition: offset, mask and exponentials in one pass per tile, with
//     the offset fixed at the row's own column term (every visible key has
//     c_j <= c_i); a tile whose row sum leaves the safe range is redone exactly and O
//     rescaled in TMEM.  Only an item's first tile can need the row mask: it runs
//     chunk by chunk (16 keys) with the two half-warps interleaved by chunks, so that
//     both halves skip wholly masked chunks and only the chunk a row's mask cuts pays
//     for it; the loop over the other tiles holds the plain code alone.
//   * The same kernel scores candidates from a KV cache (or, reading the cache in
//     place, the candidate rows of one jagged token array alone): records then hold
//     candidate tiles only, whose key tiles are the user's history plus the diagonal.
//   * Warps 10-13 (one row per thread) finish each item from its O buffer while the
//     next item runs: O is normalised and written through shared memory as whole
//     128-byte rows, and the literal LSE is stored.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
#include <type_traits>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {
namespace tc {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int DH = 64;   // head dim
constexpr int kThreads = 448;  // warp 0 MMA, 1 TMA, 2-9 softmax, 10-13 epilogue
constexpr int kSoftmaxWarps = 8;  // barrier arrivals are one per warp
constexpr int kStages = 4;     // K/V ring
constexpr uint32_t kTileBytes = BM * DH * 2;  // one Q, K or V tile (16 KB)
constexpr uint32_t kCBBytes = BN * 4;         // fp32 terms (own column terms, key times) of a tile
// The column term c_j enters S through the MMA: each key's row of the K tile is followed
// by 16 more bf16 columns holding c_j / (scale log2 e) as three bf16 parts (the rest of
// the 8-column row in memory zero, the next 8 columns read from the next key's row), and
// each query row by 16 columns (1, 1, 1, 0, ...; zeros in the second 8), so that
// S' = Q K^T + c_j / (scale log2 e) and x = S' scale log2 e - m.  The zeros meet the
// next key's entry, which the prologue has written (every entry a key tile can read is
// written on every call), so their products vanish.
constexpr uint32_t kKABytes = BN * 16;        // one key tile's 8-column rows (2 KB)
constexpr uint32_t kKAStride = kKABytes + 128;  // + a zeroed pad the last row's read reaches
constexpr uint32_t kQABytes = 2 * BM * 16;    // the query side: 1, 1, 1 rows, then zeros
constexpr float kOverflowSum = 1.2676506e30f;   // 2^100: a tile's row sum above this is redone
constexpr float kUnderflowSum = 7.8886091e-31f;  // 2^-100: a first tile's row sum below this too

// dynamic shared memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                                // 2 x 16 KB
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;           // kStages x 16 KB
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;     // kStages x 16 KB
constexpr uint32_t kOffKA = kOffV + kStages * kTileBytes;    // kStages x (2 KB + pad)
constexpr uint32_t kOffQA = kOffKA + kStages * kKAStride;    // 4 KB, written once
constexpr uint32_t kOffQCB = kOffQA + kQABytes;              // 2 x 512 B: the rows' own terms
constexpr uint32_t kOffTR = kOffQCB + 2 * kCBBytes;         // bucketed bias: key times, kStages x 512 B
constexpr uint32_t kOffQTR = kOffTR + kStages * kCBBytes;    // bucketed bias: row times, 2 x 512 B
constexpr uint32_t kOffStage = kOffQTR + 2 * kCBBytes;       // O rows staged, 16 KB
constexpr uint32_t kOffML = kOffStage + BM * DH * 2;         // (m, l) per row, 2 buffers
constexpr uint32_t kOffRec = kOffML + 2 * BM * 8;            // item record with each Q tile
constexpr uint32_t kOffBar = kOffRec + 2 * 32;               // barriers
constexpr uint32_t kNumBars = 15 + 3 * kStages;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;        // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;        // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffStage % 16 == 0 && kOffTR % 16 == 0 && kOffKA % 128 == 0 &&
                  kKAStride % 128 == 0 && kOffQA % 128 == 0,
              "aligned bulk copies and MMA operands");

// Bucketed time bias (the variant -m_p (p_i - p_j) - m_t bucket(t_i - t_j)):
//   bucket(D) = min(62, floor(4 log2(D + 1))) for a gap of D >= 0 seconds.
// floor(4 log2 x) is the binary exponent of x^4; for integer 1 <= x <= 46341 the fp32
// product fl(fl(x x) fl(x x)) has that exponent exactly (round to nearest even; checked
// exhaustively over the whole range), and floor(4 log2 46341) = 62, so capping the gap at
// 46340 saturates the bucket at 62.  The gap arrives as an int32 biased by kTimeMagic, so
// that its bits read as the float 2^23 + D + 1 (exact for D < 2^23): one subtraction
// gives x = D + 1 without a conversion instruction, and the exponent field E of x^4 ORed
// into the same pattern reads as 2^23 + E, from which the bucket E - 127 is one more
// subtraction.
constexpr int kTimeMagic = 0x4B000001;           // float bits of 2^23 + 1
constexpr int kTimeCap = kTimeMagic + 46340;      // gap cap (bucket 62)
constexpr float kTwo23 = 8388608.f;
constexpr int kMaxRelTime = 1 << 29;              // per-user times are clamped below this

// TMEM columns (the whole 512 of the SM)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // two S buffers (fp32, 128 columns each)
constexpr uint32_t kColP = 256;  // two P buffers (bf16 pairs, 64 columns each)
constexpr uint32_t kColO = 384;  // two O buffers (fp32, 64 columns each)

constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, 0, 0);   // Q K-major, K K-major

// Descriptor of a K-major operand without swizzle: core matrices of 8 rows x 16 bytes
// (rows 16 bytes apart), sbo bytes between row groups, lbo bytes between the two 8-column
// halves of a K = 16 slice.
GR_DEVICE uint64_t smem_desc_plain(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100; layout type 0: no swizzle
  return d;
}
constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, DH, 0, 1);  // P K-major (TMEM), V MN-major

// scratch layout
constexpr size_t kHeaderBytes = 256;
constexpr int kRecInts = 12;  // s, L, n, q0, nk, spad, u, kb, rb, 3 unused

struct Params {
  const int32_t* trel;  // bucketed bias: per-token time since the user's first token, [Tp]
  const __nv_bfloat16* dbias;  // dense bias: [B][Lpad][Lpad], user-local rows and columns
  long long Lpad;
  // tq: query rows; tk, tv: the history keys and values; tkc, tvc: the keys and values
  // of the query rows themselves (the diagonal tile).  For attention over one jagged
  // token array all of them cover that array and tkc, tvc equal tk, tv.
  CUtensorMap tq, tk, tv, tkc, tvc;
  AttnArgs a;
  const int4* recs;      // [count][2] work records
  const int32_t* count;  // number of records
  const float* cbias;    // [H][Tp] column terms (log2 units)
  const uint4* caug;     // [H][Tp] the same terms / (scale log2 e) as three bf16 parts
  long long Tp;
};

struct CachedArgsHolder {
  CachedAttnArgs c;
};

enum Bar {
  kQFull = 0, kQEmpty = 2, kSFull = 4, kPFull = 6, kPFree = 8, kOFull = 10, kOEmpty = 12,
  kDone = 14, kKFull = 15, kVFull = kKFull + kStages, kKVEmpty = kVFull + kStages
};
static_assert(kKVEmpty + kStages <= (int)kNumBars, "barriers");

GR_DEVICE int tiles_of(int q0, int n, int L, int nk) {
  return nk + (min(q0 + BM, L) > n ? 1 : 0);
}

// One work item: query rows [q0, q0 + 128) of a user whose sequence has L rows, the
// first n of them history.  Query row i (and the diagonal tile's key i) lives at row
// s + i of the query-side arrays; history key j at row kb + j of the key-side arrays.
// Column terms: history key j at spad + j, query row i (and diagonal key i) at rb + i;
// both spad and rb + q0 are multiples of 4 (16-byte aligned bulk copies).
struct Item {
  int s, L, n, q0, nk, spad, h, kb, u, rb;
  int nt;  // tiles visited: nk key tiles, plus the diagonal tile when candidates are present
};

GR_DEVICE Item load_item(const Params& P, int w) {
  const int pair = w / P.a.H;
  const int4 r0 = P.recs[3 * pair];
  const int4 r1 = P.recs[3 * pair + 1];
  const int4 r2 = P.recs[3 * pair + 2];
  Item it;
  it.h = w - pair * P.a.H;
  it.s = r0.x;
  it.L = r0.y;
  it.n = r0.z;
  it.q0 = r0.w;
  it.nk = r1.x;
  it.spad = r1.y;
  it.kb = r1.w;
  it.u = r1.z;
  it.rb = r2.x;
  it.nt = tiles_of(it.q0, it.n, it.L, it.nk);
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
// Candidate scoring from a cache: a user's segment holds its n history terms, padding to a
// multiple of 4, then its m candidates' terms (at most L + 3 entries), so segments start
// 8 entries apart beyond their lengths.
__host__ __device__ inline long long seg_start_cached(long long s, int u) {
  return 4 * ((s + 3) / 4) + 8LL * u;
}
__host__ __device__ inline long long scratch_tp_cached(long long T, int B) {
  return ((T + 8LL * B + 8 + BN) + 3) / 4 * 4;
}

// ------------------------------------------------------------------------------------------
// prologue: work records (block B) and column terms (blocks 0..B-1)
// ------------------------------------------------------------------------------------------
// A column term c (log2 units) as the MMA adds it: q = c / (scale log2 e) split into
// three bf16 parts (q - hi and q - hi - mid are exact in fp32, so the parts sum to q to
// within about 2^-25 of it), in the first three of the entry's eight bf16 columns.
GR_DEVICE uint4 cterm_parts(float c, float scale_log2) {
  const float q = c / scale_log2;
  const __nv_bfloat16 hi = __float2bfloat16_rn(q);
  const float r1 = q - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
  return make_uint4((uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(mid) << 16),
                    (uint32_t)__bfloat16_as_ushort(lo), 0u, 0u);
}
GR_DEVICE void put_cterm(float* cbias, uint4* caug, long long at, float c, float scale_log2) {
  cbias[at] = c;
  caug[at] = cterm_parts(c, scale_log2);
}
constexpr int kMaxTileBuckets = 257;
constexpr int kSchedThreads = 256;

// Exclusive prefix sum over the block's kSchedThreads values; returns the total.
GR_DEVICE int block_exclusive_scan(int v, int* excl, int* warp_sums) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int w = lane < kSchedThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSchedThreads / 32) warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  *excl = x - v + (wid > 0 ? warp_sums[wid - 1] : 0);
  const int total = warp_sums[kSchedThreads / 32 - 1];
  __syncthreads();
  return total;
}

// Work records go out user by user, users with the most query tiles first and each
// user's query tiles with the most key tiles first: the persistent grid takes
// consecutive records (times H heads) at the same time, so the items of one user and
// head run side by side and share their K/V tiles in L2, while the short users fill
// the tail.
// With trel != null (the bucketed time bias) the column term holds the position part
// only, and trel[i] = t_i - t_0 (clamped to [0, kMaxRelTime)) carries the time.  With
// cbias == null (a dense bias) only the records are written.
__global__ void __launch_bounds__(kSchedThreads) k_prologue(const __grid_constant__ AttnArgs a,
                                                            int max_tiles, int4* recs,
                                                            int32_t* count, int32_t* uorder,
                                                            float* cbias, uint4* caug,
                                                            int32_t* trel, long long Tp) {
  const int b = blockIdx.x;
  if (b < a.B) {
    const long long s = a.off[b], e = a.off[b + 1];
    if (s < 0 || e < s || e > a.T || !cbias) return;  // layout flagged by the schedule block
    const float sl2 = a.scale * kLog2e;
    const int L = (int)(e - s);
    const long long base = seg_start(s, b);
    const long long t0 = L > 0 ? a.ts[s] : 0;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
      const float p = (float)a.pos[s + i];
      const long long dtl = a.ts[s + i] - t0;
      if (trel) {
        trel[base + i] = (int)min(max(dtl, 0LL), (long long)kMaxRelTime - 1);
        for (int h = 0; h < a.H; ++h)
          put_cterm(cbias, caug, (long long)h * Tp + base + i, kLog2e * (a.slope_pos[h] * p), sl2);
      } else {
        const float dt = (float)dtl;
        for (int h = 0; h < a.H; ++h)
          put_cterm(cbias, caug, (long long)h * Tp + base + i,
                    kLog2e * (a.slope_pos[h] * p + a.slope_time[h] * dt), sl2);
      }
    }
    // the entries up to the next user's segment (up to the end for the last user) are
    // zeroed: a key tile reads up to 127 entries past a user's last token, and the
    // attention kernel relies on every entry it reads being finite
    const long long next = b + 1 < a.B ? seg_start(e, b + 1) : Tp;
    for (long long i = base + L + threadIdx.x; i < next; i += blockDim.x) {
      if (trel) trel[i] = 0;
      for (int h = 0; h < a.H; ++h) {
        cbias[(long long)h * Tp + i] = 0.f;
        caug[(long long)h * Tp + i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  __shared__ int hist[kMaxTileBuckets];
  __shared__ int warp_sums[kSchedThreads / 32];
  for (int i = threadIdx.x; i < kMaxTileBuckets; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  auto tiles_of_user = [&](int u, bool check) -> int {
    const long long s = a.off[u], e = a.off[u + 1];
    if (s < 0 || e < s || e > a.T) {
      if (check) flag(a.err, GENRANK_DERR_LAYOUT);
      return 0;
    }
    const int tiles_all = (int)((e - s + BM - 1) / BM);
    if (check && tiles_all > max_tiles) flag(a.err, GENRANK_DERR_LAYOUT);
    return min(tiles_all, max_tiles);
  };
  // users bucketed by query tiles, longest first
  for (int u = threadIdx.x; u < a.B; u += blockDim.x)
    atomicAdd(&hist[min(tiles_of_user(u, true), kMaxTileBuckets - 1)], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = kMaxTileBuckets - 1; q >= 0; --q) {
      const int c = hist[q];
      hist[q] = acc;
      acc += c;
    }
  }
  __syncthreads();
  for (int u = threadIdx.x; u < a.B; u += blockDim.x)
    uorder[atomicAdd(&hist[min(tiles_of_user(u, false), kMaxTileBuckets - 1)], 1)] = u;
  __syncthreads();
  // record slots: prefix sum of the ordered users' tile counts, a chunk per thread
  const int chunk = (a.B + kSchedThreads - 1) / kSchedThreads;
  const int k0 = min(a.B, (int)threadIdx.x * chunk), k1 = min(a.B, k0 + chunk);
  int mine = 0;
  for (int k = k0; k < k1; ++k) mine += tiles_of_user(uorder[k], false);
  int slot = 0;
  const int total = block_exclusive_scan(mine, &slot, warp_sums);
  for (int k = k0; k < k1; ++k) {
    const int u = uorder[k];
    const int tiles = tiles_of_user(u, false);
    if (tiles == 0) continue;
    const int s = a.off[u];
    const int L = a.off[u + 1] - s;
    const int n = max(0, min(a.hist_len[u], L));
    for (int t = tiles - 1; t >= 0; --t, ++slot) {
      const int kmax = min(t * BM + BM, n);
      const int nk = kmax > 0 ? (kmax + BN - 1) / BN : 0;
      const int seg = (int)seg_start(s, u);
      recs[3 * slot] = make_int4(s, L, n, t * BM);
      recs[3 * slot + 1] = make_int4(nk, seg, u, s);
      recs[3 * slot + 2] = make_int4(seg, 0, 0, 0);
    }
  }
  if (threadIdx.x == 0) *count = total;
}

// ------------------------------------------------------------------------------------------
// prologue of candidate scoring from a history key/value cache
// ------------------------------------------------------------------------------------------
// User u has n = hist_off[u+1] - hist_off[u] cached history rows and m candidate rows
// [off[u], off[u+1]).  Its local sequence is the history followed by the candidates, so
// the column terms and the work items are those of the full attention: candidate query
// tiles start at q0 = n + 128 t, query row i (>= n) is candidate row off[u] + i - n, and
// history key j is cache row hist_off[u] + j.  Blocks 0..B-1 write the column terms
// (history: the cached positions and times; candidates: position n + 1 and their request
// time) and check the orders the separable bias relies on; block B writes the records.
GR_DEVICE bool cached_user(const CachedAttnArgs& c, int u, int& cs, int& n, int& m, int& hs) {
  if (!c.hist_off) {  // one jagged token array: history, then candidates, per user
    const long long s = c.a.off[u], e = c.a.off[u + 1];
    if (s < 0 || e < s || e > c.a.T) return false;
    const int L = (int)(e - s);
    n = max(0, min(c.a.hist_len[u], L));
    m = L - n;
    hs = (int)s;
    cs = (int)s + n;
    return true;
  }
  const long long cs_ = c.a.off[u], ce = c.a.off[u + 1];
  const long long hs_ = c.hist_off[u], he = c.hist_off[u + 1];
  if (cs_ < 0 || ce < cs_ || ce > c.a.T || hs_ < 0 || he < hs_ || he > c.Th) return false;
  cs = (int)cs_;
  hs = (int)hs_;
  n = (int)(he - hs_);
  m = (int)(ce - cs_);
  return true;
}

__global__ void __launch_bounds__(kSchedThreads) k_prologue_cached(
    const __grid_constant__ CachedArgsHolder ch, int max_tiles, int4* recs, int32_t* count,
    int32_t* uorder, float* cbias, uint4* caug, long long Tp) {
  const CachedAttnArgs& c = ch.c;
  const AttnArgs& a = c.a;
  const int b = blockIdx.x;
  if (b < a.B) {
    const float sl2 = a.scale * kLog2e;
    int cs, n, m, hs;
    if (!cached_user(c, b, cs, n, m, hs)) return;  // flagged by the schedule block
    const int L = n + m;
    const long long base = seg_start_cached((long long)hs + cs, b);
    const int n4 = (n + 3) & ~3;  // candidates' terms start 16-byte aligned
    const long long t0 = n > 0 ? c.ts_hist[hs] : (m > 0 ? a.ts[cs] : 0);
    const long long t_last = n > 0 ? c.ts_hist[hs + n - 1] : LLONG_MIN;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
      int p;
      long long t;
      if (i < n) {
        p = c.pos_hist[hs + i];
        t = c.ts_hist[hs + i];
        if (p < 0 || p > n + 1) flag(a.err, GENRANK_DERR_POS_RANGE);
        if (i > 0 && t < c.ts_hist[hs + i - 1]) flag(a.err, GENRANK_DERR_TS_ORDER);
      } else {
        p = n + 1;
        t = a.ts[cs + i - n];
        if (t < t_last) flag(a.err, GENRANK_DERR_TS_ORDER);
      }
      const float pf = (float)p, dt = (float)(t - t0);
      const long long at = base + (i < n ? i : n4 + (i - n));
      for (int h = 0; h < a.H; ++h)
        put_cterm(cbias, caug, (long long)h * Tp + at,
                  kLog2e * (a.slope_pos[h] * pf + a.slope_time[h] * dt), sl2);
    }
    // the padding after the history and the entries up to the next user's segment (up
    // to the end for the last user) are zeroed: the attention kernel relies on every
    // column term a key tile reads being finite
    long long next = Tp;
    if (b + 1 < a.B) {
      int cs1, n1, m1, hs1;
      if (cached_user(c, b + 1, cs1, n1, m1, hs1)) next = seg_start_cached((long long)hs1 + cs1, b + 1);
    }
    for (long long i = base + n + threadIdx.x; i < next; i += blockDim.x) {
      if (i >= base + n4 && i < base + n4 + m) continue;
      for (int h = 0; h < a.H; ++h) {
        cbias[(long long)h * Tp + i] = 0.f;
        caug[(long long)h * Tp + i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  __shared__ int hist[kMaxTileBuckets];
  __shared__ int warp_sums[kSchedThreads / 32];
  for (int i = threadIdx.x; i < kMaxTileBuckets; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  auto tiles_of_user = [&](int u, bool check) -> int {
    int cs, n, m, hs;
    if (!cached_user(c, u, cs, n, m, hs)) {
      if (check) flag(a.err, GENRANK_DERR_LAYOUT);
      return 0;
    }
    const int tiles_all = (m + BM - 1) / BM;
    if (check && tiles_all > max_tiles) flag(a.err, GENRANK_DERR_LAYOUT);
    return min(tiles_all, max_tiles);
  };
  for (int u = threadIdx.x; u < a.B; u += blockDim.x)
    atomicAdd(&hist[min(tiles_of_user(u, true), kMaxTileBuckets - 1)], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = kMaxTileBuckets - 1; q >= 0; --q) {
      const int cnt = hist[q];
      hist[q] = acc;
      acc += cnt;
    }
  }
  __syncthreads();
  for (int u = threadIdx.x; u < a.B; u += blockDim.x)
    uorder[atomicAdd(&hist[min(tiles_of_user(u, false), kMaxTileBuckets - 1)], 1)] = u;
  __syncthreads();
  const int chunk = (a.B + kSchedThreads - 1) / kSchedThreads;
  const int k0 = min(a.B, (int)threadIdx.x * chunk), k1 = min(a.B, k0 + chunk);
  int mine = 0;
  for (int k = k0; k < k1; ++k) mine += tiles_of_user(uorder[k], false);
  int slot = 0;
  const int total = block_exclusive_scan(mine, &slot, warp_sums);
  for (int k = k0; k < k1; ++k) {
    const int u = uorder[k];
    const int tiles = tiles_of_user(u, false);
    if (tiles == 0) continue;
    int cs, n, m, hs;
    cached_user(c, u, cs, n, m, hs);
    const int nk = (n + BN - 1) / BN;
    const int seg = (int)seg_start_cached((long long)hs + cs, u);
    const int n4 = (n + 3) & ~3;
    for (int t = tiles - 1; t >= 0; --t, ++slot) {
      recs[3 * slot] = make_int4(cs - n, n + m, n, n + t * BM);
      recs[3 * slot + 1] = make_int4(nk, seg, u, hs);
      recs[3 * slot + 2] = make_int4(seg + n4 - n, 0, 0, 0);  // rb: rb + q0 = seg + n4 + 128 t
    }
  }
  if (threadIdx.x == 0) *count = total;
}

// ------------------------------------------------------------------------------------------
// the attention kernel
// ------------------------------------------------------------------------------------------
GR_DEVICE uint32_t par(int use) { return (uint32_t)(use & 1); }

// Every lane waits (bounded), then the warp agrees, so that the warp stays
// converged for the .sync.aligned tcgen05 instructions that follow.
// A phase that has completed already (the usual case in the tile loop) is seen by a
// non-blocking test; only a phase still open goes through the bounded wait.
GR_DEVICE bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
GR_DEVICE bool wait_warp(uint64_t* bar, uint32_t ph, volatile int* abort_flag, int32_t* err) {
  const bool ok = mbar_test(bar, ph) || mbar_wait(bar, ph, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

// Each softmax thread owns one half of a query row: key columns [64 h, 64 h + 64) of
// every tile (h = lane / 16), reached with the 16x32bx2 TMEM shape: S columns at
// offset 64, packed P columns at offset 32, O columns at offset 32.
constexpr int kHalf = BN / 2;
constexpr int CW = 16;  // key columns per chunk (of the thread's 64)
GR_DEVICE void s_load(uint32_t taddr, uint32_t (&r)[CW]) { tmem_ld_half16_async<kHalf>(taddr, r); }
template <int kOff = kHalf / 2>
GR_DEVICE void p_store(uint32_t taddr, const uint32_t (&pk)[CW / 2]) {
  tmem_st_half8_nowait<kOff>(taddr, pk);
}
// A masked tile can instead interleave the halves by 16-key chunks: threads 0-15 take
// the even chunks, threads 16-31 the odd ones, so that the two halves of a warp agree
// on which chunks a row's mask leaves visible or hides (but for the chunk it cuts).
GR_DEVICE void s_load_il(uint32_t taddr, uint32_t (&r)[CW]) { tmem_ld_half16_async<CW>(taddr, r); }

// The bucketed time bias of one softmax thread: the key times of its columns (shared
// memory, indexed like the column terms), its row's time + kTimeMagic, and -m_t log2 e
// of the item's head.  Unused (and compiled out) for the linear time bias.
struct TB {
  const int* tr;
  int ti_m;
  float nmt2;
  GR_DEVICE TB at(int off) const { return TB{tr + off, ti_m, nmt2}; }
};

// The dense bias of one softmax thread's 64 key columns: the first 32 columns' bf16
// pairs, loaded before the wait for S (which also brings the row's 128-byte line into
// L1), and the row in global memory, from which the other 32 columns are loaded when
// that half of the tile starts.  Keeping 16 words live instead of 32 avoids spilling.
struct DB {
  const uint32_t* w0;
  const uint4* src;
};

GR_DEVICE void load_bias16(const uint4* src, uint32_t (&w)[16]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = __ldg(src + c);
    w[4 * c] = v.x;
    w[4 * c + 1] = v.y;
    w[4 * c + 2] = v.z;
    w[4 * c + 3] = v.w;
  }
}

// bucket(t_i - t_j) of four consecutive keys, as two pairs of floats (see kTimeMagic).
GR_DEVICE void buckets4(const TB& tb, int c, uint64_t& b01, uint64_t& b23) {
  const int4 t = *reinterpret_cast<const int4*>(tb.tr + c);
  const uint64_t two23 = f2_pack(kTwo23, kTwo23);
  const uint64_t x01 = f2_sub(f2_pack(__int_as_float(min(tb.ti_m - t.x, kTimeCap)),
                                      __int_as_float(min(tb.ti_m - t.y, kTimeCap))), two23);
  const uint64_t x23 = f2_sub(f2_pack(__int_as_float(min(tb.ti_m - t.z, kTimeCap)),
                                      __int_as_float(min(tb.ti_m - t.w, kTimeCap))), two23);
  const uint64_t sq01 = f2_mul(x01, x01), sq23 = f2_mul(x23, x23);
  float q[4];
  f2_unpack(f2_mul(sq01, sq01), q[0], q[1]);
  f2_unpack(f2_mul(sq23, sq23), q[2], q[3]);
  float e[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) e[k] = __int_as_float((__float_as_int(q[k]) >> 23) | 0x4B000000);
  const uint64_t base = f2_pack(kTwo23 + 127.f, kTwo23 + 127.f);
  b01 = f2_sub(f2_pack(e[0], e[1]), base);
  b23 = f2_sub(f2_pack(e[2], e[3]), base);
}

// x = s * scale log2 e (- m_t bucket for the bucketed bias; s holds c_j already) for CW
// columns (key kc0 + c of the tile); keys at or beyond nvalid are masked.  Four independent running maxima
// shorten the chain.
template <bool kMasked, bool kBucket, bool kDense>
GR_DEVICE void row_max_chunk(const uint32_t (&s)[CW], const TB& tb,
                             const uint32_t* bw, int kc0, int nvalid, float scale_log2,
                             float (&mx4)[4]) {
#pragma unroll
  for (int c = 0; c < CW; c += 4) {
    float bb[4];
    if (kDense) {  // the dense bias of these keys, bf16 pairs
      bb[0] = kLog2e * bf16_lo(bw[c / 2]);
      bb[1] = kLog2e * bf16_hi(bw[c / 2]);
      bb[2] = kLog2e * bf16_lo(bw[c / 2 + 1]);
      bb[3] = kLog2e * bf16_hi(bw[c / 2 + 1]);
    } else {  // the column term is in s already
      bb[0] = bb[1] = bb[2] = bb[3] = 0.f;
    }
    if (kBucket) {
      uint64_t b01, b23;
      buckets4(tb, c, b01, b23);
      float k[4];
      f2_unpack(b01, k[0], k[1]);
      f2_unpack(b23, k[2], k[3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) bb[e] = fmaf(k[e], tb.nmt2, bb[e]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = fmaf(__uint_as_float(s[c + e]), scale_log2, bb[e]);
      mx4[e] = fmaxf(mx4[e], (!kMasked || kc0 + c + e < nvalid) ? v : -INFINITY);
    }
  }
}

// p = 2^(x - m) for CW columns, summed into two pairs of partial sums and packed to
// bf16 pairs in pk.  The bias and scale arithmetic runs on column pairs (two-wide fp32
// instructions).
template <bool kMasked, bool kBucket, bool kDense>
GR_DEVICE void exp_pack(const uint32_t (&s)[CW], const TB& tb,
                        const uint32_t* bw, int kc0, int nvalid, float scale_log2, float m_use,
                        uint64_t (&rs2)[2], uint32_t (&pk)[CW / 2]) {
  const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
  for (int c = 0; c < CW; c += 4) {
    uint64_t t01, t23;
    if (kDense) {  // bias log2 e - m, from the bf16 pairs of the dense bias
      const uint64_t l2e = f2_pack(kLog2e, kLog2e), nm2 = f2_pack(-m_use, -m_use);
      t01 = f2_fma(f2_pack(bf16_lo(bw[c / 2]), bf16_hi(bw[c / 2])), l2e, nm2);
      t23 = f2_fma(f2_pack(bf16_lo(bw[c / 2 + 1]), bf16_hi(bw[c / 2 + 1])), l2e, nm2);
    } else {  // the column term is in s already
      t01 = f2_pack(-m_use, -m_use);
      t23 = t01;
    }
    if (kBucket) {
      uint64_t b01, b23;
      buckets4(tb, c, b01, b23);
      const uint64_t nm2 = f2_pack(tb.nmt2, tb.nmt2);
      t01 = f2_fma(b01, nm2, t01);
      t23 = f2_fma(b23, nm2, t23);
    }
    const uint64_t v01 =
        f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2, t01);
    const uint64_t v23 =
        f2_fma(f2_pack(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])), sl2, t23);
    float v[4], p[4];
    f2_unpack(v01, v[0], v[1]);
    f2_unpack(v23, v[2], v[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = (!kMasked || kc0 + c + e < nvalid) ? ex2(v[e]) : 0.f;
    rs2[0] = f2_add(rs2[0], f2_pack(p[0], p[1]));
    rs2[1] = f2_add(rs2[1], f2_pack(p[2], p[3]));
    pk[c / 2] = pack_bf16(p[0], p[1]);
    pk[c / 2 + 1] = pack_bf16(p[2], p[3]);
  }
}

// One chunk of P: computed, then stored (without waiting) to CW / 2 TMEM columns at
// taddr.  A masked tile's chunk is, for each thread, wholly visible (the plain code),
// wholly masked (zeros, no exponentials) or the one chunk the row's mask cuts: there
// the masked keys' scores become -inf, so that 2^(x - m) = +0 for them (their column
// terms are finite: the prologue writes every entry a key tile can read).  The dense
// form keeps a select per key (its bias rows past a user's end are the caller's).  The
// branches only compute, so the warp is converged again for the store.
template <bool kMasked, bool kBucket, bool kDense, int kPOff = kHalf / 2>
GR_DEVICE void exp_pack_store(uint32_t (&s)[CW], const TB& tb,
                              const uint32_t* bw, int kc0, int nvalid, float scale_log2,
                              float m_use, uint64_t (&rs2)[2], uint32_t taddr) {
  uint32_t pk[CW / 2];
  if (kDense || !kMasked) {
    exp_pack<kMasked, kBucket, kDense>(s, tb, bw, kc0, nvalid, scale_log2, m_use, rs2, pk);
  } else if (kc0 >= nvalid) {
#pragma unroll
    for (int k = 0; k < CW / 2; ++k) pk[k] = 0u;
  } else {
    if (kc0 + CW > nvalid) {
#pragma unroll
      for (int e = 0; e < CW; ++e)
        if (kc0 + e >= nvalid) s[e] = 0xff800000u;  // -inf
    }
    exp_pack<false, kBucket, kDense>(s, tb, bw, kc0, nvalid, scale_log2, m_use, rs2, pk);
  }
  p_store<kPOff>(taddr, pk);
}

// Maximum of x over this thread's half of the tile (S at s_addr, first key kbase), CW
// columns at a time with the next chunk's load in flight.
template <bool kMasked, bool kBucket, bool kDense>
GR_DEVICE float tile_max(uint32_t s_addr, const TB& tb, const DB& db,
                         int kbase, int nvalid, float scale_log2) {
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  uint32_t xa[CW], xb[CW];
  uint32_t w1[kDense ? 16 : 1];
  s_load(s_addr, xa);
  tmem_ld_wait(xa);
#pragma unroll
  for (int c0 = 0; c0 < kHalf; c0 += 2 * CW) {
    const uint32_t* bw = nullptr;
    if constexpr (kDense) {
      if (c0 == 0) {
        bw = db.w0;
      } else {
        load_bias16(db.src + 4, w1);
        bw = w1;
      }
    }
    s_load(s_addr + c0 + CW, xb);
    row_max_chunk<kMasked, kBucket, kDense>(xa, tb.at(c0), bw, kbase + c0, nvalid,
                                            scale_log2, mx4);
    tmem_ld_wait(xb);
    if (c0 + 2 * CW < kHalf) s_load(s_addr + c0 + 2 * CW, xa);
    row_max_chunk<kMasked, kBucket, kDense>(xb, tb.at(c0 + CW),
                                            kDense ? bw + CW / 2 : bw, kbase + c0 + CW, nvalid,
                                            scale_log2, mx4);
    if (c0 + 2 * CW < kHalf) tmem_ld_wait(xa);
  }
  return fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
}

// P = 2^(x - m) for this thread's half of the tile, written as bf16 pairs to the P
// columns at p_addr; the stores have landed when it returns.  Returns the half's sum.
template <bool kMasked, bool kBucket, bool kDense>
GR_DEVICE float tile_exp(uint32_t s_addr, uint32_t p_addr, const TB& tb,
                         const DB& db, int kbase, int nvalid, float scale_log2, float m) {
  uint64_t rs2[2] = {0ull, 0ull};  // (+0, +0) pairs
  uint32_t xa[CW], xb[CW];
  if constexpr (kMasked && !kDense) {
    // the halves interleaved by chunks (see s_load_il); P lands in the same columns
    const int hh = kbase / kHalf;
    const TB tbr = tb.at(-kbase);
    s_load_il(s_addr, xa);
    tmem_ld_wait(xa);
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      s_load_il(s_addr + 2 * CW * (k + 1), xb);
      const int ka = 2 * CW * k + CW * hh;
      exp_pack_store<true, kBucket, false, CW / 2>(xa, tbr.at(ka), nullptr, ka, nvalid,
                                                   scale_log2, m, rs2, p_addr + CW * k);
      tmem_ld_wait(xb);
      if (k + 2 < 4) s_load_il(s_addr + 2 * CW * (k + 2), xa);
      const int kb = 2 * CW * (k + 1) + CW * hh;
      exp_pack_store<true, kBucket, false, CW / 2>(xb, tbr.at(kb), nullptr, kb, nvalid,
                                                   scale_log2, m, rs2, p_addr + CW * (k + 1));
      if (k + 2 < 4) tmem_ld_wait(xa);
    }
    tmem_wait_st();
    float r0, r1, r2, r3;
    f2_unpack(rs2[0], r0, r1);
    f2_unpack(rs2[1], r2, r3);
    return (r0 + r1) + (r2 + r3);
  }
  uint32_t w1[kDense ? 16 : 1];
  s_load(s_addr, xa);
  tmem_ld_wait(xa);
#pragma unroll
  for (int c0 = 0; c0 < kHalf; c0 += 2 * CW) {
    const uint32_t* bw = nullptr;
    if constexpr (kDense) {
      if (c0 == 0) {
        bw = db.w0;
      } else {
        load_bias16(db.src + 4, w1);
        bw = w1;
      }
    }
    s_load(s_addr + c0 + CW, xb);
    exp_pack_store<kMasked, kBucket, kDense>(xa, tb.at(c0), bw, kbase + c0, nvalid,
                                             scale_log2, m, rs2, p_addr + c0 / 2);
    tmem_ld_wait(xb);
    if (c0 + 2 * CW < kHalf) s_load(s_addr + c0 + 2 * CW, xa);
    exp_pack_store<kMasked, kBucket, kDense>(xb, tb.at(c0 + CW),
                                             kDense ? bw + CW / 2 : bw, kbase + c0 + CW, nvalid,
                                             scale_log2, m, rs2, p_addr + (c0 + CW) / 2);
    if (c0 + 2 * CW < kHalf) tmem_ld_wait(xa);
  }
  tmem_wait_st();
  float r0, r1, r2, r3;
  f2_unpack(rs2[0], r0, r1);
  f2_unpack(rs2[1], r2, r3);
  return (r0 + r1) + (r2 + r3);
}

// O (this thread's 32 columns of its row) *= alpha, once the previous P V has landed.
GR_DEVICE bool rescale_o(uint32_t o_addr, float alpha, uint64_t* prev_pv, uint32_t prev_ph,
                         volatile int* abort_flag, int32_t* err) {
  if (!wait_warp(prev_pv, prev_ph, abort_flag, err)) return false;
  tc_fence_after();
  uint32_t o[32];
  tmem_ld_half32_async<DH / 2>(o_addr, o);
  tmem_ld_wait(o);
#pragma unroll
  for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
  tmem_st_half32_nowait<DH / 2>(o_addr, o);
  tmem_wait_st();
  return true;
}

// One history key tile of the online softmax for this thread's half row.  The offset
// m starts at the row's own column term c_i: every visible key has c_j <= c_i, so
// 2^(x - m) <= 2^(scale q.k log2 e), which overflows only for extreme scores.  Each
// tile is one pass; a tile whose row sum leaves [2^-100, 2^100] on the first tile
// (every key far below the offset) or exceeds 2^100 later is redone with the exact
// offset max(m, tile max), rescaling O in TMEM.  Rows past the user's end never
// redo (their output is not written).
template <bool kMasked, bool kBucket, bool kDense>
GR_DEVICE bool softmax_tile(uint32_t s_addr, uint32_t p_addr, uint32_t o_addr,
                            const TB& tb, const DB& bw, int kbase, int nvalid,
                            float scale_log2, bool first, bool row_ok, float& m, float& l,
                            uint64_t* prev_pv, uint32_t prev_ph, volatile int* abort_flag,
                            int32_t* err) {
  float rs = tile_exp<kMasked, kBucket, kDense>(s_addr, p_addr, tb, bw, kbase, nvalid,
                                                scale_log2, m);
  const float rs_row = rs + __shfl_xor_sync(0xffffffffu, rs, 16);
  const bool redo = row_ok && (!(rs_row <= kOverflowSum) || (first && rs_row < kUnderflowSum));
  if (__any_sync(0xffffffffu, redo)) {
    // every lane takes part in the .sync.aligned TMEM accesses; only redo rows move m
    float mx = tile_max<kMasked, kBucket, kDense>(s_addr, tb, bw, kbase, nvalid, scale_log2);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = redo ? (first ? mx : fmaxf(m, mx)) : m;
    const float alpha = first ? 1.f : ex2(m - m_new);
    m = m_new;
    if (!first && !rescale_o(o_addr, alpha, prev_pv, prev_ph, abort_flag, err)) return false;
    l *= alpha;
    rs = tile_exp<kMasked, kBucket, kDense>(s_addr, p_addr, tb, bw, kbase, nvalid,
                                            scale_log2, m);
  }
  l = first ? rs : l + rs;
  return true;
}

// The diagonal tile: S = Q K^T over the item's own rows, of which a candidate row
// keeps only its own key (position and time differences 0, so the bias is 0: its S
// holds c_i, and the score is relative to the offset).  A warp's 16 rows have their own keys in one 16-key chunk
// of one half of the tile, so only that chunk is read (by the threads of that half) and
// P is zero elsewhere.  The offset moves (O rescaled) only if the term would overflow,
// or is set exactly on a first tile.
GR_DEVICE bool softmax_diag(uint32_t s_addr, uint32_t p_addr, uint32_t o_addr, int rt, int h,
                            bool cand_row, float scale_log2, bool first, float& m,
                            float& l, uint64_t* prev_pv, uint32_t prev_ph,
                            volatile int* abort_flag, int32_t* err, float diagb = 0.f) {
  const int r0 = rt & ~15;  // the warp's first row
  const int c0 = r0 & (kHalf - 1);  // their own keys: columns [r0, r0 + 16), in half r0 / 64
  uint32_t x[16];
  tmem_ld_half16_async<kHalf>(s_addr + c0, x);
  tmem_ld_wait(x);
  const bool mine = cand_row && h == r0 / kHalf;
  const int e = rt & 15;
  float sv = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) sv = e == c ? __uint_as_float(x[c]) : sv;
  const float xm = mine ? fmaf(sv, scale_log2, diagb) : -INFINITY;
  const float xr = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, 16));  // the row's self score
  const bool move = xr > -INFINITY && (first || xr - m > 100.f);
  if (!first && __any_sync(0xffffffffu, move)) {
    const float alpha = move ? ex2(m - xr) : 1.f;
    if (!rescale_o(o_addr, alpha, prev_pv, prev_ph, abort_flag, err)) return false;
    l *= alpha;
  }
  if (move) m = xr;
  const float p = mine ? ex2(xm - m) : 0.f;
  const uint32_t word = (e & 1) ? pack_bf16(0.f, p) : pack_bf16(p, 0.f);
  uint32_t pk[8], zero[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    pk[k] = (mine && k == (e >> 1)) ? word : 0u;
    zero[k] = 0u;
  }
  // the half's 32 P columns in four stores of 8: the own-key chunk, zeros elsewhere
  // (c0 is the same for the whole warp, so the branch does not diverge)
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (k * 16 == c0)
      tmem_st_half8_nowait<kHalf / 2>(p_addr + 8 * k, pk);
    else
      tmem_st_half8_nowait<kHalf / 2>(p_addr + 8 * k, zero);
  }
  tmem_wait_st();
  l = first ? p : l + p;
  return true;
}

struct Cursor {  // one key tile in the CTA's sequence: tile j of the qi-th item, g overall
  int j, g, qi, nt;
};

template <bool kBucket, bool kDense>
__global__ void __launch_bounds__(kThreads, 1) k_attn_fwd_tc(const __grid_constant__ Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnArgs& a = P.a;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float2* sML = reinterpret_cast<float2*>(smem + kOffML);  // [2][BM]: (m - c_i, l)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the query side of the column-term MMA (rows 1, 1, 1, 0, ..., then 2 KB of zeros) and
  // the pads after the key-side stages, read by the MMAs through the async proxy
  if (!kDense) {
    uint4* qa = reinterpret_cast<uint4*>(smem + kOffQA);
    for (int i = threadIdx.x; i < (int)(kQABytes / 16); i += kThreads)
      qa[i] = i < BM ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < kStages * 8; i += kThreads)
      *reinterpret_cast<uint4*>(smem + kOffKA + (i >> 3) * kKAStride + kKABytes + (i & 7) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[kQFull + b], 1);
      mbar_init(&bars[kQEmpty + b], 1 + kSoftmaxWarps);  // last S commit + c_i reads
      mbar_init(&bars[kSFull + b], 1);
      mbar_init(&bars[kPFull + b], kSoftmaxWarps);
      mbar_init(&bars[kPFree + b], 1);
      mbar_init(&bars[kOFull + b], 1 + kSoftmaxWarps);  // last P V commit + (m, l)
      mbar_init(&bars[kOEmpty + b], 4);
    }
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&bars[kKFull + st], 1);
      mbar_init(&bars[kVFull + st], 1);
      mbar_init(&bars[kKVEmpty + st], 1);
    }
    mbar_init(&bars[kDone], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&P.tq);
    tma_prefetch_desc(&P.tk);
    tma_prefetch_desc(&P.tv);
    tma_prefetch_desc(&P.tkc);
    tma_prefetch_desc(&P.tvc);
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
  const float scale_log2 = a.scale * kLog2e;

  if (warp == 1) {
    // ---------------------------------------------------------------- TMA producer
    // Each Q tile travels with the item's record (q0, n, L, nk); a record with nk < 0
    // after the last item tells the MMA and softmax warps to stop.
    int4* sRec = reinterpret_cast<int4*>(smem + kOffRec);
    int qi = 0, g = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        ok = false;
        break;
      }
      const Item it = load_item(P, w);
      if (it.nt == 0) continue;
      const int qb = qi & 1;
      if (!wait_warp(&bars[kQEmpty + qb], par(qi >> 1) ^ 1u, abort_flag, a.err)) {
        ok = false;
        break;
      }
      const float* cbr_src = P.cbias + (long long)it.h * P.Tp + it.rb;  // query rows' c_i
      const uint4* ka_src = P.caug + (long long)it.h * P.Tp + it.spad;  // history keys
      const uint4* kar_src = P.caug + (long long)it.h * P.Tp + it.rb;   // the rows as keys
      const int32_t* tr_src = kBucket ? P.trel + it.spad : nullptr;
      if (lane == 0) {
        sRec[2 * qb] = make_int4(it.q0, it.n, it.L, it.nk);
        sRec[2 * qb + 1] = make_int4(it.h, it.u, 0, 0);
        mbar_expect_tx(&bars[kQFull + qb],
                       kTileBytes + (kDense ? 0 : (kBucket ? 2 : 1) * kCBBytes));
        tma_load_3d(smem + kOffQ + qb * kTileBytes, &P.tq, &bars[kQFull + qb], 0, it.h,
                    it.s + it.q0);
        if (!kDense)
          bulk_load(smem + kOffQCB + qb * kCBBytes, cbr_src + it.q0, kCBBytes, &bars[kQFull + qb]);
        if (kBucket)
          bulk_load(smem + kOffQTR + qb * kCBBytes, tr_src + it.q0, kCBBytes, &bars[kQFull + qb]);
      }
      ++qi;
      for (int j = 0; j < it.nt; ++j) {
        const int st = g % kStages;
        if (!wait_warp(&bars[kKVEmpty + st], par(g / kStages) ^ 1u, abort_flag, a.err)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          // history key tiles most recent first, then the item's own rows
          const bool hist = j < it.nk;
          const int kv0 = hist ? (it.nk - 1 - j) * BN : it.q0;
          const int row = hist ? it.kb + kv0 : it.s + kv0;
          mbar_expect_tx(&bars[kKFull + st],
                         kTileBytes + (kDense ? 0 : kKABytes) + (kBucket ? kCBBytes : 0));
          tma_load_3d(smem + kOffK + st * kTileBytes, hist ? &P.tk : &P.tkc, &bars[kKFull + st],
                      0, it.h, row);
          if (!kDense)
            bulk_load(smem + kOffKA + st * kKAStride, hist ? ka_src + kv0 : kar_src + kv0,
                      kKABytes, &bars[kKFull + st]);
          if (kBucket)
            bulk_load(smem + kOffTR + st * kCBBytes, tr_src + kv0, kCBBytes, &bars[kKFull + st]);
          mbar_expect_tx(&bars[kVFull + st], kTileBytes);
          tma_load_3d(smem + kOffV + st * kTileBytes, hist ? &P.tv : &P.tvc, &bars[kVFull + st],
                      0, it.h, row);
        }
        ++g;
      }
    }
    if (ok && wait_warp(&bars[kQEmpty + (qi & 1)], par(qi >> 1) ^ 1u, abort_flag, a.err)) {
      if (lane == 0) {
        sRec[2 * (qi & 1)] = make_int4(0, 0, 0, -1);
        mbar_arrive(&bars[kQFull + (qi & 1)]);
      }
      ++qi;
    }
    // on the way out, the copies issued last land before the CTA exits
    if (lane == 0) {
      for (int x = max(0, g - kStages); x < g; ++x) {
        mbar_drain(&bars[kKFull + x % kStages], par(x / kStages));
        mbar_drain(&bars[kVFull + x % kStages], par(x / kStages));
      }
      for (int x = max(0, qi - 2); x < qi; ++x) mbar_drain(&bars[kQFull + (x & 1)], par(x >> 1));
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- MMA issuer (one thread)
    // Tiles in order g = 0, 1, ...: S_{g+1} = Q K_{g+1}^T goes into the other S buffer
    // before P_g V_g, so the softmax finds each S ready when it finishes the last one.
    if (lane == 0) {
      const uint32_t sQ = smem_u32(smem + kOffQ), sK = smem_u32(smem + kOffK),
                     sV = smem_u32(smem + kOffV), sQA = smem_u32(smem + kOffQA),
                     sKA = smem_u32(smem + kOffKA);
      const int4* sRec = reinterpret_cast<const int4*>(smem + kOffRec);
      // number of tiles of the qi-th item (its Q tile has landed), or -1 at the end
      auto tiles = [&](int qi) -> int {
        if (!mbar_wait(&bars[kQFull + (qi & 1)], par(qi >> 1), abort_flag, a.err)) return -1;
        const int4 r = sRec[2 * (qi & 1)];
        return r.w < 0 ? -1 : tiles_of(r.x, r.y, r.z, r.w);
      };
      auto issue_s = [&](const Cursor& t) -> bool {
        const int sb = t.g & 1, st = t.g % kStages, qb = t.qi & 1;
        // the S buffer is free once the softmax has handed over the P it computed from it
        if (!mbar_wait(&bars[kPFull + sb], par(t.g >> 1) ^ 1u, abort_flag, a.err)) return false;
        if (!mbar_wait(&bars[kKFull + st], par(t.g / kStages), abort_flag, a.err)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(sQ + qb * kTileBytes + k * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + st * kTileBytes + k * 32, 16, 1024);
          mma_bf16_ss(tmem + kColS + sb * BN, ad, bd, kIdescS, k > 0 ? 1u : 0u);
        }
        if (!kDense) {  // + c_j / (scale log2 e): the query side's second 8 columns are zero
          const uint64_t ad = smem_desc_plain(sQA, kQABytes / 2, 128);
          const uint64_t bd = smem_desc_plain(sKA + st * kKAStride, 16, 128);
          mma_bf16_ss(tmem + kColS + sb * BN, ad, bd, kIdescS, 1u);
        }
        mma_commit(&bars[kSFull + sb]);
        if (t.j == t.nt - 1) mma_commit(&bars[kQEmpty + qb]);
        return true;
      };
      auto issue_pv = [&](const Cursor& t) -> bool {
        const int pb = t.g & 1, st = t.g % kStages, ob = t.qi & 1;
        if (!mbar_wait(&bars[kPFull + pb], par(t.g >> 1), abort_flag, a.err)) return false;
        if (!mbar_wait(&bars[kVFull + st], par(t.g / kStages), abort_flag, a.err)) return false;
        if (t.j == 0 && !mbar_wait(&bars[kOEmpty + ob], par(t.qi >> 1) ^ 1u, abort_flag, a.err))
          return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t bd =
              smem_desc_sw128(sV + st * kTileBytes + k * 16 * 128, kTileBytes, 1024);
          mma_bf16_ts(tmem + kColO + ob * DH, tmem + kColP + pb * (BN / 2) + k * 8, bd, kIdescPV,
                      (t.j > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&bars[kPFree + pb]);
        mma_commit(&bars[kKVEmpty + st]);
        if (t.j == t.nt - 1) mma_commit(&bars[kOFull + ob]);
        return true;
      };
      Cursor c{0, 0, 0, tiles(0)};
      bool ok = c.nt > 0 && issue_s(c);
      while (ok) {
        Cursor n = c;
        ++n.g;
        if (++n.j == c.nt) {
          n.j = 0;
          ++n.qi;
          n.nt = tiles(n.qi);
        }
        const bool more = n.nt > 0;
        if (more && !issue_s(n)) break;
        if (!issue_pv(c) || !more) break;
        c = n;
      }
      // every MMA issued has completed before TMEM is freed
      mma_commit(&bars[kDone]);
      mbar_drain(&bars[kDone], 0);
    }
    __syncwarp();
  } else if (warp < 10) {
    // ---------------------------------------------------------------- softmax warps 2-9
    const int quad = warp & 3;  // TMEM lane quadrant of the warp
    const int rh = (warp - 2) >> 2;  // upper or lower 16 lanes of the quadrant
    const int h = lane >> 4;    // key-column half of each tile
    const int rt = quad * 32 + rh * 16 + (lane & 15);  // query row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32 + rh * 16) << 16);
    const float* sQCB = reinterpret_cast<const float*>(smem + kOffQCB);
    const int* sQTR = reinterpret_cast<const int*>(smem + kOffQTR);
    const int* sTR = reinterpret_cast<const int*>(smem + kOffTR);
    const int4* sRec = reinterpret_cast<const int4*>(smem + kOffRec);
    int g = 0;
    for (int oi = 0;; ++oi) {
      const int ob = oi & 1;
      // the item's record and the row's own column term c_i arrive with the Q tile
      if (!wait_warp(&bars[kQFull + ob], par(oi >> 1), abort_flag, a.err)) break;
      const int4 rec = sRec[2 * ob];
      if (rec.w < 0) break;
      Item it;
      it.q0 = rec.x;
      it.n = rec.y;
      it.L = rec.z;
      it.nk = rec.w;
      it.nt = tiles_of(it.q0, it.n, it.L, it.nk);
      // the fixed offset starts at the row's own column term; a dense bias has no such
      // bound, so its offset starts at 0 and the redo path moves it when needed
      const float rowcb = kDense ? 0.f : sQCB[ob * BM + rt];
      const __nv_bfloat16* brow = nullptr;  // dense bias: this thread's row of the user's block
      if (kDense)
        brow = P.dbias + ((long long)sRec[2 * ob + 1].y * P.Lpad + it.q0 + rt) * P.Lpad + kHalf * h;
      TB tb{nullptr, 0, 0.f};
      if (kBucket) {
        const int hh = sRec[2 * ob + 1].x;
        tb.ti_m = sQTR[ob * BM + rt] + kTimeMagic;
        tb.nmt2 = -a.slope_time[hh] * kLog2e;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kQEmpty + ob]);
      const int i = it.q0 + rt;
      const bool row_ok = i < it.L;
      const bool cand_row = row_ok && i >= it.n;
      const int lim = min(i, it.n - 1);
      const int mask_from = min(it.q0, it.n - 1);  // a tile needs masks if kv0 + 127 > this
      const uint32_t o_addr = lane_base + kColO + ob * DH;
      float m = rowcb, l = 0.f;
      bool ok = true;
      // One key tile: the per-row mask can only reach the first tile an item visits
      // (its diagonal history tile, or the last, partial history tile of a candidate
      // tile), so that tile runs the masked form and every later one the plain form;
      // the plain loop then holds a single copy of the tile code.
      auto step = [&](int j, auto masked_form) -> bool {
        constexpr bool kM = decltype(masked_form)::value;
        const int sb = g & 1, st = g % kStages;
        // dense bias: this thread's 64 values of the tile (one 128-byte line), requested
        // before the wait for S so that the load overlaps it
        uint32_t bw0[kDense ? 16 : 1];
        DB bw{bw0, nullptr};
        float diagb = 0.f;
        if constexpr (kDense) {
          if (j < it.nk) {
            bw.src = reinterpret_cast<const uint4*>(brow + (it.nk - 1 - j) * BN);
            load_bias16(bw.src, bw0);
          } else {  // the diagonal tile: the row's own entry
            diagb = kLog2e * __bfloat162float(brow[it.q0 + rt - kHalf * h]);
          }
        }
        // S_g's commit also covers every MMA issued before it, P_{g-2} V_{g-2} included,
        // so once S_g is here its P buffer is free as well; only the bucketed bias reads
        // the key stage itself (the key times)
        if (!wait_warp(&bars[kSFull + sb], par(g >> 1), abort_flag, a.err) ||
            (kBucket && !wait_warp(&bars[kKFull + st], par(g / kStages), abort_flag, a.err)))
          return false;
        tc_fence_after();
        const uint32_t s_addr = lane_base + kColS + sb * BN;
        const uint32_t p_addr = lane_base + kColP + sb * (BN / 2);
        uint64_t* prev_pv = &bars[kPFree + ((g + 1) & 1)];
        const uint32_t prev_ph = par((g - 1) >> 1);
        bool done;
        if (j < it.nk) {
          const int kv0 = (it.nk - 1 - j) * BN;  // most recent keys first
          if (kBucket) tb.tr = sTR + st * BN + kHalf * h;
          if constexpr (kM) {
            // keys past the row's last visible key are masked (none on an unmasked tile)
            const int nvalid = max(0, min(BN, lim - kv0 + 1));
            done = softmax_tile<true, kBucket, kDense>(
                s_addr, p_addr, o_addr, tb, bw, kHalf * h, nvalid, scale_log2, j == 0,
                row_ok, m, l, prev_pv, prev_ph, abort_flag, a.err);
          } else {
            if (kv0 + BN - 1 > mask_from) flag(a.err, GENRANK_DERR_LAYOUT);  // not reachable
            done = softmax_tile<false, kBucket, kDense>(
                s_addr, p_addr, o_addr, tb, bw, kHalf * h, BN, scale_log2, j == 0,
                row_ok, m, l, prev_pv, prev_ph, abort_flag, a.err);
          }
        } else {
          done = softmax_diag(s_addr, p_addr, o_addr, rt, h, cand_row, scale_log2,
                              j == 0, m, l, prev_pv, prev_ph, abort_flag, a.err, diagb);
        }
        if (!done) return false;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kPFull + sb]);  // P is ready and S has been read
        return true;
      };
      if constexpr (kDense) {  // one loop: peeling adds spills to this form's larger state
        for (int j = 0; ok && j < it.nt; ++j, ++g)
          ok = (j < it.nk && (it.nk - 1 - j) * BN + BN - 1 > mask_from)
                   ? step(j, std::true_type{})
                   : step(j, std::false_type{});
      } else {
        if (it.nt > 0) {
          ok = step(0, std::true_type{});
          ++g;
        }
        for (int j = 1; ok && j < it.nt; ++j, ++g) ok = step(j, std::false_type{});
      }
      if (!ok) break;
      // hand the row's softmax state to the epilogue with the O buffer
      const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
      if (!wait_warp(&bars[kOEmpty + ob], par(oi >> 1) ^ 1u, abort_flag, a.err)) break;
      if (h == 0) sML[ob * BM + rt] = make_float2(m - rowcb, l_row);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kOFull + ob]);
    }
  } else if (warp < 14) {
    // ---------------------------------------------------------------- epilogue warps 10-13
    const int ew = warp & 3;          // TMEM lane quadrant of the warp
    const int r = ew * 32 + lane;     // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(ew * 32) << 16);
    __nv_bfloat16* Og = (__nv_bfloat16*)a.o;
    uint8_t* stage = smem + kOffStage + ew * 32 * (DH * 2);  // this warp's 32 rows
    int oi = 0;
    Item nx = blockIdx.x < total ? load_item(P, blockIdx.x) : Item{};
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const Item it = nx;
      if (w + (int)gridDim.x < total) nx = load_item(P, w + gridDim.x);
      if (it.nt == 0) continue;
      const int ob = oi & 1;
      if (!wait_warp(&bars[kOFull + ob], par(oi >> 1), abort_flag, a.err)) break;
      tc_fence_after();
      const float2 ml = sML[ob * BM + r];
      float o[DH];
      tmem_ld64(lane_base + kColO + ob * DH, o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kOEmpty + ob]);
      ++oi;
      // normalise and stage the row (16-byte chunks XOR-swizzled by row), then write
      // the warp's 32 rows as whole 128-byte lines
      const float inv = 1.f / ml.y;
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = o[c * 8 + e] * inv;
        *reinterpret_cast<uint4*>(stage + lane * (DH * 2) + ((c ^ (lane & 7)) * 16)) =
            Elem<__nv_bfloat16>::pack(f);
      }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int rr = k * 4 + (lane >> 3), c = lane & 7;
        const int ii = it.q0 + ew * 32 + rr;
        if (ii < it.L) {
          const uint4 v =
              *reinterpret_cast<const uint4*>(stage + rr * (DH * 2) + ((c ^ (rr & 7)) * 16));
          *reinterpret_cast<uint4*>(Og + ((long long)it.s + ii) * a.o_stride + it.h * DH + c * 8) =
              v;
        }
      }
      __syncwarp();
      const int i = it.q0 + r;
      if (i < it.L && a.lse)
        a.lse[(long long)it.h * a.T + it.s + i] = (ml.x + __log2f(ml.y)) * kLn2;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
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

// the kernels' dynamic shared-memory limit, raised once per device and variant
static DeviceOnce fwd_smem_attr[3];

// mode: the time bias (kTimeBiasLinear, kTimeBiasBucketed) or kDenseBiasMode
constexpr int kDenseBiasMode = 2;
static int launch_kernel(const Params& p, int mode, cudaStream_t st) {
  const void* fn = mode == kTimeBiasBucketed ? (const void*)k_attn_fwd_tc<true, false>
                   : mode == kDenseBiasMode  ? (const void*)k_attn_fwd_tc<false, true>
                                             : (const void*)k_attn_fwd_tc<false, false>;
  if (!set_smem_limit_once(fwd_smem_attr[mode], fn, (int)kSmemBytes)) return GENRANK_ERR_CUDA;
  const int sms = sm_count_current();
  if (sms <= 0) return GENRANK_ERR_CUDA;
  if (mode == kTimeBiasBucketed)
    k_attn_fwd_tc<true, false><<<sms, kThreads, kSmemBytes, st>>>(p);
  else if (mode == kDenseBiasMode)
    k_attn_fwd_tc<false, true><<<sms, kThreads, kSmemBytes, st>>>(p);
  else
    k_attn_fwd_tc<false, false><<<sms, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

static size_t recs_bytes(int B, int max_seqlen) {
  return ((size_t)B * max_tiles_of(max_seqlen) * kRecInts * 4 + 15) / 16 * 16;
}
static size_t users_bytes(int B) { return ((size_t)B * 4 + 15) / 16 * 16; }

}  // namespace tc

size_t attn_fwd_tc_workspace(int B, long long T, int H, int max_seqlen) {
  using namespace tc;
  // records, user order, column terms [H][Tp], (bucketed bias) token times [Tp] and the
  // column terms in the MMA's form [H][Tp] x 16 B
  return kHeaderBytes + recs_bytes(B, max_seqlen) + users_bytes(B) +
         (size_t)(H + 1) * scratch_tp(T, B) * sizeof(float) +
         (size_t)H * scratch_tp(T, B) * sizeof(uint4);
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
  p.tkc = p.tk;
  p.tvc = p.tv;
  p.a = a;
  uint8_t* ws = (uint8_t*)a.ws;
  int32_t* count = (int32_t*)ws;
  int4* recs = (int4*)(ws + kHeaderBytes);
  int32_t* uorder = (int32_t*)(ws + kHeaderBytes + recs_bytes(a.B, a.max_seqlen));
  float* cbias = (float*)((uint8_t*)uorder + users_bytes(a.B));
  p.count = count;
  p.recs = recs;
  p.cbias = cbias;
  p.Tp = scratch_tp(a.T, a.B);
  const bool bucket = a.time_bias == kTimeBiasBucketed;
  int32_t* trel = bucket ? (int32_t*)(cbias + (size_t)a.H * p.Tp) : nullptr;
  p.trel = trel;
  uint4* caug = (uint4*)(cbias + (size_t)(a.H + 1) * p.Tp);
  p.caug = caug;
  k_prologue<<<a.B + 1, kSchedThreads, 0, st>>>(a, max_tiles, recs, count, uorder, cbias, caug,
                                                trel, p.Tp);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  p.dbias = nullptr;
  p.Lpad = 0;
  return launch_kernel(p, a.time_bias == kTimeBiasBucketed ? kTimeBiasBucketed : kTimeBiasLinear,
                       st);
}

int launch_attn_fwd_dense(const AttnArgs& a, const void* bias, long long Lpad, cudaStream_t st) {
  using namespace tc;
  if (a.dh != DH || a.dtype != GENRANK_BF16) return GENRANK_ERR_UNSUPPORTED;
  if (a.T + (long long)BM >= INT32_MAX / 2) return GENRANK_ERR_UNSUPPORTED;
  Params p;
  if (!make_map(&p.tq, a.q, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tk, a.k, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tv, a.v, a.T, a.H, a.tok_stride))
    return GENRANK_ERR_CUDA;
  p.tkc = p.tk;
  p.tvc = p.tv;
  p.a = a;
  uint8_t* ws = (uint8_t*)a.ws;
  int32_t* count = (int32_t*)ws;
  int4* recs = (int4*)(ws + kHeaderBytes);
  int32_t* uorder = (int32_t*)(ws + kHeaderBytes + recs_bytes(a.B, a.max_seqlen));
  float* cbias = (float*)((uint8_t*)uorder + users_bytes(a.B));
  p.count = count;
  p.recs = recs;
  p.cbias = cbias;  // not read by the dense-bias kernel
  p.caug = nullptr;
  p.Tp = scratch_tp(a.T, a.B);
  p.trel = nullptr;
  p.dbias = (const __nv_bfloat16*)bias;
  p.Lpad = Lpad;
  k_prologue<<<a.B + 1, kSchedThreads, 0, st>>>(a, max_tiles_of(a.max_seqlen), recs, count,
                                                uorder, nullptr, nullptr, nullptr, p.Tp);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  return launch_kernel(p, kDenseBiasMode, st);
}

size_t attn_fwd_cached_workspace(int B, long long C, long long Th, int H, int max_cand) {
  using namespace tc;
  return kHeaderBytes + recs_bytes(B, max_cand) + users_bytes(B) +
         (size_t)H * scratch_tp_cached(C + Th, B) * (sizeof(float) + sizeof(uint4));
}

int launch_attn_fwd_cached(const CachedAttnArgs& c, cudaStream_t st) {
  using namespace tc;
  const AttnArgs& a = c.a;
  if (a.dh != DH || a.dtype != GENRANK_BF16) return GENRANK_ERR_UNSUPPORTED;
  if (a.T + c.Th + (long long)BM >= INT32_MAX / 2) return GENRANK_ERR_UNSUPPORTED;
  Params p;
  if (!make_map(&p.tq, a.q, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tkc, a.k, a.T, a.H, a.tok_stride) ||
      !make_map(&p.tvc, a.v, a.T, a.H, a.tok_stride))
    return GENRANK_ERR_CUDA;
  if (c.Th > 0) {
    if (!make_map(&p.tk, c.k_hist, c.Th, a.H, c.hist_stride) ||
        !make_map(&p.tv, c.v_hist, c.Th, a.H, c.hist_stride))
      return GENRANK_ERR_CUDA;
  } else {  // no history anywhere: no history tile is ever loaded
    p.tk = p.tkc;
    p.tv = p.tvc;
  }
  p.a = a;
  uint8_t* ws = (uint8_t*)a.ws;
  int32_t* count = (int32_t*)ws;
  int4* recs = (int4*)(ws + kHeaderBytes);
  int32_t* uorder = (int32_t*)(ws + kHeaderBytes + recs_bytes(a.B, c.max_cand));
  float* cbias = (float*)((uint8_t*)uorder + users_bytes(a.B));
  p.count = count;
  p.recs = recs;
  p.cbias = cbias;
  p.Tp = scratch_tp_cached(a.T + c.Th, a.B);
  uint4* caug = (uint4*)(cbias + (size_t)a.H * p.Tp);
  p.caug = caug;
  CachedArgsHolder holder{c};
  k_prologue_cached<<<a.B + 1, kSchedThreads, 0, st>>>(holder, max_tiles_of(c.max_cand), recs,
                                                       count, uorder, cbias, caug, p.Tp);
  if (cudaGetLastError() != cudaSuccess) return GENRANK_ERR_LAUNCH;
  p.trel = nullptr;
  p.dbias = nullptr;
  p.Lpad = 0;
  return launch_kernel(p, kTimeBiasLinear, st);
}

}  // namespace gr

