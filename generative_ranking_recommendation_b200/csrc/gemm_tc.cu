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
// Design: persistent clusters of two CTAs, one per SM of an SM pair, 320 threads each.
// A tile is 256 rows x 256 columns (x 512 for res+rms), computed by one tcgen05.mma of
// M = 256 spanning both SMs (cta_group::2): each CTA holds its own 128 rows of A and half
// of the 256 Wt rows, so an SM loads 32 KB of operands per 64-wide k-step instead of
// 48 KB, and each CTA's TMEM receives its own 128 rows of the accumulator.
//   * warp 1 of each CTA issues TMA loads of its 128 x 64 A tile and 128 x 64 Wt tile
//     (128B swizzle, no multicast) into a ring of 32 KB stages (six; four for res+rms);
//     both CTAs' loads complete on the even CTA's barrier;
//   * warp 0 of the even CTA (one thread) issues the pair's MMAs, N = 256, K = 16 (four
//     per k-step), and commits each stage's release and each accumulator's completion to
//     the barriers of both CTAs.  The store and SiLU epilogues double-buffer the
//     accumulator (2 x 256 columns) so a tile's epilogue overlaps the next tile's MMAs;
//     the epilogue warps of both CTAs hand a buffer back on the even CTA's barrier.
//     res+rms computes its row (d = 512) as two 256-column halves, into columns [0, 256)
//     and [256, 512), taking turns every 16 k-steps (the A rows of a chunk are re-read
//     from L2, not DRAM): the first half completes a chunk early and its residual pass
//     overlaps the second half's last MMAs, and each half's columns are released as soon
//     as the normalisation has read them (for K >= 1024, as soon as the residual pass has
//     read them, the normalisation then re-reading the stored fp32 rows by TMA);
//   * warps 2-9 run the epilogue from TMEM, two warps per TMEM lane quadrant (one row
//     per thread), each on half of a 256-column block; res+rms combines the two warps'
//     row sums of squares (and head partial sums) through shared memory.  Outputs leave
//     through 2 KB shared-memory boxes (64-byte swizzle, so one-row-per-thread writes
//     hit every bank) as TMA stores of whole lines; res+rms loads its residual rows the
//     same way, four boxes ahead of use per warp.
// Tiles are ordered with the N tiles of one M tile adjacent, so pairs running them at the
// same time share the A tile in L2.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {
namespace tg {

constexpr int BM = 128;
constexpr int BN = 256;  // columns per MMA block (one accumulator buffer)
constexpr int BK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
// one MMA of M = 256 rows (128 per CTA of an SM pair) x N = 256; A and Wt K-major
constexpr uint32_t kIdesc = idesc_bf16_f32(2 * BM, BN, 0, 0);
constexpr int kTileRows = 2 * BM;  // rows per tile
constexpr uint32_t kABytes = BM * BK * 2;                    // 16 KB
constexpr uint32_t kBBytes = BN * BK * 2;                    // 32 KB
// res+rms: the two 256-column halves take turns in chunks of this many k-steps, so a
// tile's A rows are read from DRAM once (the other half's read of the chunk hits L2) and
// the first half still completes one chunk ahead of the second
constexpr int kChunkSteps = 16;
// res+rms for long K (K >= kReleaseMinK): each TMEM half goes back to the MMAs as soon as
// its residual pass has read it, and the normalisation re-reads the stored fp32 rows
// (still in L2) by TMA, so the next tile's MMAs overlap the rest of the epilogue
constexpr int kEpiResRmsRel = 3;
constexpr int kReleaseMinK = 1024;
constexpr uint32_t kBoxBytes = 2048;  // 32 rows x 64 bytes (32 bf16 or 16 fp32 columns)
constexpr int kXBufs = 4;             // res+rms: residual boxes in flight per epilogue warp

// Shared memory of each CTA: the operand stages (its 128 A rows and 128 Wt rows of a
// k-step, 32 KB), then per epilogue:
//   store / SiLU: six stages; two output boxes per epilogue warp (ping-pong).
//   res+rms: four stages (room for the residual boxes); per epilogue warp kXBufs boxes
//     the residual rows are loaded into and one output box; then the row partial sums
//     (one float per row and column half).
// Then the barriers: full[S], empty[S], acc_full[2], acc_empty[2], done and, for res+rms,
// one per residual box (full and acc_empty are used in the even CTA only).
template <bool kRes>
struct Layout {
  static constexpr uint32_t kStageBytes = kABytes + kBBytes / 2;
  static constexpr int kStages = kRes ? 4 : 6;
  static constexpr uint32_t kOffBox = kStages * kStageBytes;
  static constexpr uint32_t kXBytes = kRes ? kEpiWarps * kXBufs * kBoxBytes : 0;
  static constexpr uint32_t kOutBoxes = kRes ? 1 : 2;
  static constexpr uint32_t kOffOut = kOffBox + kXBytes;
  static constexpr uint32_t kOffRed = kOffOut + kEpiWarps * kOutBoxes * kBoxBytes;
  static constexpr uint32_t kOffBar = kOffRed + (kRes ? 2 * BM * 4 : 0);
  static constexpr uint32_t kNumBars = 2 * kStages + 5 + (kRes ? kEpiWarps * kXBufs : 0);
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmem = kOffMisc + 16 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "1024-byte aligned stages");
};

struct Params {
  CUtensorMap ta, tb;
  CUtensorMap tc;  // C (store / SiLU) or a_out (res+rms): bf16, box 32 x 32, 64-byte swizzle
  CUtensorMap tx;   // res+rms: x_out, fp32, box 16 x 32, 64-byte swizzle (TMA store)
  CUtensorMap txi;  // res+rms: x_in, the same geometry (TMA load)
  GemmArgs g;
};

GR_DEVICE uint32_t par(int x) { return (uint32_t)(x & 1); }

GR_DEVICE bool wait_warp(uint64_t* bar, uint32_t ph, volatile int* abort_flag, int32_t* err) {
  const bool ok = mbar_wait(bar, ph, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

// At most one committed bulk group of this thread has yet to finish reading its source.
GR_DEVICE void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

GR_DEVICE float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// SiLU(v) = v sigmoid(v) = v/2 + (v/2) tanh(v/2): one MUFU operation per element (the
// result is rounded to bf16, well above the approximation's error)
GR_DEVICE float silu(float v) {
  const float h = 0.5f * v;
  return fmaf(h, tanh_approx(h), h);
}

// Byte offset of 16-byte unit j of row r in a box of 64-byte rows written with the TMA
// engine's 64-byte swizzle (unit index XOR address bits 7-8; the box is 512-byte aligned),
// so a warp writing one row per thread spreads its stores over all banks.
GR_DEVICE uint32_t sw64(int r, int j) { return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4)); }

// 32 fp32 values to bf16, as row r of a 32 x 32 bf16 box (64-byte swizzle).
GR_DEVICE void box_bf16x32(uint8_t* box, int r, const float* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(box + sw64(r, j)) =
        make_uint4(pack_bf16(v[8 * j], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                   pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
}

// 16 fp32 values to bf16, as columns [16 half, 16 half + 16) of row r of a 32 x 32 bf16
// box (64-byte swizzle).
GR_DEVICE void box_bf16x16(uint8_t* box, int r, int half, const float* v) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
    *reinterpret_cast<uint4*>(box + sw64(r, 2 * half + j)) =
        make_uint4(pack_bf16(v[8 * j], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                   pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
}

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1) k_gemm_tc(const __grid_constant__ Params P) {
  constexpr bool kRes = kEpi == kEpiResRms || kEpi == kEpiResRmsRel;
  constexpr bool kRel = kEpi == kEpiResRmsRel;
  using L = Layout<kRes>;
  constexpr int kStages = L::kStages;
  constexpr uint32_t kStageBytes = L::kStageBytes;
  constexpr int kHalves = kRes ? 2 : 1;  // 256-column blocks per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemmArgs& g = P.g;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_full + 4;
  uint64_t* xbar = acc_full + 5;  // res+rms: [epilogue warp][kXBufs] residual box loads
  // res+rms partial sums, [warp ch 0][warp ch 1] x BM rows: the sums of squares, then
  // the head's dot products
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA `rank` of the pair holds rows [128 rank, 128 rank + 128) of each tile; the even
  // CTA issues the MMAs.  The pair runs tiles first, first + stride, ...
  const int rank = (int)cluster_ctarank();
  const int first = (int)cluster_idx();
  const int stride = (int)cluster_count();
  const int row_off = rank * BM;  // this CTA's first row within a tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      // one arrival per epilogue warp of both CTAs (the even CTA's barrier is used)
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(done, 1);
    if (kRes)
      for (int b = 0; b < kEpiWarps * kXBufs; ++b) mbar_init(&xbar[b], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&P.ta);
    tma_prefetch_desc(&P.tb);
    if (!kRes || g.a_out) tma_prefetch_desc(&P.tc);
    if (kRes) {
      tma_prefetch_desc(&P.tx);
      tma_prefetch_desc(&P.txi);
    }
  }
  if (warp == 0) {
    tmem_alloc<true>(tmem_slot, kTmemCols);
    tmem_relinquish<true>();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m_tiles = (g.M + kTileRows - 1) / kTileRows;
  const int n_tiles = kRes ? 1 : g.N / BN;
  const int tiles = m_tiles * n_tiles;
  const int ksteps = g.K / BK;

  if (warp == 1) {
    // ------------------------------------------------------------------ TMA producer
    int it = 0;
    bool ok = true;
    for (int t = first; t < tiles && ok; t += stride) {
      const int mt = t / n_tiles, nt = t - mt * n_tiles;
      for (int k0 = 0; k0 < ksteps && ok; k0 += kChunkSteps) {
        const int k1 = min(ksteps, k0 + kChunkSteps);
        for (int h = 0; h < kHalves && ok; ++h) {
          for (int ks = k0; ks < k1; ++ks, ++it) {
            const int st = it % kStages;
            if (!wait_warp(&empty[st], par(it / kStages) ^ 1u, abort_flag, g.err)) {
              ok = false;
              break;
            }
            if (lane == 0) {
              uint8_t* sa = smem + st * kStageBytes;
              // both CTAs' tiles complete on the even CTA's barrier, which expects both
              const uint32_t fb = cluster_addr(&full[st], 0);
              if (rank == 0) mbar_expect_tx(&full[st], 2 * kStageBytes);
              tma_load_2d_pair(sa, &P.ta, fb, ks * BK, mt * kTileRows + row_off);
              tma_load_2d_pair(sa + kABytes, &P.tb, fb, ks * BK, (nt + h) * BN + rank * (BN / 2));
            }
          }
        }
      }
    }
    // the copies issued last land before the CTA exits (the odd CTA of a pair: its stages
    // have been read by the pair's MMAs, which waited for them)
    if (lane == 0)
      for (int x = max(0, it - kStages); x < it; ++x) {
        if (rank == 0)
          mbar_drain(&full[x % kStages], par(x / kStages));
        else
          mbar_drain(&empty[x % kStages], par(x / kStages));
      }
  } else if (warp == 0) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = first; t < tiles && ok; t += stride, ++tc) {
        const int buf = kRes ? 0 : (tc & 1);
        const uint32_t ph_empty = kRes ? par(tc) ^ 1u : par(tc >> 1) ^ 1u;
        if (!kRes) {
          if (!mbar_wait<true>(&acc_empty[buf], ph_empty, abort_flag, g.err)) break;
          tc_fence_after();
        }
        for (int k0 = 0; k0 < ksteps && ok; k0 += kChunkSteps) {
          const int k1 = min(ksteps, k0 + kChunkSteps);
          for (int h = 0; h < kHalves && ok; ++h) {
            if (kRes && k0 == 0) {  // each half's columns are released on their own
              if (!mbar_wait<true>(&acc_empty[h], ph_empty, abort_flag, g.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint32_t acc = tmem + (uint32_t)((kRes ? h : buf) * BN);
            for (int ks = k0; ks < k1; ++ks, ++it) {
              const int st = it % kStages;
              if (!mbar_wait(&full[st], par(it / kStages), abort_flag, g.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t sa = smem_u32(smem + st * kStageBytes);
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(sa + kABytes + kk * 32, 16, 1024);
                mma_bf16_ss_pair(acc, ad, bd, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
              }
              // the stage (both CTAs' copies of it) is free once these MMAs have read it
              mma_commit_pair(&empty[st], 0x3);
            }
            if (ok && k1 == ksteps) mma_commit_pair(&acc_full[kRes ? h : buf], 0x3);
          }
        }
      }
      // every MMA issued has completed before TMEM is freed
      mma_commit_pair(done, 0x1);
      mbar_drain(done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue warps 2-9
    const int ew = warp - 2;
    const int q = warp & 3;  // TMEM lane quadrant
    const int ch = ew >> 2;  // which 128 columns of each 256-column block
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int rloc = q * 32 + lane;  // row within the tile
    const int box_row = q * 32;      // + the CTA's first row of the tile: the warp's in C
    uint8_t* out = smem + L::kOffOut + ew * L::kOutBoxes * kBoxBytes;  // output boxes
    // accumulator buffer b has been read by this warp (on the even CTA's barrier)
    auto release_acc = [&](int b) { mbar_arrive_cluster(cluster_addr(&acc_empty[b], 0)); };
    if (!kRes) {
      int tc = 0;
      for (int t = first; t < tiles; t += stride, ++tc) {
        const int mt = t / n_tiles, nt = t - mt * n_tiles;
        const int buf = tc & 1;
        if (!wait_warp(&acc_full[buf], par(tc >> 1), abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t acc = lane_base + (uint32_t)(buf * BN + ch * 128);
        // each 32 x 32 chunk (the warp's rows, 32 columns) is written to one of the warp's
        // two boxes and stored by the TMA engine as whole lines; rows past M are clipped
        // by the tensor map
        const int gcol = nt * BN + ch * 128;
        const int grow = mt * kTileRows + row_off + box_row;  // the warp's first row in C
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          float v[32];
          tmem_ld32(acc + c, v);
          if (kEpi == kEpiSilu) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = silu(v[e]);
          }
          uint8_t* box = out + ((c >> 5) & 1) * kBoxBytes;
          if (lane == 0) bulk_wait_read_1();  // the store that last read this box is done
          __syncwarp();
          box_bf16x32(box, lane, v);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && grow < g.M) {  // boxes wholly past M are skipped
            tma_store_2d(&P.tc, box, gcol + c, grow);
            bulk_commit();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(buf);
      }
    } else {
      // res+rms.  The warp's residual boxes (32 rows x 16 fp32 columns, 16 a tile: 8 per
      // 256-column half; with the early release another 16 of the stored rows for the
      // normalisation) are numbered across its tiles; box n goes to buffer n % kXBufs,
      // and the load of box n + kXBufs is issued as soon as box n has been read, so the
      // next tile's first boxes load while this tile's normalisation runs.  A re-read of
      // the stored rows is issued only once the tile's stores have completed.
      constexpr int kPerTile = kRel ? 32 : 16;
      uint8_t* xb = smem + L::kOffBox + ew * kXBufs * kBoxBytes;
      uint64_t* xw = xbar + ew * kXBufs;
      const int my_tiles = first < tiles ? (tiles - 1 - first) / stride + 1 : 0;
      const int nbox = kPerTile * my_tiles;
      auto issue = [&](int n) {  // lane 0: load box n
        const int t = first + (n / kPerTile) * stride;
        const int w = n % kPerTile;
        const int col = ((w >> 3) & 1) * BN + ch * 128 + (w & 7) * 16;
        const int b = n % kXBufs;
        mbar_expect_tx(&xw[b], kBoxBytes);
        tma_load_2d(xb + b * kBoxBytes, w < 16 ? (const void*)&P.txi : (const void*)&P.tx, &xw[b],
                    col, t * kTileRows + row_off + box_row);
      };
      int ld = 0;  // boxes whose loads were issued
      if (lane == 0)
        for (int x = 0; x < kXBufs && x < nbox; ++x) issue(x);
      ld = min(kXBufs, nbox);
      int n = 0;  // boxes consumed
      // waits for box n; false (the error recorded) when it timed out
      auto wait_box = [&](int x) { return wait_warp(&xw[x % kXBufs], par(x / kXBufs), abort_flag, g.err); };
      // after box n has been read by every lane: the next load, unless it is a re-read
      // of this tile's stored rows and the residual pass is still running
      auto next_load = [&](bool pass1) {
        __syncwarp();
        const bool go = ld < nbox && !(kRel && pass1 && (ld % kPerTile) >= 16);
        if (go && lane == 0) issue(ld);
        if (go) ++ld;
      };
      int tc = 0;
      // A failed (timed-out) wait skips the work but not the named barriers below, so the
      // other warp of the quadrant never waits for a partner that has left.
      bool ok = true;
      for (int t = first; t < tiles; t += stride, ++tc) {
        const int mt = t;
        const int grow = mt * kTileRows + row_off + box_row;  // the warp's first row
        const long long row = (long long)mt * kTileRows + row_off + rloc;
        const bool valid = row < g.M;
        const bool rows_in = grow < g.M;  // boxes wholly past M are skipped
        // pass 1 per half as soon as its MMAs are done: y = x_in + acc, kept in TMEM,
        // written to x_out through the output box, its squares summed
        float ss = 0.f;
        for (int h = 0; h < 2 && ok; ++h) {
          if (!wait_warp(&acc_full[h], par(tc), abort_flag, g.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int c0 = h * BN + ch * 128;
#pragma unroll 1
          for (int c = 0; c < 128; c += 16, ++n) {
            uint32_t a[16];
            tmem_ld16_async(lane_base + c0 + c, a);
            if (!wait_box(n)) {
              tmem_ld_wait(a);
              ok = false;
              break;
            }
            const uint8_t* xs = xb + (n % kXBufs) * kBoxBytes;
            float4 y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) y[e] = *reinterpret_cast<const float4*>(xs + sw64(lane, e));
            tmem_ld_wait(a);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              y[e].x += __uint_as_float(a[4 * e]);
              y[e].y += __uint_as_float(a[4 * e + 1]);
              y[e].z += __uint_as_float(a[4 * e + 2]);
              y[e].w += __uint_as_float(a[4 * e + 3]);
              ss = fmaf(y[e].x, y[e].x, ss);
              ss = fmaf(y[e].y, y[e].y, ss);
              ss = fmaf(y[e].z, y[e].z, ss);
              ss = fmaf(y[e].w, y[e].w, ss);
              a[4 * e] = __float_as_uint(y[e].x);
              a[4 * e + 1] = __float_as_uint(y[e].y);
              a[4 * e + 2] = __float_as_uint(y[e].z);
              a[4 * e + 3] = __float_as_uint(y[e].w);
            }
            if (!kRel) tmem_st16(lane_base + c0 + c, a);
            next_load(true);
            if (lane == 0) bulk_wait_read_all();  // the output box's previous store has read it
            __syncwarp();
#pragma unroll
            for (int e = 0; e < 4; ++e) *reinterpret_cast<float4*>(out + sw64(lane, e)) = y[e];
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && rows_in) {
              tma_store_2d(&P.tx, out, c0 + c, grow);
              bulk_commit();
            }
          }
          if (kRel && ok) {  // this half's accumulator columns go back to the MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc(h);
          }
        }
        // the row's sum of squares over both warps of this quadrant
        red[ch * BM + rloc] = ss;
        named_bar_sync(1 + q, 64);
        const float r = rsqrtf((red[rloc] + red[BM + rloc]) / (float)g.N + g.eps);
        if (kRel && ok) {
          // the stored rows are re-read once the tile's stores have completed
          if (lane == 0) bulk_wait_all();
          for (int x = 0; x < kXBufs; ++x) next_load(false);
        }
        // pass 2: the normalised row, to a_out in bf16 and into the head's dot product, 16
        // columns a step (an a_out box takes two); unless released already, each half's
        // accumulator columns go back to the MMAs as soon as they have been read, so the
        // next tile's first half overlaps this tile's second
        float z = 0.f;
        for (int h = 0; h < 2 && ok; ++h) {
          const int c0 = h * BN + ch * 128;
#pragma unroll 1
          for (int c = 0; c < 128; c += 16) {
            float v[16];
            if (kRel) {
              if (!wait_box(n)) {
                ok = false;
                break;
              }
              const uint8_t* xs = xb + (n % kXBufs) * kBoxBytes;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float4 y = *reinterpret_cast<const float4*>(xs + sw64(lane, e));
                v[4 * e] = y.x;
                v[4 * e + 1] = y.y;
                v[4 * e + 2] = y.z;
                v[4 * e + 3] = y.w;
              }
              ++n;
              next_load(false);
            } else {
              uint32_t a[16];
              tmem_ld16_async(lane_base + c0 + c, a);
              tmem_ld_wait(a);
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(a[e]);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] *= r;
            if (g.a_out) {
              const int half = (c >> 4) & 1;
              if (half == 0) {
                if (lane == 0) bulk_wait_read_all();  // the output box's previous store is done
                __syncwarp();
              }
              box_bf16x16(out, lane, half, v);
              if (half == 1) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && rows_in) {
                  tma_store_2d(&P.tc, out, c0 + c - 16, grow);
                  bulk_commit();
                }
              }
            }
            if (g.w_head) {
              const float4* w4 = reinterpret_cast<const float4*>(g.w_head + c0 + c);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float4 wv = w4[e];
                z = fmaf(v[4 * e], wv.x, z);
                z = fmaf(v[4 * e + 1], wv.y, z);
                z = fmaf(v[4 * e + 2], wv.z, z);
                z = fmaf(v[4 * e + 3], wv.w, z);
              }
            }
          }
          if (!kRel) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc(h);
          }
        }
        if (g.w_head) {
          named_bar_sync(1 + q, 64);  // both warps have read the sums of squares
          red[ch * BM + rloc] = z;
          named_bar_sync(1 + q, 64);
          if (ch == 0 && valid) g.z[row] = red[rloc] + red[BM + rloc];
        }
        // the partial-sum slots are reused by the next tile only after both warps of the
        // quadrant have read them
        named_bar_sync(1 + q, 64);
        if (!ok) break;
      }
      // boxes still in flight (a failed wait) land before the CTA exits
      if (lane == 0)
        for (int x = n; x < min(ld, nbox); ++x) mbar_drain(&xw[x % kXBufs], par(x / kXBufs));
    }
  }

  if (warp >= 2 && lane == 0) bulk_wait_all();  // the output stores have landed
  __syncwarp();
  tc_fence_before();
  // neither CTA leaves (or frees TMEM) while the other may still signal its barriers or
  // the pair's MMAs read its shared memory
  cluster_sync();
  tc_fence_after();
  if (warp == 0) tmem_dealloc<true>(tmem, kTmemCols);
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

// [rows][N] output (bf16 or fp32) with row stride ld elements, for TMA stores of 32-row
// boxes of 64 bytes (32 bf16 or 16 fp32 columns) with the 64-byte swizzle.
static bool make_store_map(CUtensorMap* m, void* base, long long rows, int N, long long ld,
                           bool f32) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * es};
  cuuint32_t box[2] = {(cuuint32_t)(64 / es), 32};
  cuuint32_t elem_strides[2] = {1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base,
            dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kEpi>
static int launch_t(const GemmArgs& g, cudaStream_t st) {
  constexpr bool kRes = kEpi >= kEpiResRms;
  Params p;
  if (!make_map(&p.ta, g.a, g.M, g.K, g.lda, BM) || !make_map(&p.tb, g.w, g.N, g.K, g.ldw, BN / 2))
    return GENRANK_ERR_CUDA;
  if (kRes) {
    if (!make_store_map(&p.tx, g.x_out, g.M, g.N, g.ldx, true) ||
        !make_store_map(&p.txi, const_cast<float*>(g.x_in), g.M, g.N, g.ldx, true) ||
        (g.a_out && !make_store_map(&p.tc, g.a_out, g.M, g.N, g.lda_out, false)))
      return GENRANK_ERR_CUDA;
  } else if (!make_store_map(&p.tc, g.c, g.M, g.N, g.ldc, false)) {
    return GENRANK_ERR_CUDA;
  }
  p.g = g;
  constexpr int kSmem = (int)Layout<kRes>::kSmem;
  static DeviceOnce smem_attr;
  if (!set_smem_limit_once(smem_attr, (const void*)k_gemm_tc<kEpi>, kSmem))
    return GENRANK_ERR_CUDA;
  const int sms = sm_count_current();
  if (sms <= 0) return GENRANK_ERR_CUDA;
  const long long tiles =
      (long long)((g.M + kTileRows - 1) / kTileRows) * (kRes ? 1 : g.N / BN);
  // clusters of two CTAs (one per SM of a pair), as many as can be resident at once
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static DeviceOnce pairs_once;
  const int pairs = pairs_once.run([&](int) {
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(2 * (unsigned)(sms / 2));
    int n = 0;
    return cudaOccupancyMaxActiveClusters(&n, (const void*)k_gemm_tc<kEpi>, &q) == cudaSuccess
               ? n
               : 0;
  });
  if (pairs <= 0) return GENRANK_ERR_CUDA;
  cfg.gridDim = dim3(2 * (unsigned)(tiles < pairs ? tiles : pairs));
  if (cudaLaunchKernelEx(&cfg, k_gemm_tc<kEpi>, p) != cudaSuccess) return GENRANK_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? GENRANK_OK : GENRANK_ERR_LAUNCH;
}

}  // namespace tg

int launch_gemm_tc(const GemmArgs& g, cudaStream_t st) {
  using namespace tg;
  if (g.M == 0) return GENRANK_OK;
  switch (g.epilogue) {
    case kEpiStore: return launch_t<kEpiStore>(g, st);
    case kEpiSilu: return launch_t<kEpiSilu>(g, st);
    case kEpiResRms:
      return g.K >= kReleaseMinK ? launch_t<kEpiResRmsRel>(g, st) : launch_t<kEpiResRms>(g, st);
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
