// halo_tc3.cuh -- stride-1 bf16 kernel for blocked local self-attention with
// haloing on sm_100a, for 16x16 query blocks (windows of 16..24 pixels) and
// 32x32 query blocks (windows of 32..38 pixels: global attention on a 32x32
// map, section 2.2, and the block-32 detection setting, section 4.5).
//
// Operation (HaloNet, "Scaling Local Self-Attention for Parameter Efficient
// Visual Backbones", sections 2.1-2.2 and appendix A; index conventions of the
// blog page's RelPosEmb / HaloAttention modules):
//   z[q, key] = s * q . (k[key] + rel_h[kr - qy + w - 1] + rel_w[kc - qx + w - 1])
//   out[q]    = sum over in-image window keys of softmax(z) * v[key]
//
// A 16x16 block has 256 queries, so one head already fills two 128-row MMA
// tiles; the window (up to 24 x 24 = 576 keys) is too wide for one TMEM pass.
//
// Work item = 256 queries of one head: a whole 16x16 block, or a quarter
// (8 query rows) of a 32x32 block.  Warpgroup g (g = 0, 1) takes half of the
// item's query rows (128 queries, TMEM lane = query):
//   * TMA (warp 8): Q [256 x d], K and V [w*w keys x d] of the item into one
//     pipeline stage; the relative table R = [rel_h; 0; rel_w; 0] (96 rows)
//     is written to shared memory once at start-up.
//   * G MMA (warp 9 + g): G = Q_g R^T, M=128, N=96 (block 16) or 160
//     (block 32): the query's dot products with every rel_h and rel_w row,
//     into the S buffer the item's first chunk will use (block 16), or
//     across both S buffers (block 32).  Each thread picks the w + w it
//     needs: the warp-uniform part of the row shift through the TMEM load
//     address, the per-lane part by selects (no scratch memory).  At block 16
//     the warpgroup gathers item k+1's before item k's epilogue, so the G MMA
//     hides behind the last A.V; at block 32 it follows the epilogue.
//   * S MMA (warp 9 + g): the window in chunks of 4 (block 16) or 2 (block
//     32) window rows, S_c = Q_g K_c^T (N = rows * w rounded to 16),
//     alternating between two TMEM buffers across chunks and items.
//   * softmax (one thread per query row): per chunk the exact chunk maximum of
//     c*S + c*rel_w + c*rel_h; the running maximum moves only when the chunk's
//     exceeds it by more than 8 (in log2 units), and only then is the fp32
//     accumulator O rescaled (a rare path).  Exponentials part on MUFU, part as
//     a cubic on the FMA pipe; bf16 P written back over the chunk's S columns.
//   * A.V (issued by the warpgroup's MMA warp once all four softmax warps
//     have stored the chunk's P, right after it issued the next chunk's S):
//     [O | l] += P_c [V_c | ones], M=128, N=d+8, P from TMEM; the ones
//     columns give the row sum of the bf16 P.  The softmax warps never wait
//     for one another within an item.
//   * epilogue: O / (row sum from the ones columns), bf16, NHWC store.
// Every wait is bounded and reports HALO_ERR_TIMEOUT.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <type_traits>
#include <utility>

#include "halo_tc.cuh"
#include "halo_tc2.cuh"
#include "sm100.cuh"

namespace halo {
namespace tc3 {

using namespace sm100;
using tc::exp2_mufu;
using tc::pack_bf16x2;
using tc::record_timeout;
using tc::swz;
using tc2::exp2_poly2;
using tc2::max3f;
using tc2::mma_f16_ts;
using tc2::pack_p;
using tc2::tmem_ld_cols;
using tc2::tmem_ld_x32;
using tc2::tmem_ld_x8;
using tc2::tmem_st_x8;
using tc2::tmem_wait_st;

constexpr int kThreads = 384;      // warpgroups 0-1 softmax, warp 8 TMA, warps 9-10 MMA
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;        // warp 9 + g issues the G and S MMAs of warpgroup g
constexpr int kSoftmaxRegs = tc::kSoftmaxRegs;
constexpr int kProducerRegs = tc::kProducerRegs;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;  // warpgroup g owns columns [256g, 256g + 256)
constexpr uint32_t kOCol = 192;      // O accumulators (two A.V streams) at [192, 192 + 2d)
// A.V: one accumulator [O | row sums] of d + 8 columns: the B operand is
// [V | ones], the ones tile's 8 columns returning the row sum of the very
// bf16 P the MMA consumed (no per-logit additions in the softmax).
constexpr float kRescale = 8.0f;     // move the running maximum when exceeded by this (log2 units)
constexpr uint64_t kWaitNs = tc::kWaitNs;

struct Params {
  // output tensor map: box {d, block, 32 / block, 1} = one warp's 32 query
  // rows (used when tma_out is set)
  CUtensorMap tmap_o;
  const __nv_bfloat16* rel_h;
  const __nv_bfloat16* rel_w;
  __nv_bfloat16* out;
  int N, H, W, heads, halo;
  int nbx, nby;
  int num_items;   // N * nby * nbx * heads
  int stages;
  int tma_out;     // 1: the epilogue stages each warp's rows in shared memory and stores them by TMA
  float c;         // log2(e) / sqrt(d)
};

template <int D, int WIN, int BLOCK>
struct Cfg {
  static constexpr int kBlock = BLOCK;
  static constexpr int QROWS = 256 / BLOCK;               // query rows of the block per item
  static constexpr int NQUART = BLOCK / QROWS;            // items per block and head (1 or 4)
  // S buffers at slot columns [0, kBufCols) and [kBufCols, 2 kBufCols)
  static constexpr uint32_t kBufCols = (BLOCK == 16) ? 96 : 80;
  static constexpr int kChunkRows = (BLOCK == 16) ? 4 : 2;   // window rows per key chunk
  // R tile: rel_h rows [0, 2w-1), rel_w rows [kRelW, kRelW + 2w-1)
  static constexpr int kRRows = (BLOCK == 16) ? 96 : 160;
  static constexpr int kRelW = (BLOCK == 16) ? 48 : 80;
  static constexpr bool kGBothBufs = (BLOCK == 32);      // G spans both S buffers
  static constexpr int ROWB = D * 2;
  // Keys per window row in shared memory: the window width, or at block 32
  // the width rounded up to 8 so that every 2-row chunk starts on a swizzle
  // atom (the TMA box loads the extra columns; they are masked out).
  static constexpr int WP = (BLOCK == 16) ? WIN : (WIN + 7) / 8 * 8;
  static constexpr int KS = WP * WIN;                      // keys the TMA writes per tile
  static constexpr int NCH = (WIN + kChunkRows - 1) / kChunkRows;
  __host__ __device__ static constexpr int rows(int c) { return (c + 1 < NCH) ? kChunkRows : WIN - kChunkRows * (NCH - 1); }
  __host__ __device__ static constexpr int start(int c) { return kChunkRows * WP * c; }      // first key of chunk c
  __host__ __device__ static constexpr int keys(int c) { return rows(c) * WP; }
  __host__ __device__ static constexpr int ns(int c) { return (keys(c) + 15) / 16 * 16; }    // S MMA N = P keys incl. padding
  __host__ __device__ static constexpr int nbuf(int b) { return (NCH + 1 - b) / 2; }         // chunks using buffer b per item
  static constexpr int KPAD = start(NCH - 1) + ns(NCH - 1);              // K / V rows incl. zero padding
  static constexpr int Q_TILE = 256 * ROWB;
  static constexpr int K_TILE = (KPAD * ROWB + 1023) / 1024 * 1024;
  static constexpr int STAGE_BYTES = Q_TILE + 2 * K_TILE;
  static constexpr int R_TILE = (kRRows * ROWB + 1023) / 1024 * 1024;
  static constexpr int TX_BYTES = (256 + 2 * KS) * ROWB;
  static constexpr SmemSwizzle SW = (ROWB == 32) ? SW_32B : (ROWB == 64 ? SW_64B : SW_128B);
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int HALO = (WIN - kBlock) / 2;
  static_assert(BLOCK == 16 || BLOCK == 32, "block 16 or 32");
  static_assert(D == 16 || D == 32, "dim_head 16 or 32");
  static_assert(WIN % 2 == 0 && WIN >= kBlock && WIN <= kBlock + 8 && WIN <= 38, "window b..b+6 (b=32), b..b+8 (b=16)");
  static_assert(ns(0) <= (int)kBufCols, "S chunk in one buffer");
  static_assert(2 * kBufCols <= kOCol, "S buffers below the O accumulators");
  static_assert(!kGBothBufs || kRRows <= 2 * (int)kBufCols, "G inside the two S buffers");
  static_assert(kGBothBufs || kRRows <= (int)kBufCols, "G inside one S buffer");
  static constexpr int ON = D + 8;                                       // A.V N: V and the ones columns
  static constexpr int ONES_BYTES = ((kChunkRows * WP + 15) / 16 * 16 * ROWB + 1023) / 1024 * 1024;
  static constexpr int OUT_WARP = 32 * ROWB;        // one softmax warp's output rows (TMA store staging)
  static constexpr int OUT_BYTES = 8 * OUT_WARP;
  static_assert(kOCol + ON <= kSlotCols, "O accumulator in the slot");
  static_assert(2 * WIN - 1 <= kRelW && kRelW + 2 * WIN - 1 <= kRRows, "relative table rows");
  static_assert((kChunkRows * WP) % 8 == 0, "chunk starts on a swizzle atom");
  static_assert(WP % 2 == 0 && WP <= 40, "row pitch");
};

template <int D, int WIN, int BLOCK>
__host__ __device__ constexpr int smem_bytes(int stages) {
  using C = Cfg<D, WIN, BLOCK>;
  return 1024 + C::R_TILE + stages * C::STAGE_BYTES + C::ONES_BYTES;
}

// Window-column pairs (kc, kc+1), kc even, whose exponentials take the
// polynomial: inside the block's own columns [h, h+b), which are never
// outside the image.  Bit kc/2 of the mask.  Measured balance of MUFU and
// FMA-pipe issue (row sums from the MMA): block 16, 4 of 12 pairs (large
// workload 549 / 542 / 539 / 563 / 582 us with 2 / 3 / 4 / 5 / 6); block 32,
// 6 of 20 (block 32 halo 3: 398 / 395 / 411 with 4 / 6 / 8).
#ifndef HALO_TC3_POLY_PAIRS
#define HALO_TC3_POLY_PAIRS 4
#endif
#ifndef HALO_TC3_POLY_PAIRS_B32
#define HALO_TC3_POLY_PAIRS_B32 6
#endif
template <int WIN, int BLOCK>
__host__ __device__ constexpr unsigned poly_pair_mask() {
  constexpr int h = (WIN - BLOCK) / 2;
  const int npairs = (BLOCK == 32) ? HALO_TC3_POLY_PAIRS_B32 : HALO_TC3_POLY_PAIRS;
  unsigned m = 0;
  int picked = 0;
  const int mid = (h + BLOCK / 2 - 1) & ~1;
  for (int d = 0; d < BLOCK && picked < npairs; ++d) {
    const int kc = mid + ((d & 1) ? -2 * ((d + 1) / 2) : 2 * (d / 2));
    if (kc >= h && kc + 1 < h + BLOCK && !((m >> (kc / 2)) & 1u)) {
      m |= 1u << (kc / 2);
      ++picked;
    }
  }
  return m;
}

// A wait's outcome, the same for every lane of the warp (a warp-collective
// tcgen05 instruction must not be reached by part of a warp).
__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

struct ItemCoord {
  int n, by, bx, head, quart;  // quart: which QROWS query rows of the block
};
template <int NQUART>
__device__ __forceinline__ ItemCoord item_coord(int item, int heads, int nbx, int nby) {
  ItemCoord c;
  c.quart = item % NQUART;
  const int hb = item / NQUART;
  c.head = hb % heads;
  const int blk = hb / heads;
  c.bx = blk % nbx;
  c.by = (blk / nbx) % nby;
  c.n = blk / (nbx * nby);
  return c;
}

template <int D, int WIN, int BLOCK>
__global__ void __launch_bounds__(kThreads, 1)
    halo_fwd_tc3(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ Params p) {
  using C = Cfg<D, WIN, BLOCK>;
  constexpr int kBlock = C::kBlock;
  constexpr uint32_t kBufCols = C::kBufCols;
  constexpr int kChunkRows = C::kChunkRows;
  constexpr int kRRows = C::kRRows;
  constexpr int kRelW = C::kRelW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sR = smem;
  uint8_t* sStage = smem + C::R_TILE;
  // stage layout: [Q 256 rows][K KPAD rows][V KPAD rows]
  constexpr int OFF_Q = 0, OFF_K = C::Q_TILE, OFF_V = C::Q_TILE + C::K_TILE;

  // Per warpgroup g, chunk t = k * NCH + c of its k-th item uses S buffer
  // t & 1; sfull / bfree of a buffer complete once per chunk on it, so the
  // phase of chunk t is t >> 1.
  __shared__ __align__(8) uint64_t bar_full[4];
  __shared__ __align__(8) uint64_t bar_empty[4];     // count 2: both warpgroups' last chunk
  __shared__ __align__(8) uint64_t bar_gfull[2];     // G MMA done
  __shared__ __align__(8) uint64_t bar_gfree[2];     // count 4: the warpgroup loaded G
  __shared__ __align__(8) uint64_t bar_sfull[2][2];  // S of the chunk in buffer b done
  __shared__ __align__(8) uint64_t bar_bfree[2][2];  // the A.V of that chunk done
  // count 4: P of chunk t stored, alternating by t & 1: a warp can be one
  // chunk ahead of another (its arrival for chunk t+1 must not complete the
  // phase of chunk t), never two (chunk t+2's S needs chunk t's A.V)
  __shared__ __align__(8) uint64_t bar_pready[2][2];
  __shared__ __align__(8) uint64_t bar_ofull[2];     // the item's last A.V done
  __shared__ __align__(8) uint64_t bar_done[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.stages;
  uint8_t* sOnes = sStage + S * C::STAGE_BYTES;  // after every stage: positive LBO from any V chunk
  uint8_t* sOut = sOnes + C::ONES_BYTES;         // output staging (when p.tma_out)

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 2);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bar_gfull[g], 1);
      mbar_init(&bar_gfree[g], 4);
      mbar_init(&bar_sfull[g][0], 1);
      mbar_init(&bar_sfull[g][1], 1);
      mbar_init(&bar_bfree[g][0], 1);
      mbar_init(&bar_bfree[g][1], 1);
      mbar_init(&bar_pready[g][0], 4);
      mbar_init(&bar_pready[g][1], 4);
      mbar_init(&bar_ofull[g], 1);
      mbar_init(&bar_done[g], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  // R tile (written once) and the K / V padding rows the TMA never writes
  for (int idx = tid; idx < kRRows * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), u = idx % (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < 2 * WIN - 1) val = *reinterpret_cast<const uint4*>(p.rel_h + r * D + u * 8);
    else if (r >= kRelW && r < kRelW + 2 * WIN - 1)
      val = *reinterpret_cast<const uint4*>(p.rel_w + (r - kRelW) * D + u * 8);
    *reinterpret_cast<uint4*>(sR + swz<C::ROWB>(r, u)) = val;
  }
  // ones tile (bf16 1.0 in every element, so the swizzle does not matter)
  for (int idx = tid; idx < C::ONES_BYTES / 16; idx += kThreads)
    reinterpret_cast<uint4*>(sOnes)[idx] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  for (int s = 0; s < S; ++s) {
    uint8_t* st = sStage + s * C::STAGE_BYTES;
    for (int idx = tid; idx < (C::KPAD - C::KS) * C::ROWB / 16; idx += kThreads) {
      reinterpret_cast<uint4*>(st + OFF_K + C::KS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(st + OFF_V + C::KS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const int my_items = (p.num_items > (int)blockIdx.x)
                           ? (p.num_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int k = 0; k < my_items; ++k) {
        const int s = k % S;
        if (k >= S && !mbar_wait(&bar_empty[s], ((k / S) - 1) & 1, kWaitNs, &abort_flag)) {
          if (!abort_flag) record_timeout(&abort_flag);
          break;
        }
        const ItemCoord ic = item_coord<C::NQUART>(blockIdx.x + k * gridDim.x, p.heads, p.nbx, p.nby);
        uint8_t* st = sStage + s * C::STAGE_BYTES;
        const int x0 = ic.bx * kBlock, y0 = ic.by * kBlock;
        mbar_arrive_expect_tx(&bar_full[s], C::TX_BYTES);
        tma_load_4d(st + OFF_Q, &tmap_q, &bar_full[s], ic.head * D, x0, y0 + ic.quart * C::QROWS, ic.n);
        tma_load_4d(st + OFF_K, &tmap_k, &bar_full[s], ic.head * D, x0 - p.halo, y0 - p.halo, ic.n);
        tma_load_4d(st + OFF_V, &tmap_v, &bar_full[s], ic.head * D, x0 - p.halo, y0 - p.halo, ic.n);
        issued = k + 1;
      }
      if (abort_flag) {
        for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
          mbar_wait(&bar_full[k % S], (k / S) & 1, kWaitNs);
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ------------------------------------------------------------ G, S and A.V MMAs of warpgroup g
    // Chunk by chunk: S of chunk t, then, once the warpgroup has stored P of
    // chunk t - 1, that chunk's A.V (the softmax warps only arrive on
    // pready and go on to chunk t).
    const int g = warp - kMmaWarp;
    if (lane == 0) {
      const uint32_t slot = tmem + g * kSlotCols;
      const uint32_t idG = idesc_bf16_f32(128, kRRows, false);
      const uint32_t idO = idesc_bf16_f32(128, C::ON, true);
      const uint32_t ra = smem_addr(sR);
      // A.V of chunk c of item k into [O | row sums]
      auto issue_av = [&](int k, int c) -> bool {
        const int t = k * C::NCH + c, b = t & 1;
        if (!mbar_wait(&bar_pready[g][b], (t >> 1) & 1, kWaitNs, &abort_flag)) return false;
        tc_fence_after();
        const int ksteps = (C::rows(c) * C::WP + 15) / 16;
        const uint32_t va = smem_addr(sStage + (k % S) * C::STAGE_BYTES + OFF_V + C::start(c) * C::ROWB);
        // B = [V | ones]: the ones atom at leading byte offset lbo, same row pitch
        const uint32_t lbo = smem_addr(sOnes) - va;
#pragma unroll 1
        for (int kk = 0; kk < ksteps; ++kk)
          mma_f16_ts(slot + kOCol, slot + b * kBufCols + 8 * kk, smem_desc(va + kk * 16 * C::ROWB, lbo, C::SBO, C::SW),
                     idO, (c > 0 || kk > 0));
        mma_commit(&bar_bfree[g][b]);
        if (c + 1 == C::NCH) {
          mma_commit(&bar_ofull[g]);
          mma_commit(&bar_empty[k % S]);
        }
        return true;
      };
      // G of item k into the buffer of its first chunk (free once chunk
      // t0 - 2's A.V is done; block 32: G spans both buffers, the other one
      // frees with chunk t0 - 1's A.V)
      auto issue_g = [&](int k) -> bool {
        const int s = k % S, t0 = k * C::NCH;
        bool got = mbar_wait(&bar_full[s], (k / S) & 1, kWaitNs, &abort_flag);
        if (got && t0 >= 2) got = mbar_wait(&bar_bfree[g][t0 & 1], ((t0 - 2) >> 1) & 1, kWaitNs, &abort_flag);
        if (C::kGBothBufs && got && t0 >= 1)
          got = mbar_wait(&bar_bfree[g][(t0 - 1) & 1], ((t0 - 1) >> 1) & 1, kWaitNs, &abort_flag);
        if (!got) return false;
        tc_fence_after();
        const uint32_t qa = smem_addr(sStage + s * C::STAGE_BYTES + OFF_Q + g * 128 * C::ROWB);
        const uint32_t gdst = slot + (C::kGBothBufs ? 0u : (t0 & 1) * kBufCols);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_f16_ss(gdst, smem_desc(qa + 32 * ks, 16, C::SBO, C::SW),
                     smem_desc(ra + 32 * ks, 16, C::SBO, C::SW), idG, ks != 0);
        mma_commit(&bar_gfull[g]);
        return true;
      };
      bool ok = my_items > 0 ? issue_g(0) : true;
      for (int k = 0; k < my_items && ok; ++k) {
        const int s = k % S, t0 = k * C::NCH;
        const uint8_t* st = sStage + s * C::STAGE_BYTES;
        const uint32_t qa = smem_addr(st + OFF_Q + g * 128 * C::ROWB);
        const uint32_t ka = smem_addr(st + OFF_K);
#pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          const int t = t0 + c, b = t & 1;
          if (c == 0) ok = mbar_wait(&bar_gfree[g], k & 1, kWaitNs, &abort_flag);
          else if (t >= 2) ok = mbar_wait(&bar_bfree[g][b], ((t - 2) >> 1) & 1, kWaitNs, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          const int n = (c + 1 < C::NCH) ? C::ns(0) : C::ns(C::NCH - 1);
          const uint32_t idS = idesc_bf16_f32(128, n, false);
          const uint32_t kb = ka + C::start(c) * C::ROWB;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_f16_ss(slot + b * kBufCols, smem_desc(qa + 32 * ks, 16, C::SBO, C::SW),
                       smem_desc(kb + 32 * ks, 16, C::SBO, C::SW), idS, ks != 0);
          mma_commit(&bar_sfull[g][b]);
          if (c > 0 && !(ok = issue_av(k, c - 1))) break;
        }
        if (!ok) break;
        // the next item's G, then this item's last A.V: the softmax gathers
        // the next item's relative logits while the last chunk finishes
        // (block 32: G needs the last chunk's buffer too, so it comes after)
        if constexpr (!C::kGBothBufs) {
          if (k + 1 < my_items) ok = issue_g(k + 1);
          if (ok) ok = issue_av(k, C::NCH - 1);
        } else {
          ok = issue_av(k, C::NCH - 1);
          if (ok && k + 1 < my_items) ok = issue_g(k + 1);
        }
      }
      if (!ok && !abort_flag) record_timeout(&abort_flag);
      mma_commit(&bar_done[g]);
      mbar_wait(&bar_done[g], 0, kWaitNs);
    }
  }
  __syncwarp();
  tc_fence_before();
  named_bar_sync(1, kThreads);
  return;
  }

  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
  {
    // ------------------------------------------------------------ softmax warpgroups
    const int g = warp >> 2;               // warpgroup = TMEM slot = half of the item's query rows
    const int wq = warp & 3;               // lane quadrant
    // query row among the item's QROWS rows, and column in the block: block
    // 16 puts two query rows in a warp (16 lanes each), block 32 one
    const int yq = (kBlock == 16) ? 8 * g + 2 * wq + (lane >> 4) : 4 * g + wq;
    const int xl = (kBlock == 16) ? (lane & 15) : lane;
    const uint32_t slot = tmem + g * kSlotCols;    // lane 0 of the slot (MMA operands)
    const uint32_t ts = slot + (static_cast<uint32_t>(32 * wq) << 16);  // this warp's lanes
    const float c = p.c;
    const int C_all = p.heads * D;
    constexpr unsigned kPoly = poly_pair_mask<WIN, kBlock>();

    float rhc[WIN], rwc[C::WP];
    // ---- relative logits of item k: rhc[kr] = c * q.rel_h[kr - qy + w - 1], rwc[kc] likewise
    auto gather = [&](int k) -> bool {
      if (!warp_ok(mbar_wait(&bar_gfull[g], k & 1, kWaitNs, &abort_flag))) return false;
      tc_fence_after();
      const ItemCoord ic = item_coord<C::NQUART>(blockIdx.x + k * gridDim.x, p.heads, p.nbx, p.nby);
      const int y0 = ic.by * kBlock - p.halo, x0 = ic.bx * kBlock - p.halo;
      const uint32_t gcol = C::kGBothBufs ? 0u : ((k * C::NCH) & 1) * kBufCols;
      float a[WIN + kBlock - 1];
      if constexpr (kBlock == 16) {
        // rel_h: columns [base, base + 32) of G hold every row this warp needs;
        // the two query rows of the warp differ by one column
        const int base = WIN - 2 - 8 * g - 2 * wq;
        float gh[32], gw[48];
        tmem_ld_x32(ts + gcol + base, gh);
        tmem_ld_x32(ts + gcol + kRelW, gw);
        tmem_ld_x8(ts + gcol + kRelW + 32, gw + 32);
        tmem_ld_x8(ts + gcol + kRelW + 40, gw + 40);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_gfree[g]);
        const bool odd = (lane >> 4) != 0;
#pragma unroll
        for (int kr = 0; kr < WIN; ++kr) {
          const int Y = y0 + kr;
          const float v = odd ? gh[kr] : gh[kr + 1];
          rhc[kr] = (Y >= 0 && Y < p.H) ? v * c : -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < WIN + 15; ++i) a[i] = gw[WIN - 16 + i];
      } else {
        // rel_h: one query row per warp, the whole shift in the load address
        const int qy = ic.quart * C::QROWS + yq;
        float gh[40], gw[72];
        tmem_ld_x32(ts + gcol + (WIN - 1 - qy), gh);
        tmem_ld_x8(ts + gcol + (WIN - 1 - qy) + 32, gh + 32);
        tmem_ld_x32(ts + gcol + kRelW + WIN - 32, gw);
        tmem_ld_x32(ts + gcol + kRelW + WIN, gw + 32);
        tmem_ld_x8(ts + gcol + kRelW + WIN + 32, gw + 64);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_gfree[g]);
#pragma unroll
        for (int kr = 0; kr < WIN; ++kr) {
          const int Y = y0 + kr;
          rhc[kr] = (Y >= 0 && Y < p.H) ? gh[kr] * c : -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < WIN + 31; ++i) a[i] = gw[i];
      }
      // rel_w: the b query columns need b different shifts; a barrel shifter
      // of selects over G[rel_w + w - b + i] by sh = b - 1 - qx
      const int sh = kBlock - 1 - xl;
      if constexpr (kBlock == 32) {
#pragma unroll
        for (int i = 0; i < WIN + 15; ++i) a[i] = (sh & 16) ? a[i + 16] : a[i];
      }
#pragma unroll
      for (int i = 0; i < WIN + 7; ++i) a[i] = (sh & 8) ? a[i + 8] : a[i];
#pragma unroll
      for (int i = 0; i < WIN + 3; ++i) a[i] = (sh & 4) ? a[i + 4] : a[i];
#pragma unroll
      for (int i = 0; i < WIN + 1; ++i) a[i] = (sh & 2) ? a[i + 2] : a[i];
#pragma unroll
      for (int i = 0; i < WIN; ++i) a[i] = (sh & 1) ? a[i + 1] : a[i];
#pragma unroll
      for (int kc = 0; kc < C::WP; ++kc) {
        const int X = x0 + kc;
        rwc[kc] = (kc < WIN && X >= 0 && X < p.W) ? a[kc] * c : -INFINITY;  // row padding masked
      }
      return true;
    };

    // ---- one key chunk (NR window rows; rhc[0..NR) are its rows' rel_h logits)
    float m_run = -INFINITY;
    auto chunk = [&](auto nr, int k, int cidx) -> bool {
      constexpr int NR = decltype(nr)::value;
      constexpr int WP = C::WP;
      constexpr int NK = NR * WP, NL = (NK + 7) / 8 * 8, NP = NK / 2, NW = (NK + 15) / 16 * 8;
      const int t = k * C::NCH + cidx, b = t & 1;
      const uint32_t buf = ts + b * kBufCols;
      if (!warp_ok(mbar_wait(&bar_sfull[g][b], (t >> 1) & 1, kWaitNs, &abort_flag))) return false;
      tc_fence_after();
      float z[NL];
      tmem_ld_cols<NL>(buf, z);
      tmem_wait_ld();
      // y = c*S + c*rel_w (pairs); chunk maximum of y + c*rel_h
      float2 y[NP];
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int kc = (2 * i) % WP;
        y[i] = __ffma2_rn(make_float2(z[2 * i], z[2 * i + 1]), make_float2(c, c), make_float2(rwc[kc], rwc[kc + 1]));
      }
      float mc = -INFINITY;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        float mr = -INFINITY;
#pragma unroll
        for (int i = r * WP / 2; i < (r + 1) * WP / 2; ++i) mr = max3f(mr, y[i].x, y[i].y);
        mc = fmaxf(mc, mr + rhc[r]);
      }
      const bool upd = mc > m_run + kRescale;
      // O and its row sums hold earlier chunks against m_run: rescale them
      // when the maximum moves (a row whose earlier chunks had no in-image key
      // has O = 0, sums included)
      if (__any_sync(0xffffffffu, upd && m_run != -INFINITY && cidx > 0)) {
        const int tp = t - 1;
        if (!warp_ok(mbar_wait(&bar_bfree[g][tp & 1], (tp >> 1) & 1, kWaitNs, &abort_flag))) return false;
        tc_fence_after();
        const float alpha = (upd && m_run != -INFINITY) ? exp2_mufu(m_run - mc) : 1.0f;
        // eight columns at a time: y[] is live, registers are short
#pragma unroll 1
        for (int e = 0; e < C::ON; e += 8) {
          float o[8];
          tmem_ld_x8(ts + kOCol + e, o);
          tmem_wait_ld();
          uint32_t ob[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) ob[i] = __float_as_uint(o[i] * alpha);
          tmem_st_x8(ts + kOCol + e, ob);
        }
      }
      if (upd) m_run = mc;
      const float mb = (m_run == -INFINITY ? 0.f : m_run);
      // exponentials, packed bf16 P over the chunk's S columns (the row sum
      // comes from the A.V's ones columns)
      uint32_t pk[NW];
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int r = (2 * i) / WP, kc = (2 * i) % WP;
        const float bias = rhc[r] - mb;
        const float2 x = __fadd2_rn(y[i], make_float2(bias, bias));
        uint32_t rx, ry;
        if ((kPoly >> (kc / 2)) & 1u) {
          exp2_poly2(x, rx, ry);
        } else {
          rx = __float_as_uint(exp2_mufu(x.x));
          ry = __float_as_uint(exp2_mufu(x.y));
        }
        pk[i] = pack_p(rx, ry);
      }
#pragma unroll
      for (int i = NP; i < NW; ++i) pk[i] = 0u;
#pragma unroll
      for (int i = 0; i < NW; i += 8) tmem_st_x8(buf + i, pk + i);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_pready[g][b]);
      // (the chunk's A.V is issued by the warpgroup's MMA warp)
      // next chunk's rows first
#pragma unroll
      for (int i = 0; i + NR < WIN; ++i) rhc[i] = rhc[i + NR];
      return true;
    };

    constexpr int kLastRows = C::rows(C::NCH - 1);
    constexpr int kLoopChunks = (kLastRows == kChunkRows) ? C::NCH : C::NCH - 1;
    bool ok = my_items > 0 ? gather(0) : true;
    for (int k = 0; k < my_items && ok; ++k) {
      const ItemCoord ic = item_coord<C::NQUART>(blockIdx.x + k * gridDim.x, p.heads, p.nbx, p.nby);
      m_run = -INFINITY;
#pragma unroll 1
      for (int ci = 0; ci < kLoopChunks && ok; ++ci) ok = chunk(std::integral_constant<int, kChunkRows>{}, k, ci);
      if constexpr (kLoopChunks < C::NCH) {
        if (ok) ok = chunk(std::integral_constant<int, kLastRows>{}, k, C::NCH - 1);
      }
      // the next item's relative logits while this item's last A.V runs
      // (block 32: G needs both S buffers, so it follows the epilogue)
      if (!C::kGBothBufs && ok && k + 1 < my_items) ok = gather(k + 1);
      // ---- epilogue: O / l, bf16, NHWC
      if (ok) ok = warp_ok(mbar_wait(&bar_ofull[g], k & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      {
        float o[C::ON];
        tmem_ld_cols<C::ON>(ts + kOCol, o);
        tmem_wait_ld();
        const float inv = 1.0f / o[D];  // row sum of the bf16 P (ones columns)
        uint32_t pk[D / 2];
#pragma unroll
        for (int t = 0; t < D / 2; ++t)
          pk[t] = pack_bf16x2(o[2 * t] * inv, o[2 * t + 1] * inv);
        if (p.tma_out) {
          // the warp's 32 rows (lane = row of its box) through shared memory,
          // one TMA store per warp: coalesced, and the warp does not wait
          uint8_t* stg = sOut + warp * C::OUT_WARP;
          if (lane == 0) bulk_wait_read_all();  // the previous store has read the buffer
          __syncwarp();
#pragma unroll
          for (int t = 0; t < D / 8; ++t)
            *reinterpret_cast<uint4*>(stg + swz<C::ROWB>(lane, t)) =
                make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int y0w = ic.by * kBlock + ic.quart * C::QROWS + (kBlock == 16 ? 8 * g + 2 * wq : 4 * g + wq);
            tma_store_4d(&p.tmap_o, stg, ic.head * D, ic.bx * kBlock, y0w, ic.n);
            bulk_commit_group();
          }
        } else {
          const int y = ic.by * kBlock + ic.quart * C::QROWS + yq, x = ic.bx * kBlock + xl;
          __nv_bfloat16* dst = p.out + ((static_cast<size_t>(ic.n) * p.H + y) * p.W + x) * C_all + ic.head * D;
#pragma unroll
          for (int t = 0; t < D / 8; ++t)
            reinterpret_cast<uint4*>(dst)[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        }
      }
      tc_fence_before();
      if (C::kGBothBufs && k + 1 < my_items) ok = gather(k + 1);
    }
    if (!ok && !abort_flag) record_timeout(&abort_flag);
    if (p.tma_out && lane == 0) bulk_wait_all();  // this warp's output stores are complete
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  named_bar_sync(1, kThreads);
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc3
}  // namespace halo
