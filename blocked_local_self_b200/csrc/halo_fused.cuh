// halo_fused.cuh -- blocked local self-attention with haloing whose q, k, v
// projections run inside the kernel (sm_100a, bf16, 8x8 query blocks,
// stride 1, dim_head 16 or 32, c_in 64 or 128, maps with an even number of
// block rows).
//
// The blog page's HaloAttention forms q = to_q(x) and [k | v] = to_kv(x) with
// bias-free linear maps of the input map x, then the operation (HaloNet,
// "Scaling Local Self-Attention for Parameter Efficient Visual Backbones",
// sections 2.1-2.2; appendix D: fusing around the op and avoiding format
// operations is where the paper's speed-ups came from).  Here x is read
// (the query blocks and the haloed window, by TMA, zero outside the image)
// instead of separately stored q, k and v:
//   * work item = two vertically adjacent 8x8 blocks of one head, ordered so
//     that one CTA takes every head of a block pair in turn: the pair's x
//     tiles (its 128 query pixels and the (w+8) x w union window, c_in
//     channels in 64-channel swizzle atoms) are loaded once for all heads;
//     the head's weight rows (wq, and the k and v halves of wkv: d x c_in
//     each, the linear layers' [out, in] layout, i.e. K-major B operands) per
//     item.
//   * projection round (lane 0 of three warps of the item's warpgroup):
//     Q = x_q Wq_h^T (M=128: both blocks' queries) and [K_t | V_t] =
//     x_kv[tile t] [Wk_h; Wv_h]^T (one N = 2d MMA chain per 128-row tile of
//     the union window), fp32 into the warpgroup's TMEM slot.
//   * the warpgroup reads them back (one TMEM lane = one row), rounds to
//     bf16 (as an unfused pipeline would store q, k, v) and writes the Q_A,
//     Q_B, K and V tiles of the two-block kernel (halo_tc4.cuh) into shared
//     memory; pixels outside the image have x = 0 and so k = v = 0.
//   * from there the two-block pipeline: S (block A on warp 0, block B on
//     warp 1) and G = Q R^T (warp 2), the two-pass softmax with the bound
//     and its exact fallback, bf16 P over the S columns, four A.V chains with
//     the ones tile for the row sums, the NHWC epilogue.
// Two warpgroups take alternate items; a TMA warp streams x and the weights;
// every wait is bounded and reports HALO_ERR_TIMEOUT.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "halo_tc.cuh"
#include "halo_tc2.cuh"
#include "halo_tc4.cuh"
#include "sm100.cuh"

namespace halo {
namespace fused {

using namespace sm100;
using tc::exp2_mufu;
using tc::pack_bf16x2;
using tc::record_timeout;
using tc::swz;
using tc2::mma_f16_ts;
using tc2::tmem_ld_x32;
using tc2::tmem_ld_x8;
using tc4::exact_row_max;
using tc4::exp_pipelined;
using tc4::own_pair;
using tc4::row_max_pipelined;
using tc4::tmem_ld_exact;
using tc4::tmem_ld_x1;

constexpr int kBlock = 8;
constexpr int kThreads = 384;        // warpgroups 0-1 compute, warpgroup 2 conversion (warp 8 also TMA)
constexpr int kTmaWarp = 8;
constexpr int kSoftmaxRegs = 200;
constexpr int kProducerRegs = 96;    // the conversion warps hold a tile row's q, k and v
static_assert(256 * kSoftmaxRegs + 128 * kProducerRegs <= kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;
constexpr uint32_t kGBase = tc4::kGBase;  // 200
constexpr int kRelW = tc4::kRelW;         // 28
constexpr int kRRows = 56;
constexpr uint64_t kWaitNs = tc::kWaitNs;

struct Params {
  const __nv_bfloat16* rel_h;
  const __nv_bfloat16* rel_w;
  __nv_bfloat16* out;
  int N, H, W, heads, halo;
  int nbx, npy;       // blocks along x, block pairs along y
  int num_pairs;      // N * npy * nbx
  int xstages;        // x pipeline stages (1 or 2)
  float c;            // log2(e) / sqrt(d)
};

template <int D, int WIN, int CIN>
struct Cfg {
  using A = tc4::Cfg<D, WIN>;                           // the attention part's layout
  static constexpr int KA = CIN / 64;                    // 64-channel atoms of x and the weights
  static constexpr int UROWS = A::UROWS;                 // (w + 8) w window pixels
  static constexpr int KVT = (UROWS + 127) / 128;        // 128-row projection tiles of the window
  static constexpr int XQ_ATOM = 128 * 128;              // 128 query pixels x 64 channels, bf16
  static constexpr int XKV_ATOM = KVT * 128 * 128;       // window pixels (padded to KVT tiles) x 64 channels
  static constexpr int XSTAGE = KA * (XQ_ATOM + XKV_ATOM);
  static constexpr int TX_X = KA * (128 + UROWS) * 128;
  // The head's weights per 64-channel atom: Wq_h (d rows), and Wk_h over
  // Wv_h (2d rows), so that one N = 2d MMA projects k and v of a tile.
  static constexpr int W_ATOM = D * 128;                 // d rows x 64 channels
  static constexpr int WKV_ATOM = 2 * W_ATOM;
  static constexpr int OFF_WKV = KA * W_ATOM;            // the [Wk_h; Wv_h] atoms after the Wq_h atoms
  static constexpr int W_BYTES = 3 * KA * W_ATOM;
  // converted attention tiles of one warpgroup: Q_A, Q_B, K union, V union
  static constexpr int OFF_QA = 0, OFF_QB = A::Q_TILE, OFF_K = 2 * A::Q_TILE, OFF_V = 2 * A::Q_TILE + A::K_TILE;
  static constexpr int TILES = 2 * A::Q_TILE + 2 * A::K_TILE;
  static constexpr int WG_BYTES = (TILES + W_BYTES + 1023) / 1024 * 1024;
  static constexpr int R_TILE = A::R_TILE;
  // EARLY (d = 16): O goes to the relative-logit columns, so that after an
  // item's exponent pass the S columns past P are dead until the next S: the
  // next item's K and V projections are issued there as soon as this item's
  // A.V is issued, and its Q projection into P's first columns once the A.V
  // is done; the projections then overlap this item's A.V and epilogue.
  // Otherwise all three are issued at the start of the item: Q at 0, K and V
  // after it.
  static constexpr bool EARLY = (int)kGBase + 2 * A::ON <= (int)kSlotCols &&
                                A::O_BASE + 2 * KVT * D <= (int)kGBase;
  static constexpr uint32_t COL_Q = 0;
  static constexpr uint32_t COL_K = EARLY ? A::O_BASE : D;
  static constexpr uint32_t COL_V = COL_K + KVT * 2 * D;  // end of the [k | v] tile columns
  static constexpr uint32_t O_COL = EARLY ? kGBase : A::O_BASE;
  static_assert(CIN == 64 || CIN == 128, "c_in 64 or 128");
  static_assert(D == 16 || D == 32, "dim_head 16 or 32");
  static_assert(COL_V <= kSlotCols, "projections in the slot");
  static_assert(A::KROWS <= KVT * 128, "window tiles cover the rows the MMAs read");
};

template <int D, int WIN, int CIN>
__host__ __device__ constexpr int smem_bytes(int xstages) {
  using C = Cfg<D, WIN, CIN>;
  return 1024 + C::R_TILE + C::A::ONES_BYTES + 2 * C::WG_BYTES + xstages * C::XSTAGE;
}

__device__ __forceinline__ bool warp_ok(bool ok) { return __all_sync(0xffffffffu, ok); }

// Barrier of one warpgroup's four warps on an mbarrier of count 4 (bounded).
__device__ __forceinline__ bool wg_sync(uint64_t* bar, int& ph, int lane, int* abort_flag) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = warp_ok(mbar_wait(bar, ph & 1, kWaitNs, abort_flag));
  ++ph;
  return ok;
}

// D consecutive TMEM columns of this thread's lane.
template <int D>
__device__ __forceinline__ void tmem_ld_d(uint32_t taddr, float* r) {
  if constexpr (D == 32) tmem_ld_x32(taddr, r);
  else tmem_ld_exact<D>(taddr, r);
}

// One row of D fp32 values as bf16 into row r of a K-major tile (rows of
// 2D bytes, the TMA / tcgen05 swizzle for that row size).
template <int D>
__device__ __forceinline__ void store_row(uint8_t* tile, int r, const float* v) {
#pragma unroll
  for (int u = 0; u < D / 8; ++u) {
    const uint4 val = make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                 pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
    *reinterpret_cast<uint4*>(tile + swz<2 * D>(r, u)) = val;
  }
}

template <int D, int WIN, int CIN>
__global__ void __launch_bounds__(kThreads, 1)
    halo_fused_tc(const __grid_constant__ CUtensorMap tmap_xq, const __grid_constant__ CUtensorMap tmap_xkv,
                  const __grid_constant__ CUtensorMap tmap_wq, const __grid_constant__ CUtensorMap tmap_wkv,
                  const Params p) {
  using C = Cfg<D, WIN, CIN>;
  using A = typename C::A;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sR = smem;
  uint8_t* sWG = sR + C::R_TILE;                           // [g][tiles | weights]
  uint8_t* sX = sWG + 2 * C::WG_BYTES;                     // [stage][atoms of x_q | atoms of x_kv]
  uint8_t* sOnes = sX + p.xstages * C::XSTAGE;             // after the V tiles: positive LBO from any of them

  __shared__ __align__(8) uint64_t bar_xfull[2];
  __shared__ __align__(8) uint64_t bar_wfull[2];
  __shared__ __align__(8) uint64_t bar_pr[2];      // count 3: Q, K, V projections
  __shared__ __align__(8) uint64_t bar_s[2];       // count 1: S_A, S_B, G
  __shared__ __align__(8) uint64_t bar_o[2];       // count 4: the A.V chains
  __shared__ __align__(8) uint64_t bar_tfree[2];   // count 4: the warpgroup has read its O
  __shared__ __align__(8) uint64_t bar_wg[2];      // count 4: the warps of warpgroup g
  __shared__ __align__(8) uint64_t bar_cv;         // count 4: the conversion warps
  __shared__ __align__(8) uint64_t bar_drain[9];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int XS = p.xstages;
  const int heads = p.heads;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < XS; ++i) mbar_init(&bar_xfull[i], 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bar_wfull[g], 1);
      mbar_init(&bar_pr[g], 3);
      mbar_init(&bar_s[g], 1);
      mbar_init(&bar_o[g], 4);
      mbar_init(&bar_tfree[g], 4);
      mbar_init(&bar_wg[g], 4);
    }
    mbar_init(&bar_cv, 4);
    for (int w = 0; w < 9; ++w) mbar_init(&bar_drain[w], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tmap_xq);
    prefetch_tensormap(&tmap_xkv);
    prefetch_tensormap(&tmap_wq);
    prefetch_tensormap(&tmap_wkv);
  }
  // R tile, ones tile, zeroed attention tiles and x stages (rows the TMA
  // never writes stay zero)
  for (int idx = tid; idx < kRRows * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), u = idx % (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < 2 * WIN - 1) val = *reinterpret_cast<const uint4*>(p.rel_h + r * D + u * 8);
    else if (r >= kRelW && r < kRelW + 2 * WIN - 1)
      val = *reinterpret_cast<const uint4*>(p.rel_w + (r - kRelW) * D + u * 8);
    *reinterpret_cast<uint4*>(sR + swz<A::ROWB>(r, u)) = val;
  }
  for (int idx = tid; idx < A::ONES_BYTES / 16; idx += kThreads)
    reinterpret_cast<uint4*>(sOnes)[idx] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  for (int idx = tid; idx < (2 * C::WG_BYTES + XS * C::XSTAGE) / 16; idx += kThreads)
    reinterpret_cast<uint4*>(sWG)[idx] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // this CTA's block pairs: blockIdx.x, blockIdx.x + gridDim.x, ...; every
  // head of a pair in turn (item j of the CTA: pair j / heads, head j % heads)
  const int my_pairs = (p.num_pairs > (int)blockIdx.x) ? (p.num_pairs - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int my_items = my_pairs * heads;

  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
  {
    // ------------------------------------------------------------ conversion warpgroup (warps 8-11)
    // Item by item (the two slots in turn): wait for the item's projections,
    // refill the weight buffer and the x stage they have released (TMA, lane
    // 0 of warp 8), wait until the slot's previous item has finished with the
    // attention tiles, round q, k, v to bf16 into them, then issue the item's
    // S and G MMAs (lane 0 of warp 9).  The softmax warpgroups meanwhile work
    // on the previous items.
    const int cw = warp - 8;  // TMEM lane quadrant
    auto load_x = [&](int pin) {
      const int pair = blockIdx.x + pin * gridDim.x;
      const int bx = pair % p.nbx, py = (pair / p.nbx) % p.npy, n = pair / (p.nbx * p.npy);
      const int sn = pin % XS;
      uint8_t* xs = sX + sn * C::XSTAGE;
      mbar_arrive_expect_tx(&bar_xfull[sn], C::TX_X);
      const int x0 = bx * kBlock, y0 = py * 2 * kBlock;
#pragma unroll 1
      for (int a = 0; a < C::KA; ++a) {
        tma_load_4d(xs + a * C::XQ_ATOM, &tmap_xq, &bar_xfull[sn], 64 * a, x0, y0, n);
        tma_load_4d(xs + C::KA * C::XQ_ATOM + a * C::XKV_ATOM, &tmap_xkv, &bar_xfull[sn], 64 * a, x0 - p.halo,
                    y0 - p.halo, n);
      }
    };
    auto load_w = [&](int jn) {
      const int head = jn % heads, gn = jn & 1;
      uint8_t* wb = sWG + gn * C::WG_BYTES + C::TILES;
      mbar_arrive_expect_tx(&bar_wfull[gn], C::W_BYTES);
#pragma unroll 1
      for (int a = 0; a < C::KA; ++a) {
        tma_load_2d(wb + a * C::W_ATOM, &tmap_wq, &bar_wfull[gn], 64 * a, head * D);
        tma_load_2d(wb + C::OFF_WKV + a * C::WKV_ATOM, &tmap_wkv, &bar_wfull[gn], 64 * a, head * D);
        tma_load_2d(wb + C::OFF_WKV + a * C::WKV_ATOM + C::W_ATOM, &tmap_wkv, &bar_wfull[gn], 64 * a,
                    heads * D + head * D);
      }
    };
    const bool tma_lane = (warp == kTmaWarp && lane == 0);
    const bool mma_lane = (warp == kTmaWarp + 1 && lane == 0);
    int nx = 0, nw = 0;  // loads issued (drained on an abort)
    if (tma_lane) {
      for (int pin = 0; pin < XS && pin < my_pairs; ++pin) {
        load_x(pin);
        nx = pin + 1;
      }
      for (int jn = 0; jn < 2 && jn < my_items; ++jn) {
        load_w(jn);
        nw = jn + 1;
      }
    }
    const uint32_t idS = idesc_bf16_f32(64, A::NS, false);
    const uint32_t idG = idesc_bf16_f32(64, kRRows, false);
    const uint32_t ra = smem_addr(sR);
    int cph = 0;
    bool ok = true;
    for (int j = 0; j < my_items && ok; ++j) {
      const int g = j & 1, jj = j >> 1;
      const int pi = j / heads, head = j % heads;
      ok = warp_ok(mbar_wait(&bar_pr[g], jj & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      // the projections of item j have read its weights, and, for the pair's
      // last head, the pair's x: refill both
      if (tma_lane) {
        if (j + 2 < my_items) {
          load_w(j + 2);
          nw = j + 3;
        }
        if (head == heads - 1 && pi + XS < my_pairs) {
          load_x(pi + XS);
          nx = pi + XS + 1;
        }
      }
      // the slot's previous item (j - 2) has finished its MMAs on the tiles
      if (j >= 2) {
        ok = warp_ok(mbar_wait(&bar_o[g], (jj - 1) & 1, kWaitNs, &abort_flag));
        if (!ok) break;
        tc_fence_after();
      }
      // ---- back to bf16 tiles: Q_A, Q_B (query rows), K and V (window rows)
      uint8_t* wgb = sWG + g * C::WG_BYTES;
      const uint32_t tsc = tmem + g * kSlotCols + (static_cast<uint32_t>(32 * cw) << 16);
      {
        float v[D];
        tmem_ld_d<D>(tsc + C::COL_Q, v);
        tmem_wait_ld();
        const int r = 32 * cw + lane;  // query pixel: rows 0-63 block A, 64-127 block B
        store_row<D>(wgb + (r < 64 ? C::OFF_QA : C::OFF_QB), r & 63, v);
#pragma unroll 1
        for (int t = 0; t < C::KVT; ++t) {
          float kv[D], vv[D];
          tmem_ld_d<D>(tsc + C::COL_K + t * 2 * D, kv);
          tmem_ld_d<D>(tsc + C::COL_K + t * 2 * D + D, vv);
          tmem_wait_ld();
          const int kr = 128 * t + 32 * cw + lane;
          if (kr < C::UROWS) {
            store_row<D>(wgb + C::OFF_K, kr, kv);
            store_row<D>(wgb + C::OFF_V, kr, vv);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      ok = wg_sync(&bar_cv, cph, lane, &abort_flag);
      if (!ok) break;
      // ---- S (both blocks) and G: G's columns (and, without EARLY, S's)
      // hold item j - 2's O until its epilogue has read it
      if (mma_lane) {
        tc_fence_after();
        if (j >= 2 && !mbar_wait(&bar_tfree[g], (jj - 1) & 1, kWaitNs, &abort_flag)) {
          if (!abort_flag) record_timeout(&abort_flag);
        } else {
          tc_fence_after();
          const uint32_t slot = tmem + g * kSlotCols;
          const uint32_t qaa = smem_addr(wgb + C::OFF_QA), qab = smem_addr(wgb + C::OFF_QB);
          const uint32_t kta = smem_addr(wgb + C::OFF_K);
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const uint32_t dst = slot + (static_cast<uint32_t>(b * 16) << 16);
            const uint32_t qa = b ? qab : qaa, ka = kta + b * A::BOFF * A::ROWB;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_f16_ss(dst, smem_desc(qa + 32 * ks, 16, A::SBO, A::SW), smem_desc(ka + 32 * ks, 16, A::SBO, A::SW),
                         idS, ks != 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_f16_ss(dst + kGBase, smem_desc(qa + 32 * ks, 16, A::SBO, A::SW),
                         smem_desc(ra + 32 * ks, 16, A::SBO, A::SW), idG, ks != 0);
          }
          mma_commit(&bar_s[g]);
        }
      }
    }
    if (!ok && !abort_flag) record_timeout(&abort_flag);
    if (tma_lane && abort_flag) {
      // loads still in flight land before the block exits
      for (int k = (nx > XS ? nx - XS : 0); k < nx; ++k) mbar_wait(&bar_xfull[k % XS], (k / XS) & 1, kWaitNs);
      for (int k = (nw > 2 ? nw - 2 : 0); k < nw; ++k) mbar_wait(&bar_wfull[k & 1], (k >> 1) & 1, kWaitNs);
    }
    // the S and G MMAs are complete before TMEM is released
    if (mma_lane) {
      mma_commit(&bar_drain[8]);
      mbar_wait(&bar_drain[8], 0, kWaitNs);
    }
  }
  __syncwarp();
  tc_fence_before();
  named_bar_sync(1, kThreads);
  return;
  }

  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
  {
    // ------------------------------------------------------------ compute warpgroups
    const int g = warp >> 2;
    const int wq = warp & 3;
    const int blk = lane >> 4;              // 0: block A (lanes 0-15), 1: block B (lanes 16-31)
    const int row = 16 * wq + (lane & 15);  // query row in the 8x8 block
    const int qy = row >> 3, qx = row & 7;
    const uint32_t slot = tmem + g * kSlotCols;
    const uint32_t ts = slot + (static_cast<uint32_t>(32 * wq) << 16);
    uint8_t* wgb = sWG + g * C::WG_BYTES;
    const uint32_t vta = smem_addr(wgb + C::OFF_V);
    const uint32_t wba = smem_addr(wgb + C::TILES);
    const float c = p.c;
    const int C_all = heads * D;
    const uint32_t idP = idesc_bf16_f32(128, D, false);       // projections: A = x (K-major), B = W (K-major)
    const uint32_t idKV = idesc_bf16_f32(128, 2 * D, false);  // k and v of a window tile in one MMA
    const uint32_t idO = idesc_bf16_f32(64, A::ON, true);
    int ph = 0;

    // Projections of item jn (the warpgroup's jjn-th): q_part issues Q (lane 0
    // of warp 0), otherwise K and V (warps 1 and 2); each commits to bar_pr.
    // Without `wait` the call returns false, issuing nothing, when x or the
    // weights have not landed yet (the caller issues them later).
    auto issue_proj = [&](int jn, int jjn, bool q_part, bool wait) {
      if (lane != 0 || (q_part ? wq != 0 : (wq != 1 && wq != 2))) return true;
      const int pin = jn / heads, sn = pin % XS;
      const uint8_t* xsn = sX + sn * C::XSTAGE;
      const uint32_t xqa = smem_addr(xsn), xkva = smem_addr(xsn + C::KA * C::XQ_ATOM);
      if (!wait && !(mbar_test(&bar_xfull[sn], (pin / XS) & 1) && mbar_test(&bar_wfull[g], jjn & 1))) return false;
      const bool got = mbar_wait(&bar_xfull[sn], (pin / XS) & 1, kWaitNs, &abort_flag) &&
                       mbar_wait(&bar_wfull[g], jjn & 1, kWaitNs, &abort_flag);
      if (got) {
        tc_fence_after();
        constexpr int KSTEPS = CIN / 16;
        if (wq == 0) {
#pragma unroll 1
          for (int ks = 0; ks < KSTEPS; ++ks)
            mma_f16_ss(slot + C::COL_Q, smem_desc(xqa + (ks >> 2) * C::XQ_ATOM + (ks & 3) * 32, 16, 1024, SW_128B),
                       smem_desc(wba + (ks >> 2) * C::W_ATOM + (ks & 3) * 32, 16, 1024, SW_128B), idP, ks != 0);
        } else {
          // [k | v] of the window tiles, N = 2d: warp 1 the first tiles, warp 2 the rest
          const int t0 = wq == 1 ? 0 : (C::KVT + 1) / 2, t1 = wq == 1 ? (C::KVT + 1) / 2 : C::KVT;
          const uint32_t wm = wba + C::OFF_WKV;
#pragma unroll 1
          for (int t = t0; t < t1; ++t)
#pragma unroll 1
            for (int ks = 0; ks < KSTEPS; ++ks)
              mma_f16_ss(slot + C::COL_K + t * 2 * D,
                         smem_desc(xkva + (ks >> 2) * C::XKV_ATOM + t * 128 * 128 + (ks & 3) * 32, 16, 1024, SW_128B),
                         smem_desc(wm + (ks >> 2) * C::WKV_ATOM + (ks & 3) * 32, 16, 1024, SW_128B), idKV, ks != 0);
        }
        mma_commit(&bar_pr[g]);
      } else if (!abort_flag) {
        record_timeout(&abort_flag);
      }
      return true;
    };

    bool ok = true;
    int jj = 0;
    bool kv_due = C::EARLY, q_due = C::EARLY;  // projections of the next item still to issue
    for (int j = g; j < my_items && ok; j += 2, ++jj) {
      const int pi = j / heads, head = j % heads;
      const int pair = blockIdx.x + pi * gridDim.x;
      const int bx = pair % p.nbx, py = (pair / p.nbx) % p.npy, n = pair / (p.nbx * p.npy);
      // ---- this item's projections, unless issued during the previous item
      if (!C::EARLY || kv_due) issue_proj(j, jj, false, true);
      if (!C::EARLY || q_due) issue_proj(j, jj, true, true);
      kv_due = q_due = true;
      ok = warp_ok(mbar_wait(&bar_s[g], jj & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();

      const int by = 2 * py + blk;
      const int y0 = by * kBlock - p.halo, x0 = bx * kBlock - p.halo;
      // ---- pass 1: per window row the maximum of the raw S values
      float rm[WIN], rmo[WIN];
#pragma unroll
      for (int r = 0; r < WIN; ++r) rm[r] = rmo[r] = -INFINITY;
      row_max_pipelined<WIN, A>(ts, rm, rmo);
      // ---- relative logits of this query, in log2 units
      float rh[WIN], rw[WIN], rwz[WIN];
      {
        float gh[WIN + 1];
        tmem_ld_exact<WIN + 1>(ts + kGBase + (WIN - 2 - 2 * wq), gh);
        float a[WIN + 7];
        tmem_ld_exact<WIN + 7>(ts + kGBase + kRelW + WIN - 8, a);
        tmem_wait_ld();
        const bool odd = ((lane >> 3) & 1) != 0;
#pragma unroll
        for (int kr = 0; kr < WIN; ++kr) {
          const int Y = y0 + kr;
          rh[kr] = (Y >= 0 && Y < p.H) ? (odd ? gh[kr] : gh[kr + 1]) * c : -INFINITY;
        }
        const int sh = 7 - qx;
#pragma unroll
        for (int i = 0; i < WIN + 3; ++i) a[i] = (sh & 4) ? a[i + 4] : a[i];
#pragma unroll
        for (int i = 0; i < WIN + 1; ++i) a[i] = (sh & 2) ? a[i + 2] : a[i];
#pragma unroll
        for (int i = 0; i < WIN; ++i) a[i] = (sh & 1) ? a[i + 1] : a[i];
#pragma unroll
        for (int kc = 0; kc < WIN; ++kc) {
          const int X = x0 + kc;
          rwz[kc] = (X >= 0 && X < p.W) ? a[kc] : -INFINITY;
          rw[kc] = rwz[kc] * c;
        }
      }
      // bound of the row maximum with the exact fallback (halo_tc4.cuh)
      float mw = -INFINITY, mwo = INFINITY;
#pragma unroll
      for (int kc = 0; kc < WIN; ++kc) {
        mw = fmaxf(mw, rw[kc]);
        if (own_pair<WIN>(kc & ~1)) mwo = fminf(mwo, rw[kc]);
      }
      float m = -INFINITY, mlo = -INFINITY;
#pragma unroll
      for (int r = 0; r < WIN; ++r) {
        if (r >= A::HALO && r < A::HALO + kBlock) mlo = fmaxf(mlo, fmaf(rmo[r], c, rh[r]));
        m = fmaxf(m, fmaf(fmaxf(rm[r], rmo[r]), c, rh[r]));
      }
      m += mw;
      mlo += mwo;
      if (__any_sync(0xffffffffu, m - mlo > 100.0f)) m = exact_row_max<WIN, A>(ts, rh, rw, c);
      // ---- pass 2: p = 2^(c*(S + rel_w) + c*rel_h - m), bf16 P over the S columns
      float brow[WIN];
#pragma unroll
      for (int r = 0; r < WIN; ++r) brow[r] = rh[r] - m;
      exp_pipelined<WIN, A>(ts, rwz, brow, c);
      tc2::tmem_wait_st();
      tc_fence_before();
      ok = wg_sync(&bar_wg[g], ph, lane, &abort_flag);
      if (!ok) break;
      // ---- A.V: warp wq issues block (wq & 1), key half (wq >> 1)
      if (lane == 0) {
        tc_fence_after();
        const int ab = wq & 1, hf = wq >> 1;
        const int kb = hf ? A::KHALF : 0, ke = hf ? A::KSTEPS : A::KHALF;
        const uint32_t lanes = static_cast<uint32_t>(16 * ab) << 16;
        const uint32_t va = vta + ab * A::BOFF * A::ROWB;
        const uint32_t lbo = smem_addr(sOnes) - va;
#pragma unroll 1
        for (int kk = kb; kk < ke; ++kk)
          mma_f16_ts(slot + lanes + C::O_COL + hf * A::ON, slot + lanes + 8 * kk,
                     smem_desc(va + kk * 16 * A::ROWB, lbo, A::SBO, A::SW), idO, kk != kb);
        mma_commit(&bar_o[g]);
      }
      // the next item's K and V projections into the dead S columns (if its
      // x and weights have landed; else at the start of that item)
      if constexpr (C::EARLY) {
        if (j + 2 < my_items && issue_proj(j + 2, jj + 1, false, false)) kv_due = false;
      }
      ok = warp_ok(mbar_wait(&bar_o[g], jj & 1, kWaitNs, &abort_flag));
      if (!ok) break;
      tc_fence_after();
      // and its Q projection into P's first columns, which the A.V has read
      if constexpr (C::EARLY) {
        if (j + 2 < my_items && issue_proj(j + 2, jj + 1, true, false)) q_due = false;
      }
      // ---- epilogue: (O_0 + O_1) / (l_0 + l_1), bf16, NHWC
      {
        float o[D], la, lb;
        tmem_ld_x1(ts + C::O_COL + D, &la);
        tmem_ld_x1(ts + C::O_COL + A::ON + D, &lb);
        constexpr int kSeg = (D % 32 == 0) ? 32 : 16;
#pragma unroll
        for (int e = 0; e < D; e += kSeg) {
          float ta[kSeg], tb[kSeg];
          if constexpr (kSeg == 32) {
            tmem_ld_x32(ts + C::O_COL + e, ta);
            tmem_ld_x32(ts + C::O_COL + A::ON + e, tb);
          } else {
            tmem_ld_x8(ts + C::O_COL + e, ta);
            tmem_ld_x8(ts + C::O_COL + e + 8, ta + 8);
            tmem_ld_x8(ts + C::O_COL + A::ON + e, tb);
            tmem_ld_x8(ts + C::O_COL + A::ON + e + 8, tb + 8);
          }
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < kSeg; ++i) o[e + i] = ta[i] + tb[i];
        }
        // O is read: the next G (and, without EARLY, S) may take its columns
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_tfree[g]);
        const float inv = 1.0f / (la + lb);
        uint32_t pk[D / 2];
#pragma unroll
        for (int t = 0; t < D / 2; ++t) pk[t] = pack_bf16x2(o[2 * t] * inv, o[2 * t + 1] * inv);
        const int y = by * kBlock + qy, x = bx * kBlock + qx;
        __nv_bfloat16* dst = p.out + ((static_cast<size_t>(n) * p.H + y) * p.W + x) * C_all + head * D;
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
          reinterpret_cast<uint4*>(dst)[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      }
      // without EARLY the next item's projections overwrite this item's
      // columns: every warp of the warpgroup is done with them first
      if constexpr (!C::EARLY) {
        tc_fence_before();
        ok = wg_sync(&bar_wg[g], ph, lane, &abort_flag);
      }
    }
    if (!ok && !abort_flag) record_timeout(&abort_flag);
    // MMAs this warp issued are complete before TMEM is released
    if (lane == 0) {
      mma_commit(&bar_drain[warp]);
      mbar_wait(&bar_drain[warp], 0, kWaitNs);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  named_bar_sync(1, kThreads);
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fused
}  // namespace halo
