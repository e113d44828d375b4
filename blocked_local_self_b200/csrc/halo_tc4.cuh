// halo_tc4.cuh -- stride-1 bf16 kernel for blocked local self-attention with
// haloing on sm_100a, 8x8 query blocks, dim_head 16, 32 or 64, maps with an
// even number of block rows.
//
// Operation (HaloNet, "Scaling Local Self-Attention for Parameter Efficient
// Visual Backbones", sections 2.1-2.2 and appendix A; index conventions of the
// blog page's RelPosEmb / HaloAttention modules):
//   z[q, key] = s * q . (k[key] + rel_h[kr - qy + w - 1] + rel_w[kc - qx + w - 1])
//   out[q]    = sum over in-image window keys of softmax(z) * v[key]
//
// Work item = two vertically adjacent 8x8 blocks of one head.  Their windows
// (w x w each) overlap in w - 8 rows, so one TMA box of (w + 8) x w pixels
// holds both: in the box's row-major order block A's window is keys
// [0, w*w) and block B's is keys [8w, 8w + w*w), both contiguous: the item
// loads (w + 8) w key and value pixels instead of the 2 w^2 of two separate
// windows, and with d = 64 two pipeline stages fit in shared memory (96 KB
// each).
//   * TMA (warp 8): Q_A, Q_B [64 x d] and the union K tile, and one item
//     later the union V tile (separate barriers, so Q/K stages free early).
//   * S MMAs (block A on warp 9, block B on warp 11): per block M=64, N=200
//     (its window) into its TMEM lane half (block A lanes 0-15 of each
//     quadrant, block B 16-31).
//   * G MMAs (warp 10, own barrier): per block G = Q R^T (N=56, R = [rel_h; 0; rel_w; 0]
//     written once) into slot columns [200, 256); each thread takes the
//     w + w relative logits of its query by a TMEM column shift and selects.
//   * softmax (one thread per TMEM lane = one query row): pass 1 takes the
//     raw S maximum of every window row (before G is needed), then an upper
//     bound of the row maximum, max over rows of c*S_max + c*rel_h plus the
//     maximum of c*rel_w (a few units above the exact one with HaloNet's
//     tables; when a lower bound from the block's own keys says it may be
//     more than 100 log2 units above, the exact maximum is taken instead);
//     pass 2 the exponentials (MUFU and the FMA-pipe cubic) and bf16 P
//     written back over the S columns.  Both passes walk the row in pieces
//     of 32 keys with the next piece's TMEM load in flight.
//   * A.V: four independent MMA chains, one per softmax warp: warp q takes
//     block q & 1 and key half q >> 1, O_h = P_blk[:, keys of half h]
//     V_blk[keys of half h] with M=64, N=d, A (P) read from the block's TMEM
//     lane half and the accumulator in the same lane half (block B's window
//     8w rows below block A's in the V tile).  The B operand's second
//     swizzle atom is a ones tile: 8 more accumulator columns hold the row
//     sum of the bf16 P.  The two halves share one maximum, so O = O_0 + O_1
//     and l = l_0 + l_1.
//   * epilogue: (O_0 + O_1) / (l_0 + l_1), bf16, NHWC.
// Two softmax warpgroups take alternate items; every wait is bounded.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <utility>

#include "halo_tc.cuh"
#include "halo_tc2.cuh"
#include "sm100.cuh"

namespace halo {
namespace tc4 {

using namespace sm100;
using tc::exp2_mufu;
using tc::pack_bf16x2;
using tc::record_timeout;
using tc::swz;
using tc2::exp2_poly2;
using tc2::max3f;
using tc2::mma_f16_ts;
using tc2::pack_p;
using tc2::poly_pair_mask;
using tc2::tmem_ld_cols;
using tc2::tmem_ld_x32;
using tc2::tmem_ld_x8;
using tc2::tmem_st_x8;
using tc2::tmem_wait_st;

constexpr int kBlock = 8;
constexpr int kThreads = 384;   // warpgroups 0-1 softmax, warp 8 TMA, warps 9/11 S MMAs, warp 10 G MMAs
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kGMmaWarp = 10;
constexpr int kSBMmaWarp = 11;
constexpr int kSoftmaxRegs = tc::kSoftmaxRegs;
constexpr int kProducerRegs = tc::kProducerRegs;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;  // warpgroup g owns columns [256g, 256g + 256)
constexpr uint32_t kGBase = 200;     // G at slot columns [200, 256): rel_h logits, then rel_w at +28
constexpr int kRelW = 28;
constexpr int kRRows = 56;
constexpr uint64_t kWaitNs = tc::kWaitNs;

struct Params {
  const __nv_bfloat16* rel_h;
  const __nv_bfloat16* rel_w;
  __nv_bfloat16* out;
  int N, H, W, heads, halo;
  int nbx, npy;    // blocks along x, block pairs along y
  int num_items;   // N * npy * nbx * heads
  int stages;
  float c;         // log2(e) / sqrt(d)
  int kmask;       // SASA mask size (MASK instantiations only): keys within kmask/2 of the query
};

template <int D, int WIN>
struct Cfg {
  static constexpr int ROWB = D * 2;
  static constexpr int KS = WIN * WIN;                    // window keys of one block
  static constexpr int NS = (KS + 7) / 8 * 8;             // S MMA N
  static constexpr int KSTEPS = (KS + 15) / 16;           // A.V K-steps
  static constexpr int KP = KSTEPS * 16;                  // keys incl. zero padding
  static constexpr int BOFF = kBlock * WIN;               // block B's first key in the union tile
  static constexpr int UROWS = (WIN + kBlock) * WIN;      // union tile rows the TMA writes
  static constexpr int KROWS = BOFF + (KP > NS ? KP : NS);  // rows read by the MMAs
  static constexpr int Q_TILE = 64 * ROWB;
  static constexpr int K_TILE = (KROWS * ROWB + 1023) / 1024 * 1024;
  static constexpr int STAGE_BYTES = 2 * Q_TILE + 2 * K_TILE;
  static constexpr int R_TILE = (kRRows * ROWB + 1023) / 1024 * 1024;
  static constexpr int TX_QK = (2 * 64 + UROWS) * ROWB;  // Q_A, Q_B and the K union tile
  static constexpr int TX_V = UROWS * ROWB;               // the V union tile
  static constexpr int PCOLS = KP / 2;                    // packed bf16 P columns
  static constexpr int O_BASE = (PCOLS + 7) / 8 * 8;      // first O column
  static constexpr int KHALF = (KSTEPS + 1) / 2;          // A.V K-steps of key half 0
  // A.V N: the block's V (d columns) and 8 columns of a ones tile, whose
  // product with P is the row sum of the bf16 P the MMA consumed
  static constexpr int ON = D + 8;
  static constexpr int O_N = 2 * ON;                      // O_0 | O_1, each in both lane halves
  // Where the columns allow (d = 16), O goes to the relative-logit columns,
  // which the softmax has consumed before the A.V: the S MMA of the slot's
  // next item then waits only for this item's A.V to finish reading P, not
  // for the epilogue to read O (only the next G waits for that).
  static constexpr bool O_IN_G = (int)kGBase + O_N <= (int)kSlotCols;
  static constexpr int O_COL = O_IN_G ? (int)kGBase : O_BASE;
  static constexpr int ONES_BYTES = (KP * ROWB + 1023) / 1024 * 1024;  // ones rows, V's row pitch
  static constexpr SmemSwizzle SW = (ROWB == 32) ? SW_32B : (ROWB == 64 ? SW_64B : SW_128B);
  static constexpr uint32_t SBO = 8 * ROWB;
  static constexpr int HALO = (WIN - kBlock) / 2;
  // window-column pairs whose exponentials take the FMA-pipe cubic: with
  // d = 64 the larger MMAs leave the exponential unit less busy and every
  // exponential goes to MUFU (deep-stage workload: 73.5 us, one pair 74.4,
  // two 76.0); at d = 16 two pairs (111.3 us against 114.9 with one)
  static constexpr int NPOLY = (D >= 64) ? 0 : HALO_TC2_POLY_PAIRS;
  static_assert(D == 16 || D == 32 || D == 64, "dim_head 16, 32 or 64");
  static_assert(WIN % 2 == 0 && WIN >= 8 && WIN <= 14, "window 8..14");
  static_assert(NS <= (int)kGBase, "S columns below the relative logits");
  static_assert(2 * WIN - 1 <= kRelW, "relative table rows");
  static_assert(O_BASE + O_N <= (int)kSlotCols, "O accumulator in the slot");
  static_assert((BOFF * ROWB) % 1024 == 0 || ROWB < 128, "block B's window on a swizzle atom");
  static_assert(Q_TILE % 1024 == 0, "tiles on 1 KB boundaries");
};

template <int D, int WIN>
__host__ __device__ constexpr int smem_bytes(int stages) {
  using C = Cfg<D, WIN>;
  return 1024 + C::R_TILE + stages * C::STAGE_BYTES + C::ONES_BYTES;
}

// Load exactly N (< 32) consecutive TMEM columns (32x32b shape, thread t <->
// lane t of the warp's quadrant) without reading past the last one.
__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, float* r) {
  uint32_t v[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] = __uint_as_float(v[i]);
}
__device__ __forceinline__ void tmem_ld_x2(uint32_t taddr, float* r) {
  uint32_t v[2];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(taddr));
  r[0] = __uint_as_float(v[0]);
  r[1] = __uint_as_float(v[1]);
}
__device__ __forceinline__ void tmem_ld_x1(uint32_t taddr, float* r) {
  uint32_t v;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v) : "r"(taddr));
  r[0] = __uint_as_float(v);
}
template <int N>
__device__ __forceinline__ void tmem_ld_exact(uint32_t taddr, float* r) {
  static_assert(N > 0 && N < 32, "at most 31 columns");
  constexpr int a = N & 16, b = N & 8, c4 = N & 4, c2 = N & 2, c1 = N & 1;
  if constexpr (a) {
    float t[16];
    tmem_ld_x8(taddr, t);
    tmem_ld_x8(taddr + 8, t + 8);
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = t[i];
  }
  if constexpr (b) tmem_ld_x8(taddr + a, r + a);
  if constexpr (c4) tmem_ld_x4(taddr + a + b, r + a + b);
  if constexpr (c2) tmem_ld_x2(taddr + a + b + c4, r + a + b + c4);
  if constexpr (c1) tmem_ld_x1(taddr + a + b + c4 + c2, r + a + b + c4 + c2);
}

struct ItemCoord {
  int n, py, bx, head;
};
__device__ __forceinline__ ItemCoord item_coord(int item, int heads, int nbx, int npy) {
  ItemCoord c;
  c.head = item % heads;
  const int blk = item / heads;
  c.bx = blk % nbx;
  c.py = (blk / nbx) % npy;
  c.n = blk / (nbx * npy);
  return c;
}

// Software-pipelined passes in pieces of 32 keys: the TMEM load of piece
// i + 1 is issued before piece i is processed, so its latency overlaps the
// arithmetic (a thread holds two 32-key buffers).
template <class C>
__host__ __device__ constexpr int pp_end(int i) { return (32 * (i + 1) < C::KS) ? 32 * (i + 1) : C::KS; }
template <class C>
__host__ __device__ constexpr int pp_pend(int i) { return (32 * (i + 1) < C::KP) ? 32 * (i + 1) : C::KP; }
template <class C>
__host__ __device__ constexpr int pp_count() { return (C::KP + 31) / 32; }

// Window-column pairs (kc, kc + 1), kc even, that lie inside the block's own
// eight columns [h, h + 8): those keys are never outside the image.
template <int WIN>
__host__ __device__ constexpr bool own_pair(int kc) {
  return kc >= (WIN - kBlock) / 2 && kc + 1 < (WIN - kBlock) / 2 + kBlock;
}

// Pass 1 keeps two maxima per window row: rmo over the own-column pairs
// (in-image keys only) and rm over the other pairs; the caller merges them.
// rmo also yields a lower bound of the exact row maximum (see the caller).
template <int WIN, class C, int I>
__device__ __forceinline__ void max_pipe(uint32_t ts, float (&rm)[WIN], float (&rmo)[WIN], float (&cur)[32],
                                         float (&nxt)[32]) {
  constexpr int J0 = 32 * I, J1 = pp_end<C>(I);
  if constexpr (I + 1 < pp_count<C>()) {
    constexpr int K0 = 32 * (I + 1), K1 = pp_end<C>(I + 1);
    tmem_ld_cols<(K1 - K0 + 7) / 8 * 8>(ts + K0, nxt);
  }
#pragma unroll
  for (int i = 0; i < (J1 - J0) / 2; ++i) {
    const int r = (J0 + 2 * i) / WIN;
    if (own_pair<WIN>((J0 + 2 * i) % WIN)) rmo[r] = max3f(rmo[r], cur[2 * i], cur[2 * i + 1]);
    else rm[r] = max3f(rm[r], cur[2 * i], cur[2 * i + 1]);
  }
  if constexpr (I + 1 < pp_count<C>()) {
    tmem_wait_ld();
    max_pipe<WIN, C, I + 1>(ts, rm, rmo, nxt, cur);
  }
}
template <int WIN, class C>
__device__ __forceinline__ void row_max_pipelined(uint32_t ts, float (&rm)[WIN], float (&rmo)[WIN]) {
  float za[32], zb[32];
  tmem_ld_cols<(pp_end<C>(0) + 7) / 8 * 8>(ts, za);
  tmem_wait_ld();
  max_pipe<WIN, C, 0>(ts, rm, rmo, za, zb);
}

// Exact row maximum of c * S + rh[row] + rw[col] over the window (masked rows
// and columns carry -inf in rh / rw).  Taken only when the cheap bound of the
// caller may lie too far above the exact maximum; not pipelined.  Whole-warp
// (tcgen05.ld): the caller takes it for every thread of the warp.
template <int WIN, class C>
__device__ __forceinline__ float exact_row_max(uint32_t ts, const float (&rh)[WIN], const float (&rw)[WIN], float c) {
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < pp_count<C>(); ++i) {
    const int j0 = 32 * i, j1 = (32 * (i + 1) < C::KS) ? 32 * (i + 1) : C::KS;
    float z[32];
    tmem_ld_x8(ts + j0, z);
    tmem_ld_x8(ts + j0 + 8, z + 8);
    tmem_ld_x8(ts + j0 + 16, z + 16);
    tmem_ld_x8(ts + j0 + 24, z + 24);
    tmem_wait_ld();
#pragma unroll
    for (int t = 0; t < 32; ++t)
      if (j0 + t < j1) m = fmaxf(m, fmaf(z[t], c, rh[(j0 + t) / WIN] + rw[(j0 + t) % WIN]));
  }
  return m;
}

template <int WIN, class C, int I>
__device__ __forceinline__ void exp_pipe(uint32_t ts, const float (&rw)[WIN], const float (&brow)[WIN], float c,
                                         float (&cur)[32], float (&nxt)[32]) {
  constexpr int J0 = 32 * I, J1 = pp_end<C>(I), JP = pp_pend<C>(I);
  constexpr int NW = (JP - J0) / 2, NP = (J1 > J0) ? (J1 - J0) / 2 : 0;
  constexpr unsigned kPoly = poly_pair_mask<WIN>(C::NPOLY);
  if constexpr (I + 1 < pp_count<C>()) {
    constexpr int K0 = 32 * (I + 1), K1 = pp_end<C>(I + 1);
    if constexpr (K1 > K0) tmem_ld_cols<(K1 - K0 + 7) / 8 * 8>(ts + K0, nxt);
  }
  uint32_t pk[NW];
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int j = J0 + 2 * i, kc = j % WIN;
    const float2 zz = __fadd2_rn(make_float2(cur[2 * i], cur[2 * i + 1]), make_float2(rw[kc], rw[kc + 1]));
    const float bias = brow[j / WIN];
    const float2 x = __ffma2_rn(zz, make_float2(c, c), make_float2(bias, bias));
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
  for (int i = 0; i < NW; i += 8) tmem_st_x8(ts + J0 / 2 + i, pk + i);
  if constexpr (I + 1 < pp_count<C>()) {
    tmem_wait_ld();
    exp_pipe<WIN, C, I + 1>(ts, rw, brow, c, nxt, cur);
  }
}
template <int WIN, class C>
__device__ __forceinline__ void exp_pipelined(uint32_t ts, const float (&rw)[WIN], const float (&brow)[WIN], float c) {
  float za[32], zb[32];
  tmem_ld_cols<(pp_end<C>(0) + 7) / 8 * 8>(ts, za);
  tmem_wait_ld();
  exp_pipe<WIN, C, 0>(ts, rw, brow, c, za, zb);
}

// MASK: the SASA-masked variant (section 2.2: halo floor(k/2) and a mask
// keeping the k x k keys centred on each query).  That mask is a band of
// window rows times a band of window columns per query, so it is applied
// through the query's rel_h / rel_w logits (-inf outside the bands), and the
// row maximum is always the exact one (the own-column lower bound of the
// unmasked kernel does not hold once own columns can be masked).
template <int D, int WIN, bool MASK>
__global__ void __launch_bounds__(kThreads, 1)
    halo_fwd_tc4(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using C = Cfg<D, WIN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sR = smem;
  uint8_t* sStage = smem + C::R_TILE;
  uint8_t* sOnes = sStage + p.stages * C::STAGE_BYTES;  // after every stage: positive LBO from any V tile
  // stage layout: [Q_A][Q_B][K union][V union]
  constexpr int OFF_QA = 0, OFF_QB = C::Q_TILE, OFF_K = 2 * C::Q_TILE, OFF_V = OFF_K + C::K_TILE;

  // Q/K and V of a stage have their own barriers: Q and K are released when
  // the S and G MMAs finish, long before the A.V releases V, so the next
  // items' Q/K loads are in flight during the softmax.
  __shared__ __align__(8) uint64_t bar_fqk[4];
  // V of item k lands on bar_fv[k % (2S)]: a barrier per stage and per
  // warpgroup, so that the A.V issuers of item k never wait on a barrier whose
  // previous phase (the other warpgroup's item k - S, at an odd stage count)
  // is still open, where a parity wait would pass one phase early.
  __shared__ __align__(8) uint64_t bar_fv[8];
  __shared__ __align__(8) uint64_t bar_eqk[4];  // count 3: S_A, S_B, G
  __shared__ __align__(8) uint64_t bar_ev[4];   // count 4: the A.V chains
  __shared__ __align__(8) uint64_t bar_sfull[2];   // count 2: the two blocks' S MMAs
  __shared__ __align__(8) uint64_t bar_gfull[2];
  __shared__ __align__(8) uint64_t bar_ofull[2];
  __shared__ __align__(8) uint64_t bar_tfree[2];   // count 4: the warpgroup read its slot's O
  __shared__ __align__(8) uint64_t bar_pready[2];  // count 4, waited by every warp of the warpgroup
  __shared__ __align__(8) uint64_t bar_done[3];
  __shared__ __align__(8) uint64_t bar_pvdone[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int S = p.stages;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&bar_fqk[i], 1);
      mbar_init(&bar_fv[i], 1);
      mbar_init(&bar_fv[S + i], 1);
      mbar_init(&bar_eqk[i], 3);
      mbar_init(&bar_ev[i], 4);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bar_sfull[g], 2);
      mbar_init(&bar_ofull[g], 4);
      mbar_init(&bar_tfree[g], 4);
      mbar_init(&bar_pready[g], 4);
      mbar_init(&bar_done[g], 1);
      mbar_init(&bar_gfull[g], 1);
      mbar_init(&bar_pvdone[g], 4);
    }
    mbar_init(&bar_done[2], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  // ones tile (bf16 1.0 in every element, so the swizzle does not matter)
  for (int idx = tid; idx < C::ONES_BYTES / 16; idx += kThreads)
    reinterpret_cast<uint4*>(sOnes)[idx] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  // R tile (once) and the union tiles' rows the TMA never writes (zero)
  for (int idx = tid; idx < kRRows * (D / 8); idx += kThreads) {
    const int r = idx / (D / 8), u = idx % (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < 2 * WIN - 1) val = *reinterpret_cast<const uint4*>(p.rel_h + r * D + u * 8);
    else if (r >= kRelW && r < kRelW + 2 * WIN - 1)
      val = *reinterpret_cast<const uint4*>(p.rel_w + (r - kRelW) * D + u * 8);
    *reinterpret_cast<uint4*>(sR + swz<C::ROWB>(r, u)) = val;
  }
  for (int s = 0; s < S; ++s) {
    uint8_t* st = sStage + s * C::STAGE_BYTES;
    for (int idx = tid; idx < (C::KROWS - C::UROWS) * C::ROWB / 16; idx += kThreads) {
      reinterpret_cast<uint4*>(st + OFF_K + C::UROWS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(st + OFF_V + C::UROWS * C::ROWB)[idx] = make_uint4(0, 0, 0, 0);
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
    // issue order QK(0), QK(1), V(0), QK(2), V(1), ...: the Q/K of an item
    // go out one item ahead of the V it does not need until its A.V
    if (lane == 0) {
      int nqk = 0, nv = 0;
      for (int t = 0; t <= my_items; ++t) {
        if (t < my_items) {
          const int s = t % S;
          if (t >= S && !mbar_wait(&bar_eqk[s], ((t / S) - 1) & 1, kWaitNs, &abort_flag)) {
            if (!abort_flag) record_timeout(&abort_flag);
            break;
          }
          const ItemCoord ic = item_coord(blockIdx.x + t * gridDim.x, p.heads, p.nbx, p.npy);
          uint8_t* st = sStage + s * C::STAGE_BYTES;
          const int x0 = ic.bx * kBlock, y0 = ic.py * 2 * kBlock;
          mbar_arrive_expect_tx(&bar_fqk[s], C::TX_QK);
          tma_load_4d(st + OFF_QA, &tmap_q, &bar_fqk[s], ic.head * D, x0, y0, ic.n);
          tma_load_4d(st + OFF_QB, &tmap_q, &bar_fqk[s], ic.head * D, x0, y0 + kBlock, ic.n);
          tma_load_4d(st + OFF_K, &tmap_k, &bar_fqk[s], ic.head * D, x0 - p.halo, y0 - p.halo, ic.n);
          nqk = t + 1;
        }
        if (t >= 1) {
          const int k = t - 1, s = k % S;
          if (k >= S && !mbar_wait(&bar_ev[s], ((k / S) - 1) & 1, kWaitNs, &abort_flag)) {
            if (!abort_flag) record_timeout(&abort_flag);
            break;
          }
          const ItemCoord ic = item_coord(blockIdx.x + k * gridDim.x, p.heads, p.nbx, p.npy);
          uint8_t* st = sStage + s * C::STAGE_BYTES;
          const int x0 = ic.bx * kBlock, y0 = ic.py * 2 * kBlock;
          uint64_t* fv = &bar_fv[k % (2 * S)];
          mbar_arrive_expect_tx(fv, C::TX_V);
          tma_load_4d(st + OFF_V, &tmap_v, fv, ic.head * D, x0 - p.halo, y0 - p.halo, ic.n);
          nv = k + 1;
        }
      }
      if (abort_flag) {
        // loads still in flight land before the block exits
        for (int k = (nqk > S ? nqk - S : 0); k < nqk; ++k) mbar_wait(&bar_fqk[k % S], (k / S) & 1, kWaitNs);
        for (int k = (nv > S ? nv - S : 0); k < nv; ++k) mbar_wait(&bar_fv[k % (2 * S)], (k / (2 * S)) & 1, kWaitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ S (warps 9, 11) and G (warp 10) MMAs
    const bool is_g = (warp == kGMmaWarp);
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(64, C::NS, false);
      const uint32_t idG = idesc_bf16_f32(64, kRRows, false);
      const uint32_t ra = smem_addr(sR);
      for (int k = 0; k < my_items; ++k) {
        const int s = k % S, g = k & 1;
        // the slot is free for S once the A.V of item k - 2 has read its P
        // (O elsewhere) or once its epilogue has read O; for G, always the latter
        uint64_t* slot_free = (C::O_IN_G && !is_g) ? &bar_ofull[g] : &bar_tfree[g];
        if (!mbar_wait(&bar_fqk[s], (k / S) & 1, kWaitNs, &abort_flag) ||
            (k >= 2 && !mbar_wait(slot_free, ((k >> 1) - 1) & 1, kWaitNs, &abort_flag))) {
          if (!abort_flag) record_timeout(&abort_flag);
          break;
        }
        tc_fence_after();
        const uint8_t* st = sStage + s * C::STAGE_BYTES;
        const uint32_t slot = tmem + g * kSlotCols;
#pragma unroll 1
        for (int blk = (warp == kSBMmaWarp); blk < (warp == kMmaWarp ? 1 : 2); ++blk) {
          const uint32_t qa = smem_addr(st + (blk ? OFF_QB : OFF_QA));
          const uint32_t dst = slot + (static_cast<uint32_t>(blk * 16) << 16);
          if (is_g) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_f16_ss(dst + kGBase, smem_desc(qa + 32 * ks, 16, C::SBO, C::SW),
                         smem_desc(ra + 32 * ks, 16, C::SBO, C::SW), idG, ks != 0);
          } else {
            const uint32_t ka = smem_addr(st + OFF_K + blk * C::BOFF * C::ROWB);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_f16_ss(dst, smem_desc(qa + 32 * ks, 16, C::SBO, C::SW), smem_desc(ka + 32 * ks, 16, C::SBO, C::SW),
                         idS, ks != 0);
          }
        }
        mma_commit(is_g ? &bar_gfull[g] : &bar_sfull[g]);
        mma_commit(&bar_eqk[s]);
      }
      const int w = warp - kMmaWarp;
      mma_commit(&bar_done[w]);
      mbar_wait(&bar_done[w], 0, kWaitNs);
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
    const int g = warp >> 2;             // warpgroup = TMEM slot
    const int wq = warp & 3;             // lane quadrant
    const int blk = lane >> 4;           // 0: block A (lanes 0-15), 1: block B (lanes 16-31)
    const int row = 16 * wq + (lane & 15);  // query row in the 8x8 block
    const int qy = row >> 3, qx = row & 7;
    const uint32_t slot = tmem + g * kSlotCols;
    const uint32_t ts = slot + (static_cast<uint32_t>(32 * wq) << 16);
    const float c = p.c;
    const int C_all = p.heads * D;
    const uint32_t idO = idesc_bf16_f32(64, C::ON, true);

    int j = 0;
    for (int k = g; k < my_items; k += 2, ++j) {
      if (!mbar_wait(&bar_sfull[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();
      const ItemCoord ic = item_coord(blockIdx.x + k * gridDim.x, p.heads, p.nbx, p.npy);
      const int by = 2 * ic.py + blk;
      const int y0 = by * kBlock - p.halo, x0 = ic.bx * kBlock - p.halo;

      // ---- pass 1: per window row the maximum of the raw S values
      float rm[WIN], rmo[WIN];
#pragma unroll
      for (int r = 0; r < WIN; ++r) rm[r] = rmo[r] = -INFINITY;
      row_max_pipelined<WIN, C>(ts, rm, rmo);
      if (!mbar_wait(&bar_gfull[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();
      // ---- relative logits of this query, in log2 units:
      //   rh[kr] = c * q.rel_h[kr - qy + w - 1], rw[kc] = c * q.rel_w[kc - qx + w - 1]
      float rh[WIN], rw[WIN], rwz[WIN];  // rwz: rel_w logits unscaled (S units)
      {
        // rel_h: the warp's two query rows differ by one column; the shift by
        // the warp's first row goes into the load address
        float gh[WIN + 1];
        tmem_ld_exact<WIN + 1>(ts + kGBase + (WIN - 2 - 2 * wq), gh);
        // rel_w: a[i] = G[rel_w + w - 8 + i], shifted by sh = 7 - qx (3 bits)
        float a[WIN + 7];
        tmem_ld_exact<WIN + 7>(ts + kGBase + kRelW + WIN - 8, a);
        tmem_wait_ld();
        const bool odd = ((lane >> 3) & 1) != 0;
#pragma unroll
        for (int kr = 0; kr < WIN; ++kr) {
          const int Y = y0 + kr;
          const float v = odd ? gh[kr] : gh[kr + 1];
          bool keep = Y >= 0 && Y < p.H;
          if constexpr (MASK) keep = keep && kr - qy - p.halo <= (p.kmask >> 1) && qy + p.halo - kr <= (p.kmask >> 1);
          rh[kr] = keep ? v * c : -INFINITY;
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
          bool keep = X >= 0 && X < p.W;
          if constexpr (MASK) keep = keep && kc - qx - p.halo <= (p.kmask >> 1) && qx + p.halo - kc <= (p.kmask >> 1);
          rwz[kc] = keep ? a[kc] : -INFINITY;
          rw[kc] = rwz[kc] * c;
        }
      }

      // Upper bound of the row maximum: max over rows of (c * raw row max +
      // rel_h) plus the largest rel_w.  It lies above the exact maximum by at
      // most the spread of the rel_w logits, plus, at the image border, the
      // gap between the valid keys' logits and the zero-filled masked keys'
      // S = 0.  A lower bound comes from the own-column pairs of the block's
      // own rows (in-image keys only): max over those rows of (c * own row
      // max + rel_h) plus the smallest rel_w of those columns.  While the two
      // are within 100 log2 units the largest p is at least 2^-100 (no
      // underflow of the row sum); beyond that (huge relative tables, or
      // strongly negative logits at a border) the exact maximum is taken.
      float mw = -INFINITY, mwo = INFINITY;
#pragma unroll
      for (int kc = 0; kc < WIN; ++kc) {
        mw = fmaxf(mw, rw[kc]);
        if (own_pair<WIN>(kc & ~1)) mwo = fminf(mwo, rw[kc]);
      }
      float m = -INFINITY, mlo = -INFINITY;
#pragma unroll
      for (int r = 0; r < WIN; ++r) {
        if (r >= C::HALO && r < C::HALO + kBlock) mlo = fmaxf(mlo, fmaf(rmo[r], c, rh[r]));
        m = fmaxf(m, fmaf(fmaxf(rm[r], rmo[r]), c, rh[r]));
      }
      m += mw;  // finite: the query's own block is in the image
      mlo += mwo;
      if (MASK || __any_sync(0xffffffffu, m - mlo > 100.0f)) m = exact_row_max<WIN, C>(ts, rh, rw, c);
      // ---- pass 2: p = 2^(c*(S + rel_w) + c*rel_h - m)
      float brow[WIN];
#pragma unroll
      for (int r = 0; r < WIN; ++r) brow[r] = rh[r] - m;
      exp_pipelined<WIN, C>(ts, rwz, brow, c);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_pready[g]);
      if (!mbar_wait(&bar_pready[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();

      // ---- A.V: warp wq issues block (wq & 1), key half (wq >> 1)
      const int s = k % S;
      if (lane == 0 && !mbar_wait(&bar_fv[k % (2 * S)], (k / (2 * S)) & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
      } else if (lane == 0) {
        const int ab = wq & 1, hf = wq >> 1;
        const int kb = hf ? C::KHALF : 0, ke = hf ? C::KSTEPS : C::KHALF;
        const uint32_t lanes = static_cast<uint32_t>(16 * ab) << 16;
        const uint32_t va = smem_addr(sStage + s * C::STAGE_BYTES + OFF_V) + ab * C::BOFF * C::ROWB;
        // B = [V | ones]: the ones atom at leading byte offset lbo, same row pitch
        const uint32_t lbo = smem_addr(sOnes) - va;
#pragma unroll 1
        for (int kk = kb; kk < ke; ++kk)
          mma_f16_ts(slot + lanes + C::O_COL + hf * C::ON, slot + lanes + 8 * kk,
                     smem_desc(va + kk * 16 * C::ROWB, lbo, C::SBO, C::SW), idO, kk != kb);
        mma_commit(&bar_ofull[g]);
        mma_commit(&bar_ev[s]);
      }
      __syncwarp();

      // ---- epilogue: O / l, bf16, NHWC
      if (!mbar_wait(&bar_ofull[g], j & 1, kWaitNs, &abort_flag)) {
        if (!abort_flag) record_timeout(&abort_flag);
        break;
      }
      tc_fence_after();
      {
        // this thread's row of both key halves' accumulators
        float o[D], la, lb;
        tmem_ld_x1(ts + C::O_COL + D, &la);
        tmem_ld_x1(ts + C::O_COL + C::ON + D, &lb);
        constexpr int kSeg = (D % 32 == 0) ? 32 : 16;  // columns per load
#pragma unroll
        for (int e = 0; e < D; e += kSeg) {
          float ta[kSeg], tb[kSeg];
          if constexpr (kSeg == 32) {
            tmem_ld_x32(ts + C::O_COL + e, ta);
            tmem_ld_x32(ts + C::O_COL + C::ON + e, tb);
          } else {
            tmem_ld_x8(ts + C::O_COL + e, ta);
            tmem_ld_x8(ts + C::O_COL + e + 8, ta + 8);
            tmem_ld_x8(ts + C::O_COL + C::ON + e, tb);
            tmem_ld_x8(ts + C::O_COL + C::ON + e + 8, tb + 8);
          }
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < kSeg; ++i) o[e + i] = ta[i] + tb[i];
        }
        const float l = la + lb;  // row sum of the bf16 P (ones columns)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_tfree[g]);
        const float inv = 1.0f / l;
        uint32_t pk[D / 2];
#pragma unroll
        for (int t = 0; t < D / 2; ++t) pk[t] = pack_bf16x2(o[2 * t] * inv, o[2 * t + 1] * inv);
        const int y = by * kBlock + qy, x = ic.bx * kBlock + qx;
        __nv_bfloat16* dst = p.out + ((static_cast<size_t>(ic.n) * p.H + y) * p.W + x) * C_all + ic.head * D;
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
          reinterpret_cast<uint4*>(dst)[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      }
    }
    // A.V MMAs this warp issued are complete before TMEM is released
    if (lane == 0) {
      mma_commit(&bar_pvdone[g]);
      mbar_wait(&bar_pvdone[g], 0, kWaitNs);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  named_bar_sync(1, kThreads);
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc4
}  // namespace halo
